// psi_scan.cu - the row scan of the sampled linear verify's streaming path
// (T > 0, every row starting on a 16-byte boundary).
//
// Sources (page title, section): "Uno Psi-Spec 是什麼？Diffusion-Augmented LLM
// 如何保留 AR 分布、一次驗證多個 Token" (alphalab.site), "Uno Psi-Spec 怎麼運作？
// 完整走一次四個 Token", steps 3-4 (p_i and q_i are the temperature softmax
// of the AR and draft rows); "想跑 Uno：先確認官方程式需要的環境" (temperature,
// top-p).
//
// What one scan leaves per logit row r (an AR or draft row of a listed unit),
// the row being split into g.slices contiguous slices of 16-byte vectors:
//   - per slice c, a record: m_c (the larger of the slice maximum and a known
//     element of the row: the drafted token's logit, or on a rescan the row
//     maximum; either way at most the row maximum) and z_c = sum of
//     exp2((x - m_c) * log2(e) / T) over the slice's elements that were not
//     set aside, summed in fp32 by a fixed thread / accumulator assignment
//     and reduced in double in a fixed order, so it is a deterministic
//     function of the slice and that known element;
//   - per slice c, its set-aside list: with top-p, every element above the
//     running threshold of its stage (the reference so far, which starts at
//     the known element, minus the top-p window, rounded down to the element
//     type), and the tail elements.  The
//     threshold of a stage is at most the row's final one, so every element
//     the top-p cut can keep is in the lists; the finish (psi_finish.cuh)
//     sorts them into candidates and the rest of the sum.
//
// Design: one CTA per SM; CTAs form groups of g.slices, CTA c of a group
// scanning slice c of each of the group's rows (rows are dealt to the groups
// round robin; the slices of a row are independent).  Warp roles:
//   producer  (one warp, one lane) keeps a ring of kStages shared-memory
//             stages filled with cp.async.bulk copies (no multicast), each
//             completing on its stage's mbarrier, and runs ahead through row
//             ends.
//   consumers (kConsumerWarps) load each stage once into registers.  Pass 1
//             takes each vector's maximum; the CTA's stage maximum is
//             combined through a per-stage mbarrier.  Pass 2 runs one stage
//             later (so that combine never stalls them): the running
//             reference becomes the row maximum so far (every exponent <= 0)
//             and the exponentials are added to fp32 accumulators (rescaled
//             when the reference rises).  With top-p, a vector holding an
//             element above the running threshold (reference minus the
//             window; the reference looks one stage ahead for it) is left out
//             of the sum whole, and its bit is set in the thread's flag byte.
//   aux       (kAuxWarps warps) take each stage after the consumers' pass
//             2: the flagged vectors are split among them by their index u
//             within the consumer thread; each warp queues its share, reads
//             those vectors again from the stage buffer (32 per round),
//             appends their elements above the threshold to the slice's
//             set-aside list in global memory (positions from a shared
//             counter: the list's order is free), adds their other elements
//             to its own fp32 sums (against the consumers' reference of the
//             stage), and hands the buffer back to the producer.  At a row
//             end aux warp 0 sets the V % 8 tail elements aside and writes
//             the slice record.  The consumers never wait on the aux warps:
//             their only effect on them is how long a buffer stays out of
//             the ring.
// Every wait is bounded: a wait that gives up sets the CTA's abort flag, every
// role then leaves its loop, and the kernel reports PSI_DEV_TIMEOUT.
#include <algorithm>

#include "psi_internal.h"

namespace psi {

namespace {

constexpr int kConsumerWarps = 8;
constexpr int kAuxWarps = 3;  // with the producer, one extra warp per SM sub-partition
constexpr int kScanWarps = kConsumerWarps + 1 + kAuxWarps;
constexpr int kScanThreads = kScanWarps * 32;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kAuxWarp0 = kConsumerWarps + 1;
constexpr int kStages = 6;
constexpr int kStageBytes = 32768;
constexpr int kStageVecs = kStageBytes / 16;
constexpr int kVecsPerThread = kStageVecs / kConsumerThreads;
constexpr int kMaxSlots = 2 * kStages;  // stage-maximum slots (see the consumer loop)
// rows whose set-aside lists the aux warps may be filling at once: an aux
// warp at stage q has every aux warp past stage q - kStages (the stage's full
// arrive needs the slot handed back by all of them), so they are at most
// kStages rows apart
constexpr int kRowSlots = 8;
static_assert(kRowSlots > kStages, "row slots cover the aux warps' spread");
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint64_t kDrainLimitNs = 100000000ull;
constexpr unsigned kSleepNs = 128;  // poll interval of the sleeping waits

static_assert(kStageVecs % kConsumerThreads == 0, "stage vectors per consumer thread");
static_assert(kConsumerWarps % 4 == 0, "stage maxima are read four at a time");
static_assert(kConsumerWarps <= 32, "queue counts are read one per lane");

// Everything per ring slot belongs to the stage in that slot: the producer
// writes the slot's row data before the stage's full arrive, the consumers
// write their queues, reference, threshold and (last stage of a row) their
// sums before the stage's fready arrive, and nobody writes them again before the
// aux warps' empty arrives hand the slot back.
struct ScanSmem {
  uint64_t full[kStages];       // stage filled (producer arrive + copy bytes)
  uint64_t fready[kStages];     // every consumer warp finished pass 2 of the stage
  uint64_t empty[kStages];      // the aux warp is done with the stage
  uint64_t maxbar[kMaxSlots];   // every consumer warp posted its stage maximum
  int32_t stage_row[kStages];   // row of the stage
  float stage_off[kStages];     // the row's candidate window
  float stage_known[kStages];   // a lower bound of the row maximum (see drafted_logit)
  float stage_ref[kStages];     // the consumers' reference for the stage
  uint32_t stage_thr[kStages];  // the stage's threshold (Threshold::pair)
  float stage_thrv[kStages];    // (Threshold::value)
  double wsum[kStages][kConsumerWarps];  // last stage of a row: each warp's sum
  __align__(16) float wmax[kMaxSlots][kConsumerWarps];
  // each consumer warp's flagged vectors of the stage (index within the
  // stage, in the warp's ballot order) and their count
  uint16_t queue[kStages][kConsumerWarps][32 * kVecsPerThread];
  int qcnt[kStages][kConsumerWarps];
  // per row slot (local row t -> t % kRowSlots): every aux warp is done with
  // the row; the length of its set-aside list; each aux warp's sum
  uint64_t rowdone[kRowSlots];
  int list_n[kRowSlots];
  double asum[kRowSlots][kAuxWarps];
  int abort;
};

constexpr size_t kScanDynSmem = (size_t)kStages * kStageBytes;

// ---- element-type helpers ----------------------------------------------------

// Candidate threshold in the element type: bf16 thresholds are rounded down,
// so rounding can only add candidates; the vector flags, the set-aside
// lists and the finish use the same test (x > value).  `pair` holds the
// threshold in both bf16 halves.
struct Threshold {
  uint32_t pair;
  float value;
};

template <typename Bits>
__device__ __forceinline__ Threshold make_threshold(float thr) {
  Threshold t;
  if constexpr (sizeof(Bits) == 2) {
    const __nv_bfloat16 h = __float2bfloat16_rd(thr);
    const __nv_bfloat162 h2 = __bfloat162bfloat162(h);
    t.pair = *reinterpret_cast<const uint32_t *>(&h2);
    t.value = __bfloat162float(h);
  } else {
    t.pair = __float_as_uint(thr);
    t.value = thr;
  }
  return t;
}

// Per-vector maximum: bf16 -> the bf16x2 of the pairwise maxima of its four
// words (two candidates); f32 -> the bits of the largest element.  NaN
// elements are ignored (they surface in the sum).
template <typename Bits>
__device__ __forceinline__ uint32_t vec_max(const uint4 &w) {
  if constexpr (sizeof(Bits) == 2) {
    const __nv_bfloat162 a = __hmax2(*reinterpret_cast<const __nv_bfloat162 *>(&w.x),
                                     *reinterpret_cast<const __nv_bfloat162 *>(&w.y));
    const __nv_bfloat162 b = __hmax2(*reinterpret_cast<const __nv_bfloat162 *>(&w.z),
                                     *reinterpret_cast<const __nv_bfloat162 *>(&w.w));
    const __nv_bfloat162 m = __hmax2(a, b);
    return *reinterpret_cast<const uint32_t *>(&m);
  } else {
    const float m = fmaxf(fmaxf(__uint_as_float(w.x), __uint_as_float(w.y)),
                          fmaxf(__uint_as_float(w.z), __uint_as_float(w.w)));
    return __float_as_uint(m);
  }
}

template <typename Bits>
__device__ __forceinline__ uint32_t max_fold(uint32_t a, uint32_t b) {
  if constexpr (sizeof(Bits) == 2) {
    const __nv_bfloat162 m = __hmax2(*reinterpret_cast<const __nv_bfloat162 *>(&a),
                                     *reinterpret_cast<const __nv_bfloat162 *>(&b));
    return *reinterpret_cast<const uint32_t *>(&m);
  } else {
    return __float_as_uint(fmaxf(__uint_as_float(a), __uint_as_float(b)));
  }
}

template <typename Bits>
__device__ __forceinline__ float max_to_float(uint32_t m) {
  if constexpr (sizeof(Bits) == 2)
    return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
  else
    return __uint_as_float(m);
}

template <typename Bits>
__device__ __forceinline__ uint32_t neg_inf_max() {
  return sizeof(Bits) == 2 ? 0xFF80FF80u : 0xFF800000u;
}

// Does a vector maximum (vec_max) exceed the threshold?
template <typename Bits>
__device__ __forceinline__ bool max_above(uint32_t m, const Threshold &t) {
  if constexpr (sizeof(Bits) == 2)
    return __hgt2_mask(*reinterpret_cast<const __nv_bfloat162 *>(&m),
                       *reinterpret_cast<const __nv_bfloat162 *>(&t.pair)) != 0u;
  else
    return __uint_as_float(m) > t.value;
}

// Adds exp2(x * coef + shift) of every element of the vector to the packed
// accumulators (a fixed assignment of elements to accumulator lanes: word q
// of a bf16 vector to acc[q], f32 element pairs to acc[0] and acc[1]).
template <typename Bits>
__device__ __forceinline__ void add_exps(const uint4 &w, float2 c2, float2 s2, float2 (&acc)[4]) {
  if constexpr (sizeof(Bits) == 2) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 x = make_float2(__uint_as_float(ws[q] << 16), __uint_as_float(ws[q] & 0xFFFF0000u));
      const float2 u = __ffma2_rn(x, c2, s2);
      acc[q] = __fadd2_rn(acc[q], make_float2(fast_exp2(u.x), fast_exp2(u.y)));
    }
  } else {
    const float2 x0 = make_float2(__uint_as_float(w.x), __uint_as_float(w.y));
    const float2 x1 = make_float2(__uint_as_float(w.z), __uint_as_float(w.w));
    const float2 u0 = __ffma2_rn(x0, c2, s2), u1 = __ffma2_rn(x1, c2, s2);
    acc[0] = __fadd2_rn(acc[0], make_float2(fast_exp2(u0.x), fast_exp2(u0.y)));
    acc[1] = __fadd2_rn(acc[1], make_float2(fast_exp2(u1.x), fast_exp2(u1.y)));
  }
}

// add_exps for a vector holding an element above the threshold: those
// elements are left out of the sum (replaced by -inf) and returned as a bit
// mask (bit e = element e).
template <typename Bits>
__device__ __forceinline__ uint32_t add_exps_masked(uint4 w, const Threshold &t, float2 c2,
                                                    float2 s2, float2 (&acc)[4]) {
  uint32_t em = 0u;
  if constexpr (sizeof(Bits) == 2) {
    const __nv_bfloat162 t2 = *reinterpret_cast<const __nv_bfloat162 *>(&t.pair);
    uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t m = __hgt2_mask(*reinterpret_cast<const __nv_bfloat162 *>(&ws[q]), t2);
      ws[q] = (ws[q] & ~m) | (0xFF80FF80u & m);
      em |= ((m & 1u) | ((m >> 15) & 2u)) << (2 * q);
    }
    w = make_uint4(ws[0], ws[1], ws[2], ws[3]);
  } else {
    uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (__uint_as_float(ws[q]) > t.value) {
        em |= 1u << q;
        ws[q] = 0xFF800000u;
      }
    w = make_uint4(ws[0], ws[1], ws[2], ws[3]);
  }
  add_exps<Bits>(w, c2, s2, acc);
  return em;
}

// Largest value over the warp (NaN ignored), by one reduction over an
// order-preserving integer image of the float.
__device__ __forceinline__ float warp_max_redux(float f) {
  if (f != f) f = -INFINITY;
  const uint32_t b = __float_as_uint(f);
  uint32_t key = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  key = __reduce_max_sync(0xFFFFFFFFu, key);
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

template <typename Bits>
__device__ __forceinline__ const Bits *scan_row_ptr(const FastArgs &a, int64_t r) {
  const int64_t nar = (int64_t)a.s.N * (a.s.B + 1);
  if (r < nar) return static_cast<const Bits *>(a.s.ar) + r * a.s.ar_stride;
  return static_cast<const Bits *>(a.s.draft) + (r - nar) * a.s.draft_stride;
}

// Row of list item `item` and its candidate window (logit units).
__device__ __forceinline__ int64_t scan_row(const FastArgs &a, int64_t item, float &off) {
  if (!a.rlist) {
    off = a.win_narrow;
    return item;
  }
  const int32_t e = a.rlist[item];
  off = (e & kWideBit) ? a.win_wide : a.win_narrow;
  return (int64_t)(e & ~kWideBit);
}

// A lower bound of row r's maximum known before the scan: the logit of the
// drafted token at the row's position (AR row i < B, or draft row i), an
// element of the row; -inf for the bonus rows and without draft ids.  A
// sampled draft token usually lies near the top of the row, so the first
// stages' set-aside threshold starts close to its final value.
template <typename Bits>
__device__ __forceinline__ float drafted_logit(const FastArgs &a, int64_t r, const Bits *row) {
  if (!a.s.ids) return -INFINITY;
  const int32_t B = a.s.B;
  const int64_t nar = (int64_t)a.s.N * (B + 1);
  int64_t n, i;
  if (r < nar) {
    n = r / (B + 1);
    i = r % (B + 1);
    if (i == B) return -INFINITY;  // the bonus row has no drafted token
  } else {
    n = (r - nar) / B;
    i = (r - nar) % B;
  }
  const int32_t x = a.s.ids[n * B + i];
  if (x < 0 || x >= a.s.V) return -INFINITY;
  return Elem<Bits>::to_float((uint32_t)row[x]);
}

// What the producer tells the consumers about a stage.
struct StageMeta {
  int slot;     // ring slot
  float off;    // candidate window of the row (logit units)
  float known;  // a lower bound of the row maximum (rescan: the maximum itself)
};

// The vectors [vb, ve) of slice c of a row; stage k covers
// [vb + k * stage_vecs, min(ve, vb + (k + 1) * stage_vecs)).
struct SliceSpan {
  int32_t vb, ve, sv;
  __device__ __forceinline__ int32_t v0(int k) const { return vb + k * sv; }
  __device__ __forceinline__ int32_t nv(int k) const {
    const int32_t a = vb + k * sv;
    return max(0, min(ve, a + sv) - a);
  }
};

// Walks this CTA's stages in order: stage k of local row t, and a ring slot
// whose phase parity flips at every wrap (no divisions on the way).
struct StageCursor {
  int64_t t = 0;
  int k = 0;
  int slot = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void advance(int K, int n_slots) {
    if (++k == K) {
      k = 0;
      ++t;
    }
    if (++slot == n_slots) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

// How a role waits between tests of an mbarrier phase.
enum class Wait {
  kSpin,     // consumers: test again at once
  kSleep,    // producer: sleep kSleepNs between tests, leaving issue slots to the consumers
  kSuspend,  // aux: the hardware may suspend the warp until the phase completes
};

// Bounded wait for an mbarrier phase.  False when it gave up (the abort flag
// is then set) or when another role already gave up.
template <Wait kMode>
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, int *abort,
                                           uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (kMode == Wait::kSleep) __nanosleep(kSleepNs);
    const bool done =
        kMode == Wait::kSuspend ? mbar_try_wait(bar, parity, 1000u) : mbar_test(bar, parity);
    if (done) return true;
    if (kMode != Wait::kSpin || (it & 15u) == 0u) {
      if (*(volatile int *)abort) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *(volatile int *)abort = 1;
        return false;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// row_scan_kernel
// ---------------------------------------------------------------------------
template <typename Bits, int C>
__global__ void __launch_bounds__(kScanThreads, 1) row_scan_kernel(const __grid_constant__ FastArgs a) {
  pdl_wait();  // the previous kernel's results are visible
  pdl_trigger();
  constexpr int VEC = Elem<Bits>::kVec;
  constexpr int U = kVecsPerThread;
  extern __shared__ __align__(128) unsigned char scan_dsm[];
  __shared__ ScanSmem sm;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const ScanGeom &g = a.g;
  const int c = C > 1 ? (int)(blockIdx.x % C) : 0;  // the slice this CTA scans
  const int64_t cl = blockIdx.x / C, n_cl = gridDim.x / C;
  const int64_t R = a.rlist ? (int64_t)*a.rcount : a.rows;
  const int64_t my_rows = R > cl ? (R - 1 - cl) / n_cl + 1 : 0;
  if (my_rows == 0) return;
  const int K = g.stages;
  const int64_t Q = my_rows * K;  // stages this CTA scans
  const float coef = a.coef;
  const uint32_t stage0 = smem_addr(scan_dsm);
  SliceSpan span;
  span.vb = (int32_t)(((int64_t)c * g.nvec) / C);
  span.ve = (int32_t)(((int64_t)(c + 1) * g.nvec) / C);
  span.sv = g.stage_vecs;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.fready[i], kConsumerWarps);
      mbar_init(&sm.empty[i], kAuxWarps);
    }
    for (int i = 0; i < kMaxSlots; ++i) mbar_init(&sm.maxbar[i], kConsumerWarps);
    for (int i = 0; i < kRowSlots; ++i) {
      mbar_init(&sm.rowdone[i], kAuxWarps);
      sm.list_n[i] = 0;
    }
    sm.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kProducerWarp) {
    // ---- producer: one lane issues the bulk copies
    if (lane == 0) {
      int64_t issued = 0;
      StageCursor cur;
      const Bits *row = nullptr;
      int64_t r = 0;
      float off = 0.f, known = -INFINITY;
      for (int64_t q = 0; q < Q; ++q, cur.advance(K, kStages)) {
        // the aux warp is done with the slot's previous stage (q - kStages)
        if (q >= kStages &&
            !wait_phase<Wait::kSleep>(&sm.empty[cur.slot], cur.phase ^ 1u, &sm.abort))
          break;
        if (cur.k == 0) {
          r = scan_row(a, cl + cur.t * n_cl, off);
          row = scan_row_ptr<Bits>(a, r);
          known = a.pass == 2 ? a.known_max[r] : -INFINITY;
          known = fmaxf(known, drafted_logit<Bits>(a, r, row));
        }
        sm.stage_row[cur.slot] = (int32_t)r;
        sm.stage_off[cur.slot] = off;
        sm.stage_known[cur.slot] = known;
        const int32_t nv = span.nv(cur.k);
        if (nv > 0) {
          mbar_arrive_expect_tx(&sm.full[cur.slot], (uint32_t)nv * 16u);
          bulk_load(scan_dsm + (size_t)cur.slot * kStageBytes,
                    reinterpret_cast<const uint4 *>(row) + span.v0(cur.k), (uint32_t)nv * 16u,
                    &sm.full[cur.slot]);
        } else {
          mbar_arrive(&sm.full[cur.slot]);
        }
        issued = q + 1;
      }
      // copies still in flight must land before this CTA may exit (on the
      // normal path the consumers have already waited for every one)
      for (int64_t q = issued > kStages ? issued - kStages : 0; q < issued; ++q) {
        int never = 0;
        wait_phase<Wait::kSpin>(&sm.full[q % kStages], (uint32_t)((q / kStages) & 1), &never,
                                kDrainLimitNs);
      }
    }
    __syncwarp();
  } else if (warp >= kAuxWarp0) {
    // ---- aux: each warp takes the flagged vectors of its class of every
    // stage, then hands the buffer back; aux warp 0 closes each row (tail
    // elements, slice record) once every aux warp is done with it
    const int aw = warp - kAuxWarp0;
    StageCursor ac;
    float aref = -INFINITY;  // the reference of this warp's sums
    float2 acc[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
    int64_t r = 0;
    uint64_t *list = nullptr;
    for (int64_t q = 0; q < Q; ++q, ac.advance(K, kStages)) {
      bool ok = wait_phase<Wait::kSuspend>(&sm.fready[ac.slot], ac.phase, &sm.abort);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      const int slot = ac.slot, k = ac.k;
      const int rs = (int)(ac.t % kRowSlots);
      const float sref = sm.stage_ref[slot];
      if (k == 0) {
        r = sm.stage_row[slot];
        list = a.cand + r * (int64_t)kCandCap + (int64_t)c * g.cap;
        aref = sref;
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[u] = make_float2(0.f, 0.f);
      } else if (sref > aref) {
        const float f = (aref == -INFINITY) ? 0.f : fast_exp2((aref - sref) * coef);
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[u] = make_float2(acc[u].x * f, acc[u].y * f);
        aref = sref;
      }
      if (a.use_window) {
        Threshold th;
        th.pair = sm.stage_thr[slot];
        th.value = sm.stage_thrv[slot];
        // the consumer warps' queues, one after the other: entry i of the
        // stage goes to aux warp (i / 32) % kAuxWarps
        int end[kConsumerWarps];  // running ends of the queues
        int n = 0;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          n += sm.qcnt[slot][w];
          end[w] = n;
        }
        const float shift = (aref == -INFINITY) ? 0.f : -aref * coef;
        const float2 c2 = make_float2(coef, coef), s2 = make_float2(shift, shift);
        const uint32_t base = stage0 + (uint32_t)slot * kStageBytes;
        const uint32_t v0 = (uint32_t)span.v0(k);
        for (int i = aw * 32 + lane; i - lane < n; i += kAuxWarps * 32) {
          if (i < n) {
            int w = 0, start = 0;
#pragma unroll
            for (int x = 0; x < kConsumerWarps - 1; ++x)
              if (i >= end[x]) {
                w = x + 1;
                start = end[x];
              }
            const uint32_t j = sm.queue[slot][w][i - start];
            const uint4 v = lds128(base + j * 16u);
            const uint32_t em = add_exps_masked<Bits>(v, th, c2, s2, acc);
            const int pos = atomicAdd(&sm.list_n[rs], __popc(em));
            const uint32_t idx0 = (v0 + j) * VEC;
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
              const int p = pos + __popc(em & ((1u << e) - 1u));
              if (((em >> e) & 1u) && p < g.cap)
                list[p] = ((uint64_t)vec_elem<Bits>(v, e) << 32) | (idx0 + (uint32_t)e);
            }
          }
        }
      }
      if (k == K - 1) {  // the row's last stage
        double zl = 0.0;
#pragma unroll
        for (int u = 0; u < 4; ++u) zl += (double)acc[u].x + (double)acc[u].y;
        const double za = warp_sum_d(zl);  // relative to sref, as the consumers' sums
        if (lane == 0) {
          sm.asum[rs][aw] = za;
          __threadfence_block();
          mbar_arrive(&sm.rowdone[rs]);
        }
        if (aw == 0) {  // every aux warp's list entries and sum, then the record
          ok = wait_phase<Wait::kSuspend>(&sm.rowdone[rs], (uint32_t)((ac.t / kRowSlots) & 1),
                                          &sm.abort);
          if (!__all_sync(0xFFFFFFFFu, ok)) break;
          double zc = 0.0;
#pragma unroll
          for (int w = 0; w < kAuxWarps; ++w) zc += sm.asum[rs][w];
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) zc += sm.wsum[slot][w];
          int n_list = sm.list_n[rs];
          // the V % VEC elements after the last whole vector (last slice;
          // plain loads) are all set aside: the finish sorts them with the
          // others
          const bool has_tail = c == C - 1 && lane < g.tail;
          const Bits *row = scan_row_ptr<Bits>(a, r);
          const uint32_t tbits = has_tail ? (uint32_t)row[(int64_t)g.nvec * VEC + lane]
                                          : (uint32_t)Elem<Bits>::kNegInf;
          const float mc = fmaxf(sref, warp_max(Elem<Bits>::to_float(tbits)));  // slice maximum
          if (has_tail && n_list + lane < g.cap)
            list[n_list + lane] = ((uint64_t)tbits << 32) | (uint32_t)(g.nvec * VEC + lane);
          if (c == C - 1) n_list += g.tail;
          __syncwarp();
          if (lane == 0) {
            SliceRecord rec;
            rec.m = mc;
            rec.n_cand = n_list;
            rec.flags = n_list > g.cap ? kRowLost : 0;
            rec.off = sm.stage_off[slot];
            rec.z = (sref == -INFINITY || !(mc > sref))
                        ? zc
                        : zc * exp2(((double)sref - (double)mc) * a.coef64);
            a.srec[r * kMaxSlices + c] = rec;
            sm.list_n[rs] = 0;  // reused kRowSlots rows later
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
    }
  } else {
    // ---- consumers
    const int cw = warp, ct = tid;
    uint4 neg;
    neg.x = neg.y = neg.z = neg.w = neg_inf_max<Bits>();
    bool dead = false;
    // per-row state (the same in every consumer thread except the sums)
    float ref = -INFINITY, off = 0.f;
    float2 acc[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);

    // next stage to load (ring slot, full-barrier phase), its stage-maximum
    // slot, and the next stage for pass 2 (stage-maximum slot and phase)
    StageCursor lc, pc;
    int lms = 0;

    // a stage: registers <- shared memory, then the warp's maximum to the
    // stage's maximum slot.  A maximum slot is reused 2 * kStages stages
    // later; by then every consumer warp has read the old one (the stage
    // kStages later can only be loaded once the aux warp has handed its
    // buffer back, which it does after every warp's pass 2 of that stage).
    auto load_stage = [&](uint4(&Rv)[U], uint32_t(&Tm)[U], StageMeta &Mt) {
      bool ok = wait_phase<Wait::kSpin>(&sm.full[lc.slot], lc.phase, &sm.abort);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        dead = true;
        return;
      }
      const int32_t nv = span.nv(lc.k);
      const uint32_t base = stage0 + (uint32_t)lc.slot * kStageBytes;
      Mt.slot = lc.slot;
      Mt.off = sm.stage_off[lc.slot];
      Mt.known = sm.stage_known[lc.slot];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = ct + u * kConsumerThreads;
        Rv[u] = (nv == kStageVecs || j < nv) ? lds128(base + (uint32_t)j * 16u) : neg;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) Tm[u] = vec_max<Bits>(Rv[u]);
      uint32_t run[U];  // the stage maximum, folded as a tree
#pragma unroll
      for (int u = 0; u < U; ++u) run[u] = Tm[u];
#pragma unroll
      for (int h = 1; h < U; h <<= 1)
#pragma unroll
        for (int u = 0; u + h < U; u += 2 * h) run[u] = max_fold<Bits>(run[u], run[u + h]);
      const float wm = warp_max_redux(max_to_float<Bits>(run[0]));
      if (lane == 0) sm.wmax[lms][cw] = wm;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.maxbar[lms]);
      lc.advance(K, kStages);
      if (++lms == kMaxSlots) lms = 0;
    };

    // a stage from registers: reference, exponentials, flags
    auto pass2 = [&](const uint4(&Rv)[U], const uint32_t(&Tm)[U], const StageMeta &Mt) {
      const int ms = pc.slot;
      bool ok = wait_phase<Wait::kSpin>(&sm.maxbar[ms], pc.phase, &sm.abort);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        dead = true;
        return;
      }
      float smax = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; w += 4) {
        const float4 m4 = *reinterpret_cast<const float4 *>(&sm.wmax[ms][w]);
        smax = fmaxf(fmaxf(smax, fmaxf(m4.x, m4.y)), fmaxf(m4.z, m4.w));
      }
      const int k = pc.k;
      pc.advance(K, kMaxSlots);
      if (k == 0) {  // first stage of a row
        off = Mt.off;
        ref = fmaxf(smax, Mt.known);
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
      } else if (smax > ref) {
        const float f = (ref == -INFINITY) ? 0.f : fast_exp2((ref - smax) * coef);
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] = make_float2(acc[q].x * f, acc[q].y * f);
        ref = smax;
      }
      const float shift = (ref == -INFINITY) ? 0.f : -ref * coef;
      const float2 c2 = make_float2(coef, coef), s2 = make_float2(shift, shift);
      if (a.use_window) {
        // the set-aside threshold looks one stage ahead within the row (every
        // warp posted the next stage's maximum when it loaded that stage,
        // which it did before this pass): a higher threshold flags fewer
        // vectors
        float thr_ref = ref;
        if (k + 1 < K) {
          ok = wait_phase<Wait::kSpin>(&sm.maxbar[pc.slot], pc.phase, &sm.abort);
          if (!__all_sync(0xFFFFFFFFu, ok)) {
            dead = true;
            return;
          }
#pragma unroll
          for (int w = 0; w < kConsumerWarps; w += 4) {
            const float4 m4 = *reinterpret_cast<const float4 *>(&sm.wmax[pc.slot][w]);
            thr_ref = fmaxf(fmaxf(thr_ref, fmaxf(m4.x, m4.y)), fmaxf(m4.z, m4.w));
          }
        }
        const Threshold th = make_threshold<Bits>(thr_ref - off);
        // a vector with an element above the threshold stays out of this sum
        // whole; the warp queues it for the aux warps (one ballot per u)
        uint32_t fl = 0u;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const bool f = max_above<Bits>(Tm[u], th);
          fl |= (f ? 1u : 0u) << u;
          add_exps<Bits>(f ? neg : Rv[u], c2, s2, acc);
        }
        int nq = 0;
        if (__any_sync(0xFFFFFFFFu, fl != 0u)) {
          uint16_t *qw = sm.queue[Mt.slot][cw];
          const unsigned below = (1u << lane) - 1u;
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const bool f = (fl >> u) & 1u;
            const unsigned bal = __ballot_sync(0xFFFFFFFFu, f);
            if (f) qw[nq + __popc(bal & below)] = (uint16_t)(ct + u * kConsumerThreads);
            nq += __popc(bal);
          }
        }
        if (lane == 0) sm.qcnt[Mt.slot][cw] = nq;
        if (ct == 0) {
          sm.stage_thr[Mt.slot] = th.pair;
          sm.stage_thrv[Mt.slot] = th.value;
        }
      } else {
#pragma unroll
        for (int u = 0; u < U; ++u) add_exps<Bits>(Rv[u], c2, s2, acc);
      }
      if (ct == 0) sm.stage_ref[Mt.slot] = ref;
      if (k == K - 1) {  // end of the row: this warp's sum
        double zl = 0.0;
#pragma unroll
        for (int q = 0; q < 4; ++q) zl += (double)acc[q].x + (double)acc[q].y;
        const double zs = warp_sum_d(zl);
        if (lane == 0) sm.wsum[Mt.slot][cw] = zs;
      }
      __threadfence_block();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.fready[Mt.slot]);
    };

    uint4 R0[U], R1[U];
    uint32_t T0[U], T1[U];
    StageMeta M0, M1;
    // pass 2 of a stage runs after the next stage's load (two register sets)
    for (int64_t q = 0; q <= Q && !dead; q += 2) {
      if (q < Q) load_stage(R0, T0, M0);
      if (dead) break;
      if (q >= 1) pass2(R1, T1, M1);
      if (dead || q + 1 > Q) break;
      if (q + 1 < Q) load_stage(R1, T1, M1);
      if (dead) break;
      pass2(R0, T0, M0);
    }
  }

  if (tid == 0 && *(volatile int *)&sm.abort && a.s.dev_status)
    atomicOr(a.s.dev_status, PSI_DEV_TIMEOUT);
}

template <typename Bits, int C>
cudaError_t launch_scan_typed(const FastArgs &fa, cudaStream_t stream) {
  static DeviceOnce configure;
  cudaError_t e = configure([] {
    cudaError_t err = cudaFuncSetAttribute(row_scan_kernel<Bits, C>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)kScanDynSmem);
    if (err == cudaSuccess) err = prefer_max_shared(row_scan_kernel<Bits, C>);
    return err;
  });
  if (e != cudaSuccess) return e;
  // one CTA per SM: groups of C CTAs, each group scanning its rows' C slices
  const int64_t groups =
      std::min<int64_t>(std::max(1, device_sm_count() / C), std::max<int64_t>(fa.rows, 1));
  return launch_pdl(row_scan_kernel<Bits, C>, dim3((unsigned)(groups * C)), dim3(kScanThreads),
                    kScanDynSmem, stream, fa);
}

template <typename Bits>
cudaError_t launch_scan_bits(const FastArgs &fa, cudaStream_t stream) {
  switch (fa.g.slices) {
    case 1: return launch_scan_typed<Bits, 1>(fa, stream);
    case 2: return launch_scan_typed<Bits, 2>(fa, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

ScanGeom plan_scan(int32_t V, int elem_bytes) {
  ScanGeom g;
  const int32_t vec = 16 / elem_bytes;
  g.nvec = V / vec;
  g.tail = V - g.nvec * vec;
  // rows of at least four stages are split in two slices (two CTAs)
  g.slices = (int64_t)g.nvec * 16 >= 4 * (int64_t)kStageBytes ? 2 : 1;
  const int32_t per = (g.nvec + g.slices - 1) / g.slices;
  g.stages = std::max<int32_t>(1, (per + kStageVecs - 1) / kStageVecs);
  g.stage_vecs = std::min<int32_t>(per, kStageVecs);  // full stages, then the rest
  g.cap = kCandCap / g.slices;
  return g;
}

cudaError_t launch_row_scan(const FastArgs &fa, psi_dtype dtype, cudaStream_t stream) {
  if (dtype == PSI_DTYPE_BF16) return launch_scan_bits<uint16_t>(fa, stream);
  return launch_scan_bits<uint32_t>(fa, stream);
}

}  // namespace psi
