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
//   - per slice c, a record: m_c (the slice maximum; on a rescan the known row
//     maximum) and z_c = sum over the slice of exp2((x - m_c) * log2(e) / T),
//     summed in fp32 by a fixed thread / accumulator assignment and reduced in
//     double in a fixed order, so it is a deterministic function of the slice;
//   - per slice c, its candidates: every element x > thr, where thr is the
//     row maximum minus the top-p window, rounded down to the element type.
//     Every element the top-p cut can keep is a candidate (the window holds
//     at least top_p of the mass, which the finish checks), and no other
//     element is.
//
// Design: one CTA per SM, clusters of g.slices CTAs; CTA `rank` of a cluster
// scans slice `rank` of each of the cluster's rows (rows are dealt to the
// clusters round robin).  Warp roles:
//   producer  (one warp, one lane) keeps a ring of kStages shared-memory
//             stages filled with cp.async.bulk copies (no multicast), each
//             completing on its stage's mbarrier, and runs ahead through row
//             ends.
//   consumers (kConsumerWarps) load each stage once into registers and hand
//             the buffer back at once.  Pass 1 takes each vector's maximum;
//             the CTA's stage maximum is combined through a per-stage
//             mbarrier.  Pass 2 runs one stage later (so that combine never
//             stalls them): the running reference becomes the row maximum so
//             far (every exponent <= 0), the exponentials are added to fp32
//             accumulators (rescaled when the reference rises), and the
//             elements above the running threshold are parked in a
//             shared-memory list for the row.
//   row end   (one warp) adds the V % 8 tail elements, exchanges the slice
//             maximum with the cluster's other CTAs over DSMEM (a store into
//             each CTA's shared memory and a remote mbarrier arrive), filters
//             the parked elements against the row's final threshold into the
//             slice's candidate list in global memory and writes the slice
//             record, off the consumers' path.
// Every wait is bounded: a wait that gives up sets the CTA's abort flag, every
// role then leaves its loop, and the kernel reports PSI_DEV_TIMEOUT.
#include <algorithm>

#include "psi_internal.h"

namespace psi {

namespace {

constexpr int kConsumerWarps = 8;
constexpr int kRowEndWarps = 2;  // row t is finished by row-end warp t % 2
constexpr int kScanWarps = kConsumerWarps + 1 + kRowEndWarps;
constexpr int kScanThreads = kScanWarps * 32;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kRowEndWarp0 = kConsumerWarps + 1;
constexpr int kStages = 5;
constexpr int kStageBytes = 32768;
constexpr int kStageVecs = kStageBytes / 16;
constexpr int kVecsPerThread = kStageVecs / kConsumerThreads;
constexpr int kMaxSlots = 2 * kStages;  // stage-maximum slots (see the consumer loop)
constexpr int kParkSlots = kRowEndWarps;  // rows whose set-aside vectors await a row-end warp
constexpr int kParkCap = 1536;            // set-aside vectors per row and slice
constexpr int kXSlots = 2 * kRowEndWarps; // slice-maximum exchange slots (see the row-end warps)
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint64_t kDrainLimitNs = 100000000ull;
constexpr unsigned kSleepNs = 128;  // poll interval of the sleeping waits

static_assert(kStageVecs % kConsumerThreads == 0, "stage vectors per consumer thread");
static_assert(kConsumerWarps % 4 == 0, "stage maxima are read four at a time");

struct ScanSmem {
  uint64_t full[kStages];       // stage filled (producer arrive + copy bytes)
  uint64_t empty[kStages];      // stage read by every consumer warp
  uint64_t maxbar[kMaxSlots];   // every consumer warp posted its stage maximum
  uint64_t rowbar[kParkSlots];  // every consumer warp finished the row
  uint64_t parkfree[kParkSlots];// the row-end warp is done with the row's parked list
  uint64_t xbar[kXSlots];       // slice maxima of a row arrived from every CTA of the cluster
  int32_t stage_row[kStages];   // row of the stage in the slot (written before its full arrive)
  float stage_off[kStages];     // the row's candidate window
  float stage_known[kStages];   // rescan: the row maximum found by the first pass
  int32_t park_row[kParkSlots]; // row handed to the row-end warp
  float park_off[kParkSlots];
  double wsum[kParkSlots][kConsumerWarps];
  __align__(16) float wmax[kMaxSlots][kConsumerWarps];
  float sref[kParkSlots];
  float xmax[kXSlots][kMaxSlices];
  int park_count[kParkSlots];
  int abort;
};

constexpr size_t kScanDynSmem = (size_t)kStages * kStageBytes +
                                (size_t)kParkSlots * kParkCap * (sizeof(uint4) + sizeof(uint32_t));

// ---- element-type helpers ----------------------------------------------------

// Candidate threshold in the element type: bf16 thresholds are rounded down,
// so rounding can only add candidates; parking and filtering use the same
// test (x > value).  `pair` holds the threshold in both bf16 halves.
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

__device__ __forceinline__ Threshold no_threshold() {  // nothing is above it
  Threshold t;
  t.pair = 0x7F807F80u;  // bf16x2 (+inf, +inf)
  t.value = INFINITY;
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

// Bit q set iff element q of the vector is above the threshold.
template <typename Bits>
__device__ __forceinline__ uint32_t above_mask(const uint4 &w, const Threshold &t) {
  if constexpr (sizeof(Bits) == 2) {
    const __nv_bfloat162 t2 = *reinterpret_cast<const __nv_bfloat162 *>(&t.pair);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    uint32_t mask = 0u;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t m = __hgt2_mask(*reinterpret_cast<const __nv_bfloat162 *>(&ws[q]), t2);
      mask |= ((m & 1u) | ((m >> 15) & 2u)) << (2 * q);
    }
    return mask;
  } else {
    return (__uint_as_float(w.x) > t.value ? 1u : 0u) | (__uint_as_float(w.y) > t.value ? 2u : 0u) |
           (__uint_as_float(w.z) > t.value ? 4u : 0u) | (__uint_as_float(w.w) > t.value ? 8u : 0u);
  }
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

// What the producer tells the consumers about a stage.
struct StageMeta {
  int32_t r;    // row
  float off;    // candidate window of the row (logit units)
  float known;  // rescan: the row maximum found by the first pass, else -inf
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

// Bounded wait for an mbarrier phase.  False when it gave up (the abort flag
// is then set) or when another role already gave up.  Roles off the
// consumers' path (producer, row end) wait with kSleep: between tests they
// sleep, so that their polling does not take issue slots from the consumer
// warps that share their scheduler.
template <bool kClusterScope, bool kSleep = false>
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, int *abort,
                                           uint64_t limit_ns = kWaitLimitNs) {
  if (kClusterScope ? mbar_test_cluster(bar, parity) : mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (kSleep) __nanosleep(kSleepNs);
    if (kClusterScope ? mbar_test_cluster(bar, parity) : mbar_test(bar, parity)) return true;
    if (kSleep || (it & 15u) == 0u) {
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
  constexpr int VEC = Elem<Bits>::kVec;
  constexpr int U = kVecsPerThread;
  extern __shared__ __align__(128) unsigned char scan_dsm[];
  __shared__ ScanSmem sm;
  // set-aside vectors of a row: copies and their indices in the row
  uint4 *park_vec = reinterpret_cast<uint4 *>(scan_dsm + (size_t)kStages * kStageBytes);
  uint32_t *park_idx = reinterpret_cast<uint32_t *>(park_vec + (size_t)kParkSlots * kParkCap);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const ScanGeom &g = a.g;
  const int c = C > 1 ? (int)(blockIdx.x % C) : 0;  // == %cluster_ctarank for 1-D clusters
  const int64_t cl = blockIdx.x / C, n_cl = gridDim.x / C;
  const int64_t R = a.rlist ? (int64_t)*a.rcount : a.rows;
  const int64_t my_rows = R > cl ? (R - 1 - cl) / n_cl + 1 : 0;
  if (my_rows == 0) return;  // the same for every CTA of the cluster
  const int K = g.stages;
  const int64_t Q = my_rows * K;  // stages this CTA scans
  const float coef = a.coef;
  SliceSpan span;
  span.vb = (int32_t)(((int64_t)c * g.nvec) / C);
  span.ve = (int32_t)(((int64_t)(c + 1) * g.nvec) / C);
  span.sv = g.stage_vecs;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], kConsumerWarps);
    }
    for (int i = 0; i < kMaxSlots; ++i) mbar_init(&sm.maxbar[i], kConsumerWarps);
    for (int i = 0; i < kParkSlots; ++i) {
      mbar_init(&sm.rowbar[i], kConsumerWarps);
      mbar_init(&sm.parkfree[i], 1);
      sm.park_count[i] = 0;
    }
    for (int i = 0; i < kXSlots; ++i) mbar_init(&sm.xbar[i], C);
    sm.abort = 0;
    fence_mbar_init();
  }
  if constexpr (C > 1)
    cluster_sync();  // every CTA's barriers exist before any remote arrive
  else
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
        // the slot's previous stage (q - kStages) has been read by every consumer
        if (q >= kStages &&
            !wait_phase<false, true>(&sm.empty[cur.slot], cur.phase ^ 1u, &sm.abort))
          break;
        if (cur.k == 0) {
          r = scan_row(a, cl + cur.t * n_cl, off);
          row = scan_row_ptr<Bits>(a, r);
          known = a.pass == 2 ? a.known_max[r] : -INFINITY;
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
        wait_phase<false>(&sm.full[q % kStages], (uint32_t)((q / kStages) & 1), &never,
                          kDrainLimitNs);
      }
    }
    __syncwarp();
  } else if (warp >= kRowEndWarp0) {
    // ---- row end: tail, cluster exchange, final split, slice record.  Row-end
    // warp e takes rows e, e + 2, ... (parking slot e).  Its exchange slots are
    // e and e + 2 (t % 4): a CTA sends row t + 4's maximum only after it
    // received every peer's maximum of row t + 2, which each peer sent after
    // it had read its slot for row t.
    const int e_warp = warp - kRowEndWarp0;
    for (int64_t t = e_warp; t < my_rows; t += kRowEndWarps) {
      const int s = (int)(t % kParkSlots);
      bool ok =
          wait_phase<false, true>(&sm.rowbar[s], (uint32_t)((t / kParkSlots) & 1), &sm.abort);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      const int64_t r = sm.park_row[s];
      const float off = sm.park_off[s];
      const float ref = sm.sref[s];  // maximum over the slice's whole vectors
      double zc = 0.0;  // the consumers' sums, relative to ref
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) zc += sm.wsum[s][w];
      const int n_park = sm.park_count[s];
      const int n = min(n_park, kParkCap);
      const uint4 *pv = park_vec + (size_t)s * kParkCap;
      const uint32_t *pi = park_idx + (size_t)s * kParkCap;
      const Bits *row = scan_row_ptr<Bits>(a, r);
      // the V % VEC elements after the last whole vector (last slice; plain loads)
      const bool has_tail = c == C - 1 && lane < g.tail;
      const uint32_t tbits =
          has_tail ? (uint32_t)row[(int64_t)g.nvec * VEC + lane] : (uint32_t)Elem<Bits>::kNegInf;
      const float tx = Elem<Bits>::to_float(tbits);
      const float mc = fmaxf(ref, warp_max(tx));  // the slice maximum
      float M = mc;
      if constexpr (C > 1) {  // the row maximum, from every CTA of the cluster
        const int s2 = (int)(t % kXSlots);
        if (lane == 0) {
#pragma unroll
          for (int p = 0; p < C; ++p) {
            dsmem_st_f32(dsmem_map(&sm.xmax[s2][c], (uint32_t)p), mc);
            mbar_arrive_remote(dsmem_map(&sm.xbar[s2], (uint32_t)p));
          }
        }
        ok = wait_phase<true, true>(&sm.xbar[s2], (uint32_t)((t / kXSlots) & 1), &sm.abort);
        if (!__all_sync(0xFFFFFFFFu, ok)) break;
#pragma unroll
        for (int p = 0; p < C; ++p) M = fmaxf(M, sm.xmax[s2][p]);
      }
      const Threshold thf = a.use_top_p ? make_threshold<Bits>(M - off) : no_threshold();
      // the set-aside vectors (copies in shared memory) and the tail: elements
      // above the final threshold are the slice's candidates, the others join
      // the sum, in 2^48 fixed point relative to mc (order-free)
      const float shc = (mc == -INFINITY) ? 0.f : -mc * coef;
      uint64_t *dst = a.cand + r * (int64_t)kCandCap + (int64_t)c * g.cap;
      unsigned long long tfx = 0ull;
      int pos = 0;
      for (int base = 0; base < n; base += 32) {
        const int j = base + lane;
        const uint32_t vi = j < n ? pi[j] : 0u;
        uint4 w;
        w.x = w.y = w.z = w.w = neg_inf_max<Bits>();
        if (j < n) w = pv[j];
        const uint32_t cm = above_mask<Bits>(w, thf);
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const float ex = fast_exp2(fmaf(Elem<Bits>::to_float(vec_elem<Bits>(w, e)), coef, shc));
          if (!((cm >> e) & 1u) && ex > 0.f) tfx += __float2ull_rn(ex * 281474976710656.0f);
        }
        int cnt = __popc(cm), incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += v;
        }
        int d = pos + incl - cnt;
        uint32_t m = cm;
        while (m) {
          const int e = __ffs(m) - 1;
          m &= m - 1;
          if (d < g.cap) dst[d] = ((uint64_t)vec_elem<Bits>(w, e) << 32) | (vi * VEC + (uint32_t)e);
          ++d;
        }
        pos += __shfl_sync(0xFFFFFFFFu, incl, 31);
      }
      {
        const bool cand = has_tail && tx > thf.value;
        const unsigned bal = __ballot_sync(0xFFFFFFFFu, cand);
        const int d = pos + __popc(bal & ((1u << lane) - 1u));
        if (cand && d < g.cap) dst[d] = ((uint64_t)tbits << 32) | (uint32_t)(g.nvec * VEC + lane);
        pos += __popc(bal);
      }
      // every element that is not a candidate, relative to mc: the consumers'
      // sums (rescaled if the tail holds the maximum), the tail, the rest
      double z = (ref == -INFINITY || !(mc > ref)) ? zc : zc * exp2(((double)ref - (double)mc) * a.coef64);
      const double et = (has_tail && !(tx > thf.value) && mc > -INFINITY)
                            ? exp2(((double)tx - (double)mc) * a.coef64)
                            : 0.0;
      z += warp_sum_d(et);
      z += (double)warp_sum_u64(tfx) * (1.0 / 281474976710656.0);
      if (lane == 0) {
        SliceRecord rec;
        rec.m = mc;
        rec.n_cand = pos;
        rec.flags = n_park > kParkCap ? kRowLost : 0;
        rec.n_parked = n_park;
        rec.z = (ref == -INFINITY && mc == -INFINITY) ? 0.0 : z;
        a.srec[r * kMaxSlices + c] = rec;
        sm.park_count[s] = 0;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.parkfree[s]);
    }
  } else {
    // ---- consumers
    const int cw = warp, ct = tid;
    const uint32_t stage0 = smem_addr(scan_dsm);
    uint4 neg;
    neg.x = neg.y = neg.z = neg.w = neg_inf_max<Bits>();
    bool dead = false;
    // per-row state (the same in every consumer thread except the sums)
    float ref = -INFINITY, off = 0.f;
    int64_t r = 0;
    float2 acc[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);

    // next stage to load (ring slot, full-barrier phase), its stage-maximum
    // slot, and the next stage for pass 2 (stage-maximum slot and phase)
    StageCursor lc, pc;
    int lms = 0;

    // a stage: registers <- shared memory, then the warp's maximum to the
    // stage's maximum slot, then the buffer back to the producer.  A maximum
    // slot is reused 2 * kStages stages later; by then every consumer warp
    // has read the old one (the producer refilled the stage buffer in
    // between only after every warp released it, i.e. finished pass 2 of the
    // stage before).
    auto load_stage = [&](uint4(&Rv)[U], uint32_t(&Tm)[U], StageMeta &Mt) {
      bool ok = wait_phase<false>(&sm.full[lc.slot], lc.phase, &sm.abort);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        dead = true;
        return;
      }
      const int32_t nv = span.nv(lc.k);
      const uint32_t base = stage0 + (uint32_t)lc.slot * kStageBytes;
      Mt.r = sm.stage_row[lc.slot];
      Mt.off = sm.stage_off[lc.slot];
      Mt.known = sm.stage_known[lc.slot];
      uint32_t run = neg_inf_max<Bits>();
      if (nv == kStageVecs) {
#pragma unroll
        for (int u = 0; u < U; ++u) Rv[u] = lds128(base + (uint32_t)(ct + u * kConsumerThreads) * 16u);
      } else {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int j = ct + u * kConsumerThreads;
          Rv[u] = j < nv ? lds128(base + (uint32_t)j * 16u) : neg;
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        Tm[u] = vec_max<Bits>(Rv[u]);
        run = max_fold<Bits>(run, Tm[u]);
      }
      const float wm = warp_max_redux(max_to_float<Bits>(run));
      if (lane == 0) sm.wmax[lms][cw] = wm;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.maxbar[lms]);
        mbar_arrive(&sm.empty[lc.slot]);
      }
      lc.advance(K, kStages);
      if (++lms == kMaxSlots) lms = 0;
    };

    // a stage from registers: reference, exponentials, parked elements
    auto pass2 = [&](const uint4(&Rv)[U], const uint32_t(&Tm)[U], const StageMeta &Mt) {
      const int ms = pc.slot;
      bool ok = wait_phase<false>(&sm.maxbar[ms], pc.phase, &sm.abort);
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
      const int64_t t = pc.t;
      const int k = pc.k;
      pc.advance(K, kMaxSlots);
      const int s = (int)(t % kParkSlots);
      if (k == 0) {  // first stage of a row
        r = Mt.r;
        off = Mt.off;
        ref = fmaxf(smax, Mt.known);
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
        if (t >= kParkSlots) {  // the row-end warp is done with this parking slot
          ok = wait_phase<false>(&sm.parkfree[s], (uint32_t)((t / kParkSlots - 1) & 1), &sm.abort);
          if (!__all_sync(0xFFFFFFFFu, ok)) {
            dead = true;
            return;
          }
        }
      } else if (smax > ref) {
        const float f = (ref == -INFINITY) ? 0.f : fast_exp2((ref - smax) * coef);
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] = make_float2(acc[q].x * f, acc[q].y * f);
        ref = smax;
      }
      const float shift = (ref == -INFINITY) ? 0.f : -ref * coef;
      const float2 c2 = make_float2(coef, coef), s2 = make_float2(shift, shift);
      const float2 s_off = make_float2(-INFINITY, -INFINITY);
      const Threshold th = a.use_top_p ? make_threshold<Bits>(ref - off) : no_threshold();
      // a vector holding an element above the running threshold is left out
      // of the fp32 sum (its shift makes every exponential 0; NaN and +inf
      // still reach the sum) and handed to the row-end warp whole
      uint32_t flags = 0u;
#pragma unroll
      for (int u = 0; u < U; ++u) flags |= (max_above<Bits>(Tm[u], th) ? 1u : 0u) << u;
#pragma unroll
      for (int u = 0; u < U; ++u)
        add_exps<Bits>(Rv[u], c2, ((flags >> u) & 1u) ? s_off : s2, acc);
      if (__any_sync(0xFFFFFFFFu, flags != 0u)) {  // one shared atomic per warp
        uint32_t bal[U];
        int total = 0;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          bal[u] = __ballot_sync(0xFFFFFFFFu, (flags >> u) & 1u);
          total += __popc(bal[u]);
        }
        int base = 0;
        if (lane == 0) base = atomicAdd(&sm.park_count[s], total);
        int pos = __shfl_sync(0xFFFFFFFFu, base, 0);
        uint4 *pv = park_vec + (size_t)s * kParkCap;
        uint32_t *pi = park_idx + (size_t)s * kParkCap;
        const int32_t v0 = span.v0(k);
        const unsigned below = (1u << lane) - 1u;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int d = pos + __popc(bal[u] & below);
          if (((flags >> u) & 1u) && d < kParkCap) {
            pv[d] = Rv[u];
            pi[d] = (uint32_t)(v0 + ct + u * kConsumerThreads);
          }
          pos += __popc(bal[u]);
        }
      }
      if (k == K - 1) {  // end of the row: this warp's sum, then hand the row over
        double zl = 0.0;
#pragma unroll
        for (int q = 0; q < 4; ++q) zl += (double)acc[q].x + (double)acc[q].y;
        const double zs = warp_sum_d(zl);
        if (lane == 0) {
          sm.wsum[s][cw] = zs;
          if (cw == 0) {
            sm.sref[s] = ref;
            sm.park_row[s] = (int32_t)r;
            sm.park_off[s] = off;
          }
        }
        __threadfence_block();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.rowbar[s]);
      }
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

  if constexpr (C > 1) cluster_sync();  // peers write into this CTA's shared memory until here
  if (tid == 0 && *(volatile int *)&sm.abort && a.s.dev_status)
    atomicOr(a.s.dev_status, PSI_DEV_TIMEOUT);
}

// Clusters that fit on the device at once (queried once per device and
// kernel; falls back to one per C SMs).
template <typename Bits, int C>
int max_clusters() {
  static std::atomic<int> cached[PerDevice::kMax] = {};
  const int dev = PerDevice::current();
  const bool slot = dev >= 0 && dev < PerDevice::kMax;
  int n = slot ? cached[dev].load(std::memory_order_relaxed) : 0;
  if (n > 0) return n;
  int sms = 0;
  if (dev < 0 || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms <= 0)
    sms = 148;
  n = sms / C;
  if (C > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(n * C));
    cfg.blockDim = dim3(kScanThreads);
    cfg.dynamicSmemBytes = kScanDynSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int q = 0;
    if (cudaOccupancyMaxActiveClusters(&q, row_scan_kernel<Bits, C>, &cfg) == cudaSuccess && q > 0)
      n = std::min(n, q);
    else
      (void)cudaGetLastError();
  }
  if (n < 1) n = 1;
  if (slot) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

template <typename Bits, int C>
cudaError_t launch_scan_typed(const FastArgs &fa, cudaStream_t stream) {
  static DeviceOnce configure;
  cudaError_t e = configure([] {
    return cudaFuncSetAttribute(row_scan_kernel<Bits, C>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kScanDynSmem);
  });
  if (e != cudaSuccess) return e;
  const int64_t clusters = std::min<int64_t>(max_clusters<Bits, C>(), std::max<int64_t>(fa.rows, 1));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(clusters * C));
  cfg.blockDim = dim3(kScanThreads);
  cfg.dynamicSmemBytes = kScanDynSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (C > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  e = cudaLaunchKernelEx(&cfg, row_scan_kernel<Bits, C>, fa);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
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
  // rows of at least four stages are split over a cluster of two CTAs
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
