// psi_fast.cu - streaming pipeline of the sampled linear verify (T > 0) for
// 16-byte aligned rows.
//
// Sources (page title, section): "Uno Psi-Spec 是什麼？Diffusion-Augmented LLM
// 如何保留 AR 分布、一次驗證多個 Token" (alphalab.site), "Uno Psi-Spec 怎麼運作？
// 完整走一次四個 Token", steps 3-4 and the bonus paragraph (accept while
// u < p/q, longest accepted prefix, residual correction, bonus token);
// "想跑 Uno：先確認官方程式需要的環境" (temperature, top-p).
//
// Kernels, in launch order:
//   round_advance  (early-exit rounds only) One thread per sequence: lists
//              the rows and units of the next round of positions for the
//              sequences whose drafts were all accepted so far.
//   row_scan   Persistent CTAs stream every listed logit row ONCE from HBM
//              with 16-byte non-allocating loads (8 per thread in flight,
//              double buffered in registers, plus an L2 bulk prefetch).  A row
//              is read in batches of 2048 vectors; inside a batch every
//              thread uses the same reference (a lower bound of the row
//              maximum, raised between batches), so all sums are independent
//              of timing.  Elements within the window below the reference
//              ("candidates", ~0.3% of a row) are masked out of the fp32 sum
//              of exponentials; the vectors that hold them are parked in
//              shared memory and, at the row's end, split into candidates
//              (to a per-row list in global memory) and elements that fell
//              below the final threshold (a 2^31 fixed-point sum).
//   unit       One CTA of two warps per (sequence, row) unit: finishes the
//              unit's p and q rows from their candidates (row maximum, Z, the
//              top-p threshold and renormaliser), decides the drafted token
//              and draws the correction or bonus token over p's nucleus.
//   row_scan / unit, second pass   Rows whose window held less than top_p of
//              the mass (rescanned with a wider window) or whose candidates
//              overflowed (rescanned with the exact maximum known).
//   (cluster kernel, list mode)  Units the second pass could not settle.
//   fast_emit  First rejected row per sequence; emitted tokens.  Without
//              top-p the emitting row's draw needs the whole row again: it is
//              queued for the cluster kernel in sample mode.
#include <algorithm>

#include "psi_internal.h"

namespace psi {

namespace {

constexpr float kFix31F = 2147483648.0f;  // 2^31: dropped masses (each <= 1)
constexpr int kInFlight = 8;        // 16-byte loads per thread per batch
constexpr int kRing = 4096;         // parked vectors per row (shared memory)
constexpr int kListClusters = 16;
constexpr int kCounters = 8;  // work-list counters (see FastArgs::counters)
constexpr int32_t kWideBit = int32_t(1) << 30;  // second-pass row entry: wide window
// Candidate window, in log2 units below the reference.  The first pass uses
// a narrow window (13 units for top_p <= 0.95, wider as top_p approaches 1);
// the second pass the wide one.
constexpr float kWindowBaseLog2 = 13.f;
constexpr float kWindowWideLog2 = 20.f;

struct FastArgs {
  SampledArgs s;
  int64_t rows;        // N*(B+1) AR rows followed by N*B draft rows
  float coef;          // log2(e) / T
  double coef64;
  float win_narrow;    // window widths in logit units
  float win_wide;
  int use_top_p;
  int pass;            // 1: a first scan / finish; 2: a rescan of rows that failed
  const int32_t *rlist;   // rows to scan (nullptr: every row); entries may carry kWideBit
  const int32_t *rcount;  // their number
  const int32_t *ulist;   // units to finish (nullptr: every unit)
  const int32_t *ucount;  // their number
  int32_t *active;        // [N] sequence still verifying (early-exit rounds)
  int32_t *round_rows;    // rows of the current round
  int32_t *round_units;   // units of the current round
  UnitRecord *rec;     // [N*(B+1)]
  RowRecord *rowrec;   // [rows]
  uint64_t *cand;      // [rows][kCandCap]: (bits << 32) | vocabulary index
  int32_t *counters;   // [0] general units, [1] sample-mode units, [2] wide rows, [3] wide units,
                       // [4 + 2k], [5 + 2k] rows and units of round parity k
  int32_t *list_a;     // units for the general path
  int32_t *list_b;     // units whose draw needs the whole row
  int32_t *wide_rows;  // rows for the second scan (| kWideBit: wide window)
  int32_t *wide_units; // units for the second unit pass
};

template <typename Bits>
__device__ __forceinline__ const Bits *row_ptr(const FastArgs &a, int64_t r) {
  const int64_t nar = (int64_t)a.s.N * (a.s.B + 1);
  if (r < nar) return static_cast<const Bits *>(a.s.ar) + r * a.s.ar_stride;
  return static_cast<const Bits *>(a.s.draft) + (r - nar) * a.s.draft_stride;
}

// Largest element of a 16-byte vector (NaN if it holds one).
template <typename Bits>
__device__ __forceinline__ float raw_vec_max(const uint4 &w) {
  if constexpr (sizeof(Bits) == 2) {
    const __nv_bfloat162 m = __hmax2_nan(
        __hmax2_nan(*reinterpret_cast<const __nv_bfloat162 *>(&w.x),
                    *reinterpret_cast<const __nv_bfloat162 *>(&w.y)),
        __hmax2_nan(*reinterpret_cast<const __nv_bfloat162 *>(&w.z),
                    *reinterpret_cast<const __nv_bfloat162 *>(&w.w)));
    return __bfloat162float(__hmax_nan(__low2bfloat16(m), __high2bfloat16(m)));
  } else {
    const float a = __uint_as_float(w.x), b = __uint_as_float(w.y);
    const float c = __uint_as_float(w.z), d = __uint_as_float(w.w);
    return (a != a || b != b || c != c || d != d) ? NAN : fmaxf(fmaxf(a, b), fmaxf(c, d));
  }
}

template <typename T>
__device__ __forceinline__ T warp_sum_any(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Block-wide maximum, broadcast to every thread.
template <int W>
__device__ __forceinline__ float block_max_all(float v, float *scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  float r = -INFINITY;
#pragma unroll
  for (int w = 0; w < W; ++w) r = fmaxf(r, scratch[w]);
  return r;
}

__device__ __forceinline__ double exact_exp2d(float x, float m, double coef64) {
  return exp2(((double)x - (double)m) * coef64);
}

template <typename Bits>
__device__ __forceinline__ uint32_t key_to_bits(uint32_t key) {
  if constexpr (sizeof(Bits) == 2)
    return (key & 0x8000u) ? (key & 0x7FFFu) : (~key & 0xFFFFu);
  else
    return (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
}

// Candidate threshold in the element type: bf16 thresholds are rounded
// down, so the candidate set can only grow; the streaming sum and the
// extraction use this same test (x > value).
template <typename Bits>
struct Threshold {
  uint32_t pair;  // bf16x2 (both halves) or the f32 bits
  float value;
};

template <typename Bits>
__device__ __forceinline__ Threshold<Bits> make_threshold(float thr) {
  Threshold<Bits> t;
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

// The streaming step on one 16-byte vector: elements above the threshold
// are replaced by -inf, the exponentials of the others are added to the two
// packed accumulators.  Returns nonzero iff the vector holds a candidate.
template <typename Bits>
__device__ __forceinline__ uint32_t stream_vec(uint4 w, const Threshold<Bits> &t, float2 c2,
                                               float2 s2, float2 &acc_a, float2 &acc_b) {
  uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  uint32_t any = 0u;
  if constexpr (sizeof(Bits) == 2) {
    const __nv_bfloat162 t2 = *reinterpret_cast<const __nv_bfloat162 *>(&t.pair);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t m = __hgt2_mask(*reinterpret_cast<const __nv_bfloat162 *>(&ws[q]), t2);
      ws[q] = (ws[q] & ~m) | (0xFF80FF80u & m);
      any |= m;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 x = make_float2(__uint_as_float(ws[q] << 16), __uint_as_float(ws[q] & 0xFFFF0000u));
      const float2 u = __ffma2_rn(x, c2, s2);
      const float2 e = make_float2(fast_exp2(u.x), fast_exp2(u.y));
      if (q & 1) acc_b = __fadd2_rn(acc_b, e);
      else acc_a = __fadd2_rn(acc_a, e);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (__uint_as_float(ws[q]) > t.value) {
        any = 1u;
        ws[q] = 0xFF800000u;
      }
#pragma unroll
    for (int q = 0; q < 4; q += 2) {
      const float2 x = make_float2(__uint_as_float(ws[q]), __uint_as_float(ws[q + 1]));
      const float2 u = __ffma2_rn(x, c2, s2);
      const float2 e = make_float2(fast_exp2(u.x), fast_exp2(u.y));
      if (q & 2) acc_b = __fadd2_rn(acc_b, e);
      else acc_a = __fadd2_rn(acc_a, e);
    }
  }
  return any;
}

// Appends the candidates of two vectors per lane (masks m0, m1: bit q is
// element q of vector w, vector index j in the row) to the row's list in
// global memory with one warp scan and one shared-memory atomic per warp;
// every lane of the warp takes part.
template <typename Bits>
__device__ __forceinline__ void append_candidates2(uint32_t m0, const uint4 &w0, int32_t j0,
                                                   uint32_t m1, const uint4 &w1, int32_t j1,
                                                   int *s_cand, uint64_t *dst) {
  constexpr int VEC = Elem<Bits>::kVec;
  const int lane = threadIdx.x & 31;
  const int c = __popc(m0) + __popc(m1);
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
  if (total == 0) return;
  int base = 0;
  if (lane == 31) base = atomicAdd(s_cand, total);
  int pos = __shfl_sync(0xFFFFFFFFu, base, 31) + incl - c;
  while (m0) {
    const int q = __ffs(m0) - 1;
    m0 &= m0 - 1;
    if (pos < kCandCap) dst[pos] = ((uint64_t)vec_elem<Bits>(w0, q) << 32) | (uint32_t)(j0 * VEC + q);
    ++pos;
  }
  while (m1) {
    const int q = __ffs(m1) - 1;
    m1 &= m1 - 1;
    if (pos < kCandCap) dst[pos] = ((uint64_t)vec_elem<Bits>(w1, q) << 32) | (uint32_t)(j1 * VEC + q);
    ++pos;
  }
}

// Sum of exp2(x * coef + shift) over the elements of `w` selected by `mask`
// (fixed order; every selected term <= 1).
template <typename Bits>
__device__ __forceinline__ float masked_exp_sum(const uint4 &w, uint32_t mask, float coef,
                                                float shift) {
  constexpr int VEC = Elem<Bits>::kVec;
  float sum = 0.f;
#pragma unroll
  for (int q = 0; q < VEC; ++q) {
    const float e = fast_exp2(fmaf(Elem<Bits>::to_float(vec_elem<Bits>(w, q)), coef, shift));
    sum += ((mask >> q) & 1u) ? e : 0.f;
  }
  return sum;
}

// ---------------------------------------------------------------------------
// row_scan
// ---------------------------------------------------------------------------
// Running maximum of a 16-byte vector into `vm` (bf16: two lanes; f32: one).
template <typename Bits>
__device__ __forceinline__ void vec_max_into(const uint4 &w, uint32_t &vm) {
  if constexpr (sizeof(Bits) == 2) {
    __nv_bfloat162 m = *reinterpret_cast<const __nv_bfloat162 *>(&vm);
    m = __hmax2(m, *reinterpret_cast<const __nv_bfloat162 *>(&w.x));
    m = __hmax2(m, *reinterpret_cast<const __nv_bfloat162 *>(&w.y));
    m = __hmax2(m, *reinterpret_cast<const __nv_bfloat162 *>(&w.z));
    m = __hmax2(m, *reinterpret_cast<const __nv_bfloat162 *>(&w.w));
    vm = *reinterpret_cast<const uint32_t *>(&m);
  } else {
    float m = __uint_as_float(vm);
    m = fmaxf(fmaxf(m, __uint_as_float(w.x)), fmaxf(__uint_as_float(w.y), __uint_as_float(w.z)));
    vm = __float_as_uint(fmaxf(m, __uint_as_float(w.w)));
  }
}

template <typename Bits>
__device__ __forceinline__ float vm_to_float(uint32_t vm) {
  if constexpr (sizeof(Bits) == 2)
    return fmaxf(__uint_as_float(vm << 16), __uint_as_float(vm & 0xFFFF0000u));
  else
    return __uint_as_float(vm);
}

// Candidate bits of a parked vector: bit q set iff element q > t.
template <typename Bits>
__device__ __forceinline__ uint32_t above_bits(const uint4 &w, float t) {
  uint32_t mask = 0u;
  if constexpr (sizeof(Bits) == 2) {
    const __nv_bfloat162 t2 = __float2bfloat162_rn(t);  // t is a bf16 value: exact
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t m = __hgt2_mask(*reinterpret_cast<const __nv_bfloat162 *>(&ws[q]), t2);
      mask |= ((m & 1u) | ((m >> 15) & 2u)) << (2 * q);
    }
  } else {
    mask = (__uint_as_float(w.x) > t ? 1u : 0u) | (__uint_as_float(w.y) > t ? 2u : 0u) |
           (__uint_as_float(w.z) > t ? 4u : 0u) | (__uint_as_float(w.w) > t ? 8u : 0u);
  }
  return mask;
}

constexpr int kMaxBatches = 32;  // batches per row
constexpr int kPrefetch = 3;     // L2 prefetch distance, in batches beyond the register loads

// Each CTA walks its rows (item = blockIdx.x + t * gridDim.x) as one stream
// of batches; the loads of the next batch (the next row's first batch at a
// row's end) are in flight while a batch is consumed.  Vectors that hold an
// element above their batch's threshold are parked (with the batch) in a
// shared-memory ring; at the row's end, with the reference final, their
// elements above the final threshold become candidates and the others go to
// the 2^31 fixed-point sum.
template <typename Bits>
__global__ void __launch_bounds__(kThreads, 2) row_scan_kernel(const __grid_constant__ FastArgs a) {
  constexpr int VEC = Elem<Bits>::kVec;
  constexpr int U = kInFlight;
  constexpr int BATCH = U * kThreads;  // vectors per batch
  constexpr int kMaxVec = (sizeof(Bits) == 2 ? PSI_MAX_V : PSI_MAX_V / 2) / VEC;
  static_assert((kMaxVec + BATCH - 1) / BATCH <= kMaxBatches, "batch index too wide");
  static_assert(kMaxVec <= 0xFFFF, "vector index too wide");
  extern __shared__ __align__(16) unsigned char smem[];
  uint4 *fring = reinterpret_cast<uint4 *>(smem);                 // [kRing] parked vectors
  uint32_t *fidx = reinterpret_cast<uint32_t *>(fring + kRing);  // (batch << 16) | vector index
  __shared__ float s_wmax[2][kWarps];
  __shared__ float s_red[kWarps];
  __shared__ float s_thr[kMaxBatches];  // threshold of each batch of the row
  __shared__ double s_zsum[kWarps];
  __shared__ unsigned long long s_dsum[kWarps];
  __shared__ int s_nflag;               // parked vectors of the current row
  __shared__ int s_cand;                // candidates of the current row

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t V = a.s.V;
  const int32_t nvec = V / VEC;  // whole 16-byte vectors per row
  const int32_t tail = V - nvec * VEC;
  const int32_t nb = nvec > 0 ? (nvec + BATCH - 1) / BATCH : 1;
  const int64_t R = a.rlist ? (int64_t)*a.rcount : a.rows;
  if ((int64_t)blockIdx.x >= R) return;
  const int64_t my_rows = (R - 1 - (int64_t)blockIdx.x) / gridDim.x + 1;
  const float coef = a.coef;
  const float2 c2 = make_float2(coef, coef);
  uint4 neg;
  neg.x = neg.y = neg.z = neg.w = sizeof(Bits) == 2 ? 0xFF80FF80u : 0xFF800000u;
  if (tid == 0) {
    s_nflag = 0;
    s_cand = 0;
  }

  // row of local index t, and its window (logit units)
  auto row_entry = [&](int64_t t, float &off) -> int64_t {
    const int64_t item = (int64_t)blockIdx.x + t * gridDim.x;
    if (!a.rlist) {
      off = a.use_top_p ? a.win_narrow : 0.f;
      return item;
    }
    const int32_t e = a.rlist[item];
    off = !a.use_top_p ? 0.f : (e & kWideBit) ? a.win_wide : a.win_narrow;
    return (int64_t)(e & ~kWideBit);
  };

  // ---- loader: batch lk of local row lt; thread 0 also asks L2 for the
  // batch kPrefetch batches ahead (pt, pk), so that HBM keeps streaming while
  // the CTA is busy at a row's end
  int64_t lt = 0;
  int32_t lk = 0;
  float unused_off;
  const uint4 *lrv = reinterpret_cast<const uint4 *>(row_ptr<Bits>(a, row_entry(0, unused_off)));
  int64_t pt = 0;
  int32_t pk = 0;
  const uint4 *prv = lrv;
  auto advance_prefetch = [&]() {
    if (pt >= my_rows) return;
    if (tid == 0 && nvec > 0) {
      const int32_t v0 = pk * BATCH;
      const int32_t nv = min(BATCH, nvec - v0);
      prefetch_l2_bulk(prv + v0, (uint32_t)nv * 16u);
    }
    if (++pk == nb) {
      pk = 0;
      if (++pt < my_rows)
        prv = reinterpret_cast<const uint4 *>(row_ptr<Bits>(a, row_entry(pt, unused_off)));
    }
  };
  for (int d = 0; d < kPrefetch; ++d) advance_prefetch();
  auto load = [&](uint4(&buf)[U]) {
    advance_prefetch();
    if (lt >= my_rows) return;
    const int32_t j0 = lk * BATCH + tid;
    if ((lk + 1) * BATCH <= nvec) {
#pragma unroll
      for (int u = 0; u < U; ++u) buf[u] = ldg_stream(lrv + j0 + u * kThreads);
    } else {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int32_t j = j0 + u * kThreads;
        buf[u] = j < nvec ? ldg_stream(lrv + j) : neg;
      }
    }
    if (++lk == nb) {
      lk = 0;
      if (++lt < my_rows)
        lrv = reinterpret_cast<const uint4 *>(row_ptr<Bits>(a, row_entry(lt, unused_off)));
    }
  };

  // ---- consumer state (the same in every thread, except the partial sums)
  int64_t ct = 0, r = 0;
  int32_t ck = 0;
  const Bits *row = nullptr;
  float off = 0.f, ref = -INFINITY, shift = -INFINITY, z_t = 0.f;
  float2 acc_a = make_float2(0.f, 0.f), acc_b = make_float2(0.f, 0.f);

  auto consume = [&](const uint4(&buf)[U], const uint4(&nxt)[U]) {
    if (ck == 0) {
      // start of a row: the first reference is the maximum of its first two
      // batches (the second one's loads are already in flight)
      r = row_entry(ct, off);
      row = row_ptr<Bits>(a, r);
      uint32_t vm = sizeof(Bits) == 2 ? 0xFF80FF80u : 0xFF800000u;
#pragma unroll
      for (int u = 0; u < U; ++u) vec_max_into<Bits>(buf[u], vm);
      if (nb > 1) {
#pragma unroll
        for (int u = 0; u < U; ++u) vec_max_into<Bits>(nxt[u], vm);
      }
      float mx = vm_to_float<Bits>(vm);
      if (tid < tail) {
        const float x = Elem<Bits>::to_float(row[(int64_t)nvec * VEC + tid]);
        if (x == x) mx = fmaxf(mx, x);
      }
      ref = block_max_all<kWarps>(mx, s_red);
      // second pass: the row maximum is known from the first
      if (a.pass == 2) ref = fmaxf(ref, a.rowrec[r].ref);
      if (!(ref < INFINITY)) ref = -INFINITY;  // +inf: every finite element is a candidate
      shift = (ref == -INFINITY) ? -INFINITY : -ref * coef;
      z_t = 0.f;
      acc_a = acc_b = make_float2(0.f, 0.f);
    }
    // ---- stream the batch
    const Threshold<Bits> th = make_threshold<Bits>(ref - off);
    if (tid == 0) s_thr[ck] = th.value;
    const float2 s2 = make_float2(shift, shift);
    uint32_t hm = 0u;  // bit u: vector u holds an element above the threshold
    uint32_t vm = sizeof(Bits) == 2 ? 0xFF80FF80u : 0xFF800000u;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      hm |= (stream_vec<Bits>(buf[u], th, c2, s2, acc_a, acc_b) != 0u ? 1u : 0u) << u;
      vec_max_into<Bits>(buf[u], vm);
    }
    // ---- park the flagged vectors
    if (__any_sync(0xFFFFFFFFu, hm != 0u)) {
      const int c = __popc(hm);
      int idx = 0;
      if (c) idx = atomicAdd(&s_nflag, c);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if ((hm >> u) & 1u) {
          if (idx < kRing) {
            fring[idx] = buf[u];
            fidx[idx] = ((uint32_t)ck << 16) | (uint32_t)(ck * BATCH + tid + u * kThreads);
          }
          ++idx;
        }
      }
    }
    // ---- raise the reference to the batch maximum (same value in every thread)
    const float cmx = warp_max(vm_to_float<Bits>(vm));
    if (lane == 0) s_wmax[ck & 1][warp] = cmx;
    __syncthreads();
    float nr = ref;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) nr = fmaxf(nr, s_wmax[ck & 1][w]);
    if (!(nr < INFINITY)) nr = ref;
    if (nr > ref) {
      const float f = (ref == -INFINITY) ? 0.f : fast_exp2((ref - nr) * coef);
      z_t = (z_t + (acc_a.x + acc_a.y) + (acc_b.x + acc_b.y)) * f;
      acc_a = acc_b = make_float2(0.f, 0.f);
      ref = nr;
      shift = -nr * coef;
    }
    if (++ck < nb) return;

    // ---- end of the row: the reference is final
    ck = 0;
    ++ct;
    const float thf = make_threshold<Bits>(ref - off).value;
    uint64_t *dst = a.cand + r * (int64_t)kCandCap;
    if (tid < tail) {  // the ragged end (never streamed)
      const uint32_t bits = row[(int64_t)nvec * VEC + tid];
      const float x = Elem<Bits>::to_float(bits);
      if (x > thf) {
        const int slot = atomicAdd(&s_cand, 1);
        if (slot < kCandCap) dst[slot] = ((uint64_t)bits << 32) | (uint32_t)(nvec * VEC + tid);
      } else {
        z_t += fast_exp2(fmaf(x, coef, shift));
      }
    }
    z_t += (acc_a.x + acc_a.y) + (acc_b.x + acc_b.y);
    // parked vectors: elements above the final threshold are candidates, the
    // rest of what their batch masked goes to the 2^31 fixed-point sum (one
    // rounded fp32 sum per vector, <= 8; at most 4096 of them: order-free,
    // no overflow)
    const int n_flag = s_nflag;
    const int nf = min(n_flag, kRing);
    unsigned long long dsum = 0ull;
    // two parked vectors per thread per step: more shared-memory loads and
    // exponentials in flight, one warp scan for both appends
    for (int b = 0; b < nf; b += 2 * kThreads) {
      uint32_t cm[2] = {0u, 0u};
      uint4 w[2] = {neg, neg};
      int32_t j[2] = {0, 0};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int e = b + h * kThreads + tid;
        if (e < nf) {
          w[h] = fring[e];
          const uint32_t tag = fidx[e];
          j[h] = (int32_t)(tag & 0xFFFFu);
          cm[h] = above_bits<Bits>(w[h], thf);
          const uint32_t dm = above_bits<Bits>(w[h], s_thr[tag >> 16]) & ~cm[h];
          if (dm) dsum += __float2ull_rn(masked_exp_sum<Bits>(w[h], dm, coef, shift) * kFix31F);
        }
      }
      append_candidates2<Bits>(cm[0], w[0], j[0], cm[1], w[1], j[1], &s_cand, dst);
    }
    const double zs = warp_sum_any((double)z_t);
    const unsigned long long ds = warp_sum_any(dsum);
    if (lane == 0) {
      s_zsum[warp] = zs;
      s_dsum[warp] = ds;
    }
    __syncthreads();
    if (tid == 0) {
      double zt = 0.0;
      unsigned long long zd = 0ull;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        zt += s_zsum[w];
        zd += s_dsum[w];
      }
      RowRecord rec;
      rec.ref = ref;
      rec.n_cand = s_cand;
      rec.flags = n_flag > kRing ? kRowLost : 0;
      rec.n_parked = n_flag;
      rec.zt = zt;
      rec.zd = zd;
      a.rowrec[r] = rec;
      // (the next row parks and appends only after its first barrier)
      s_nflag = 0;
      s_cand = 0;
    }
  };

  uint4 b0[U], b1[U];
  const int64_t total = my_rows * nb;
  load(b0);
  for (int64_t g = 0; g < total; g += 2) {
    load(b1);
    consume(b0, b1);
    if (g + 1 >= total) break;
    load(b0);
    consume(b1, b0);
  }
}

// ---------------------------------------------------------------------------
// unit: one CTA of two warps per (sequence, row) unit
// ---------------------------------------------------------------------------
// Statistics of one finished row (the same in every lane of its warp).
struct RowFinal {
  float m;            // row maximum
  double zp;          // normaliser after top-p (Z without top-p)
  uint32_t tau_bits;  // top-p threshold (raw bits): keep x >= tau
  uint32_t tau_key;   // its order-preserving key (0 without top-p)
  int n;              // candidates of the row
  int status;         // kFin* bits
};
constexpr int kFinOverflow = 1;   // candidates lost: rescan with the exact maximum
constexpr int kFinCoverage = 2;   // the window holds less than top_p: rescan wider
constexpr int kFinNonfinite = 4;  // NaN / +inf logit, or no finite logit

constexpr int kLoadChunk = 16;           // global loads per lane in flight together
constexpr int kQChunk = 16;              // q loads per lane in flight together
constexpr int kRegCand = 16;             // candidates per lane a search keeps in registers
constexpr double kFix31 = 2147483648.0;  // 2^31: exact mass sums (each term <= 1) in u32 steps

struct WarpScratch {
  uint32_t key[kCandCap];  // candidate keys (order-preserving image of the logit); later the
                           // nucleus masses
  uint32_t idx[kCandCap];  // vocabulary indices; later the nucleus indices
  uint32_t m[kCandCap];    // 2^31 fixed-point masses exp2((x - M) * log2(e)/T); later the
                           // draw weights
};

// A candidate's mass in 2^31 fixed point: the same function of the fp32 mass
// wherever it is summed, so every exact sum is order-free.
__device__ __forceinline__ uint32_t fixed31(float m) { return __float2uint_rn(m * kFix31F); }

// Row maximum, Z, top-p threshold tau and renormaliser Z' of row r from its
// record and candidate list, by one warp.  The top-p threshold is the largest
// logit key t whose suffix mass S(t) (every x with key >= t) reaches
// top_p * Z: a binary search over the candidates' key range on exact 2^31
// fixed-point sums of the masses (integer sums: independent of candidate
// order).  Only candidates can be at or above tau when they hold at least
// top_p of the mass.  The global candidate list stays unchanged, so a second
// pass may finish the row again.
template <typename Bits>
__device__ RowFinal finish_row(const FastArgs &a, int64_t r, WarpScratch *ws) {
  const int lane = threadIdx.x & 31;
  RowFinal out;
  out.m = -INFINITY;
  out.zp = 0.0;
  out.tau_bits = Elem<Bits>::kNegInf;
  out.tau_key = 0u;
  out.n = 0;
  out.status = 0;
  const RowRecord rs = a.rowrec[r];
  if (rs.n_cand > kCandCap || (rs.flags & kRowLost)) {
    out.status = kFinOverflow;
    return out;
  }
  const int n = rs.n_cand;
  out.n = n;
  const unsigned long long *src =
      reinterpret_cast<const unsigned long long *>(a.cand + r * (int64_t)kCandCap);
  float cm = -INFINITY;
  uint32_t kmax = 0u, kmin_inv = 0u;
  for (int base = 0; base < n; base += 32 * kLoadChunk) {
    unsigned long long e[kLoadChunk];
#pragma unroll
    for (int c = 0; c < kLoadChunk; ++c) {
      const int j = base + 32 * c + lane;
      e[c] = j < n ? __ldcg(src + j) : 0ull;
    }
#pragma unroll
    for (int c = 0; c < kLoadChunk; ++c) {
      const int j = base + 32 * c + lane;
      if (j < n) {
        const uint32_t b = (uint32_t)(e[c] >> 32);
        cm = fmaxf(cm, Elem<Bits>::to_float(b));
        const uint32_t key = Elem<Bits>::key(b);
        ws->key[j] = key;
        ws->idx[j] = (uint32_t)e[c];
        kmax = max(kmax, key);
        kmin_inv = max(kmin_inv, ~key);
      }
    }
  }
  const float M = fmaxf(rs.ref, warp_max(cm));
  kmax = warp_max_u32(kmax);
  kmin_inv = warp_max_u32(kmin_inv);
  out.m = M;
  if (!(M > -INFINITY) || !(fabsf(M * a.coef) < INFINITY) || rs.zt != rs.zt) {
    out.status = kFinNonfinite;
    return out;
  }
  const float shm = -M * a.coef;
  unsigned long long zin = 0ull;
  for (int j = lane; j < n; j += 32) {
    const uint32_t m =
        fixed31(fast_exp2(fmaf(Elem<Bits>::to_float(key_to_bits<Bits>(ws->key[j])), a.coef, shm)));
    ws->m[j] = m;
    zin += m;
  }
  zin = warp_sum_any(zin);
  __syncwarp();
  double Z = (double)zin / kFix31;
  if (rs.ref > -INFINITY)
    Z += (rs.zt + (double)rs.zd / kFix31) * exp2(((double)rs.ref - (double)M) * a.coef64);
  out.zp = Z;
  if (!(Z < INFINITY)) {
    out.status = kFinNonfinite;
    return out;
  }
  if (!a.use_top_p) return out;
  const unsigned long long target = (unsigned long long)ceil((double)a.s.top_p * Z * kFix31);
  if (zin < target) {
    out.status = kFinCoverage;
    return out;
  }
  // binary search over [kmin, kmax] with exact integer sums (order-free):
  // S(kmin) = zin reaches the target
  uint32_t lo = ~kmin_inv, hi = kmax + 1u;
  unsigned long long s_lo = zin;
  if (n <= 32 * kRegCand) {
    uint32_t kr[kRegCand], mr[kRegCand];  // the row's candidates in registers
#pragma unroll
    for (int c = 0; c < kRegCand; ++c) {
      const int j = lane + 32 * c;
      kr[c] = j < n ? ws->key[j] : 0u;
      mr[c] = j < n ? ws->m[j] : 0u;
    }
    while (hi - lo > 1u) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      unsigned long long part = 0ull;
#pragma unroll
      for (int c = 0; c < kRegCand; ++c) part += kr[c] >= mid ? mr[c] : 0u;
      part = warp_sum_any(part);
      if (part >= target) {
        lo = mid;
        s_lo = part;
      } else {
        hi = mid;
      }
    }
  } else {
    while (hi - lo > 1u) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      unsigned long long part = 0ull;
      for (int j = lane; j < n; j += 32)
        if (ws->key[j] >= mid) part += ws->m[j];
      part = warp_sum_any(part);
      if (part >= target) {
        lo = mid;
        s_lo = part;
      } else {
        hi = mid;
      }
    }
  }
  out.zp = (double)s_lo / kFix31;
  out.tau_key = lo;
  out.tau_bits = key_to_bits<Bits>(lo);
  return out;
}

struct UnitShared {
  WarpScratch ws[2];  // warp 0: the p row, warp 1: the q row
  RowFinal fq;
  int need;
};

template <typename Bits>
__global__ void __launch_bounds__(64) unit_kernel(const __grid_constant__ FastArgs a) {
  extern __shared__ __align__(16) unsigned char unit_smem[];  // one UnitShared (> 48 KB)
  UnitShared &sh = *reinterpret_cast<UnitShared *>(unit_smem);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const SampledArgs &s = a.s;
  const int32_t B = s.B, N = s.N, V = s.V;
  const int64_t n_items = a.ulist ? (int64_t)*a.ucount : (int64_t)N * (B + 1);
  for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int64_t unit = a.ulist ? (int64_t)a.ulist[item] : item;
    const int32_t n = (int32_t)(unit / (B + 1)), i = (int32_t)(unit % (B + 1));
    const bool has_q = i < B;
    const int64_t rp_idx = unit;
    const int64_t rq_idx = (int64_t)N * (B + 1) + (int64_t)n * B + i;
    // the two rows in parallel
    RowFinal fp;
    if (warp == 0) {
      fp = finish_row<Bits>(a, rp_idx, &sh.ws[0]);
    } else if (has_q) {
      const RowFinal f = finish_row<Bits>(a, rq_idx, &sh.ws[1]);
      if (lane == 0) sh.fq = f;
    } else if (lane == 0) {
      sh.fq.m = -INFINITY;
      sh.fq.zp = 0.0;
      sh.fq.tau_bits = 0u;
      sh.fq.tau_key = 0u;
      sh.fq.n = 0;
      sh.fq.status = 0;
    }
    __syncthreads();
    if (warp == 0) {
      const RowFinal fq = sh.fq;
      const int fail_q = fq.status & (kFinOverflow | kFinCoverage);
      const int fail_p = fp.status & (kFinOverflow | kFinCoverage);
      const uint64_t seq = s.seq_ids ? s.seq_ids[n] : (uint64_t)n;
      const Bits *row_p = static_cast<const Bits *>(s.ar) + unit * s.ar_stride;
      const Bits *row_q =
          has_q ? static_cast<const Bits *>(s.draft) + ((int64_t)n * B + i) * s.draft_stride : nullptr;
      const float tau_p = Elem<Bits>::to_float(fp.tau_bits);
      const float tau_q = Elem<Bits>::to_float(fq.tau_bits);
      int need = 0;
      if (fail_q || fail_p) {
        if (lane == 0) {
          if (a.pass == 1) {  // rescan the failed rows, then finish the unit again
            if (fail_q)
              a.wide_rows[atomicAdd(&a.counters[2], 1)] =
                  (int32_t)rq_idx | ((fail_q & kFinCoverage) ? kWideBit : 0);
            if (fail_p)
              a.wide_rows[atomicAdd(&a.counters[2], 1)] =
                  (int32_t)rp_idx | ((fail_p & kFinCoverage) ? kWideBit : 0);
            a.wide_units[atomicAdd(&a.counters[3], 1)] = (int32_t)unit;
          } else {  // the general path verifies this unit (records included)
            a.list_a[atomicAdd(&a.counters[0], 1)] = (int32_t)unit;
            a.rec[unit].accept = -1;  // decided at the end; a later round treats it as accepted
          }
        }
      } else {
        // ---- accept / reject the drafted token (lane 0, double precision)
        need = 1;
        if (lane == 0) {
          if (has_q) {
            const int32_t x = s.ids[(int64_t)n * B + i];
            double p = 0.0, q = 0.0;
            const bool valid = x >= 0 && x < V;
            if (valid) {
              const float xp = Elem<Bits>::to_float(row_p[x]);
              const float xq = Elem<Bits>::to_float(row_q[x]);
              if (xp >= tau_p && fp.zp > 0.0) p = exact_exp2d(xp, fp.m, a.coef64) / fp.zp;
              if (xq >= tau_q && fq.zp > 0.0) q = exact_exp2d(xq, fq.m, a.coef64) / fq.zp;
            }
            const double u = (double)uniform24(s.seed, seq, s.step, (uint64_t)i, PSI_PURPOSE_ACCEPT);
            const int accept = (u * q < p) ? 1 : 0;
            need = !accept;
            if (s.out_p) s.out_p[(int64_t)n * B + i] = (float)p;
            if (s.out_q) s.out_q[(int64_t)n * B + i] = (float)q;
            a.rec[unit].accept = accept;
            if (accept) a.rec[unit].token = -1;
            if (!valid && s.dev_status) atomicOr(s.dev_status, PSI_DEV_BAD_TOKEN_ID);
          } else {
            a.rec[unit].accept = 1;
          }
          if (((fp.status | fq.status) & kFinNonfinite) && s.dev_status)
            atomicOr(s.dev_status, PSI_DEV_NONFINITE);
        }
        need = __shfl_sync(0xFFFFFFFFu, need, 0);
        if (need && !a.use_top_p) {  // the draw needs whole rows: decided after the emit step
          if (lane == 0) a.rec[unit].token = -2;
          need = 0;
        }
      }
      if (need) {
        // ---- correction / bonus draw over p's nucleus (its candidates with
        // key >= tau), inverse CDF in vocabulary order, exact integer sums
        WarpScratch *ws = &sh.ws[0];
        const int nc = (fp.status & kFinNonfinite) ? 0 : fp.n;
        const float inv_zp = fp.zp > 0.0 ? (float)(1.0 / fp.zp) : 0.f;
        const float shq = -fq.m * a.coef, inv_zq = fq.zp > 0.0 ? (float)(1.0 / fq.zp) : 0.f;
        // compact the nucleus to the front, in candidate order: index in
        // idx[], mass in key[] (reads of a group precede its writes, which
        // land at or before the group)
        const unsigned below = (1u << lane) - 1u;
        int nn = 0;
        for (int base = 0; base < nc; base += 32) {
          const int j = base + lane;
          const bool in = j < nc && ws->key[j] >= fp.tau_key;
          uint32_t v = 0u, m = 0u;
          if (in) {
            v = ws->idx[j];
            m = ws->m[j];
          }
          const unsigned bal = __ballot_sync(0xFFFFFFFFu, in);
          __syncwarp();
          if (in) {
            const int d = nn + __popc(bal & below);
            ws->idx[d] = v;
            ws->key[d] = m;
          }
          nn += __popc(bal);
        }
        __syncwarp();
        int32_t token = 0;
        for (int pass = 0; pass < 2; ++pass) {
          const bool p_only = !has_q || pass == 1;
          unsigned long long part = 0ull;
          for (int base = 0; base < nn; base += 32 * kQChunk) {
            uint32_t xqb[kQChunk];  // q logits of the chunk, loads in flight together
#pragma unroll
            for (int c = 0; c < kQChunk; ++c) {
              const int j = base + 32 * c + lane;
              xqb[c] = (!p_only && j < nn) ? (uint32_t)row_q[ws->idx[j]] : 0u;
            }
#pragma unroll
            for (int c = 0; c < kQChunk; ++c) {
              const int j = base + 32 * c + lane;
              if (j < nn) {
                float pv = (float)ws->key[j] * (1.f / kFix31F) * inv_zp;
                if (!p_only) {
                  const float xq = Elem<Bits>::to_float(xqb[c]);
                  const float qv = xq >= tau_q ? fast_exp2(fmaf(xq, a.coef, shq)) * inv_zq : 0.f;
                  pv = fmaxf(pv - qv, 0.f);
                }
                const uint32_t wj = fixed31(fminf(pv, 1.f));
                ws->m[j] = wj;
                part += wj;
              }
            }
          }
          const unsigned long long W = warp_sum_any(part);
          __syncwarp();
          if (W == 0ull && !p_only) continue;  // residual vanished: draw from p itself
          if (W > 0ull) {
            // t = floor(u' * W) exactly (u' = k / 2^24)
            const float u2 = uniform24(s.seed, seq, s.step, (uint64_t)i, PSI_PURPOSE_RESID);
            const unsigned long long k = (unsigned long long)(u2 * 16777216.0f);
            const unsigned long long t = (__umul64hi(k, W) << 40) | ((k * W) >> 24);
            // smallest X with C(X) = (weight of entries with index < X) > t;
            // the token is X - 1 (C(V) = W > t)
            uint32_t lo = 0u, hi = (uint32_t)V;
            if (nn <= 32 * kRegCand) {
              uint32_t ir[kRegCand], wr[kRegCand];
#pragma unroll
              for (int c = 0; c < kRegCand; ++c) {
                const int j = lane + 32 * c;
                ir[c] = j < nn ? ws->idx[j] : 0xFFFFFFFFu;
                wr[c] = j < nn ? ws->m[j] : 0u;
              }
              while (hi - lo > 1u) {
                const uint32_t mid = (lo + hi) >> 1;
                unsigned long long c = 0ull;
#pragma unroll
                for (int q = 0; q < kRegCand; ++q) c += ir[q] < mid ? wr[q] : 0u;
                c = warp_sum_any(c);
                if (c > t) hi = mid;
                else lo = mid;
              }
            } else {
              while (hi - lo > 1u) {
                const uint32_t mid = (lo + hi) >> 1;
                unsigned long long c = 0ull;
                for (int j = lane; j < nn; j += 32)
                  if (ws->idx[j] < mid) c += ws->m[j];
                c = warp_sum_any(c);
                if (c > t) hi = mid;
                else lo = mid;
              }
            }
            token = (int32_t)lo;
          }
          break;
        }
        if (lane == 0) a.rec[unit].token = token;
      }
    }
    __syncthreads();  // shared memory free for the next unit
  }
}

// ---------------------------------------------------------------------------
// fast_emit: one thread per sequence.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) fast_emit_kernel(const __grid_constant__ FastArgs a) {
  const int32_t n = blockIdx.x * blockDim.x + threadIdx.x;
  const SampledArgs &s = a.s;
  if (n >= s.N) return;
  const int32_t B = s.B;
  const UnitRecord *r = a.rec + (int64_t)n * (B + 1);
  int32_t L = B;
  for (int32_t i = 0; i < B; ++i)
    if (!r[i].accept) {
      L = i;
      break;
    }
  int32_t *tok = s.out_tokens + (int64_t)n * (B + 1);
  for (int32_t i = 0; i < L; ++i) tok[i] = s.ids[(int64_t)n * B + i];
  const int32_t t = r[L].token;
  tok[L] = t;
  for (int32_t i = L + 1; i <= B; ++i) tok[i] = -1;
  s.out_n[n] = L + 1;
  if (t == -2) a.list_b[atomicAdd(&a.counters[1], 1)] = n * (B + 1) + L;
}

// SM count of the current device (queried once per device).
int sm_count() {
  static std::atomic<int> cached[PerDevice::kMax] = {};
  const int dev = PerDevice::current();
  const bool slot = dev >= 0 && dev < PerDevice::kMax;
  int count = slot ? cached[dev].load(std::memory_order_relaxed) : 0;
  if (count > 0) return count;
  if (dev < 0 || cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      count <= 0)
    count = 148;
  if (slot) cached[dev].store(count, std::memory_order_relaxed);
  return count;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

constexpr size_t kScanSmem = (sizeof(uint4) + sizeof(uint32_t)) * kRing;

// ---------------------------------------------------------------------------
// round_advance: one thread per sequence.  Early-exit rounds: round k covers
// positions [round_begin(k), round_begin(k + 1)) of B + 1.
// A sequence takes part in round k when every drafted token of the earlier
// rounds was accepted (a unit left to the general path counts as accepted:
// its rows are then read although a rejection may make them unused).  The
// kernel lists the round's rows and units, and resets the lists that the
// round's finish step and the next round fill.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) round_advance_kernel(const __grid_constant__ FastArgs a,
                                                            int k) {
  const int32_t n = blockIdx.x * blockDim.x + threadIdx.x;
  const SampledArgs &s = a.s;
  const int32_t B = s.B, N = s.N;
  if (n == 0) {
    a.counters[2] = 0;  // this round's second-pass lists
    a.counters[3] = 0;
    a.counters[4 + 2 * ((k + 1) & 1)] = 0;  // the next round's lists
    a.counters[5 + 2 * ((k + 1) & 1)] = 0;
  }
  if (n >= N) return;
  const int32_t i0 = round_begin(k, B, PSI_SAMPLED_SHORT_ROUNDS);
  const int32_t i1 = round_begin(k + 1, B, PSI_SAMPLED_SHORT_ROUNDS);
  int act = 1;
  if (k > 0) {
    act = a.active[n];
    const UnitRecord *r = a.rec + (int64_t)n * (B + 1);
    for (int32_t i = round_begin(k - 1, B, PSI_SAMPLED_SHORT_ROUNDS); act && i < i0; ++i)
      if (i < B && r[i].accept == 0) act = 0;
  }
  a.active[n] = act;
  if (!act || i0 >= i1) return;
  int32_t *rc = a.counters + 4 + 2 * (k & 1);
  const int32_t nu = i1 - i0;
  const int32_t nd = min(i1, B) - i0;  // draft rows (the bonus row has none)
  const int32_t su = atomicAdd(rc + 1, nu);
  const int32_t sr = atomicAdd(rc, nu + nd);
  for (int32_t i = i0; i < i1; ++i) {
    const int32_t unit = n * (B + 1) + i;
    a.round_units[su + (i - i0)] = unit;
    a.round_rows[sr + (i - i0)] = unit;  // the AR row has the unit's index
  }
  for (int32_t i = i0; i < i0 + nd; ++i)
    a.round_rows[sr + nu + (i - i0)] = N * (B + 1) + n * B + i;
}

template <typename Bits>
cudaError_t launch_fast_typed(const FastArgs &fa, const SampledPlan &plan, bool early_exit,
                              const KernelEvents &ev, cudaStream_t stream) {
  const int64_t units = (int64_t)fa.s.N * (fa.s.B + 1);
  const int64_t persistent = (int64_t)sm_count() * 2;
  const int64_t grid_scan = std::min<int64_t>(fa.rows, persistent);
  const int64_t grid_unit = units;
  cudaError_t e;
  static DeviceOnce configure;  // shared memory above 48 KB, once per device
  e = configure([] {
    cudaError_t err = cudaFuncSetAttribute(row_scan_kernel<Bits>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)kScanSmem);
    if (err != cudaSuccess) return err;
    return cudaFuncSetAttribute(unit_kernel<Bits>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)sizeof(UnitShared));
  });
  if (e != cudaSuccess) return e;
  // the work-list counters of this call start at zero
  if ((e = cudaMemsetAsync(fa.counters, 0, kCounters * sizeof(int32_t), stream)) != cudaSuccess)
    return e;
  // rows / units of one pass (first scan or rescan), then finish them
  auto scan_and_finish = [&](const FastArgs &f, bool timed) -> cudaError_t {
    cudaError_t err;
    if (timed && ev.before && (err = cudaEventRecord(ev.before, stream)) != cudaSuccess) return err;
    row_scan_kernel<Bits><<<(unsigned)grid_scan, kThreads, kScanSmem, stream>>>(f);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    if (timed && ev.after && (err = cudaEventRecord(ev.after, stream)) != cudaSuccess) return err;
    const int64_t g = f.pass == 1 ? grid_unit : std::min<int64_t>(grid_unit, persistent);
    unit_kernel<Bits><<<(unsigned)g, 64, sizeof(UnitShared), stream>>>(f);
    return cudaGetLastError();
  };
  // the second pass over the rows and units a first pass could not settle
  // (usually none: the CTAs find empty lists and exit)
  FastArgs f2 = fa;
  f2.pass = 2;
  f2.rlist = fa.wide_rows;
  f2.rcount = fa.counters + 2;
  f2.ulist = fa.wide_units;
  f2.ucount = fa.counters + 3;
  if (!early_exit) {
    if ((e = scan_and_finish(fa, true)) != cudaSuccess) return e;
    if ((e = scan_and_finish(f2, false)) != cudaSuccess) return e;
  } else {
    const int rounds = round_count(fa.s.B, PSI_SAMPLED_SHORT_ROUNDS);
    for (int k = 0; k < rounds; ++k) {
      round_advance_kernel<<<(fa.s.N + 127) / 128, 128, 0, stream>>>(fa, k);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      FastArgs f1 = fa;
      f1.rlist = fa.round_rows;
      f1.rcount = fa.counters + 4 + 2 * (k & 1);
      f1.ulist = fa.round_units;
      f1.ucount = fa.counters + 5 + 2 * (k & 1);
      if ((e = scan_and_finish(f1, k == 0)) != cudaSuccess) return e;
      if ((e = scan_and_finish(f2, false)) != cudaSuccess) return e;
    }
  }
  const psi_dtype dt = sizeof(Bits) == 2 ? PSI_DTYPE_BF16 : PSI_DTYPE_F32;
  SampledArgs sa = fa.s;
  sa.records = fa.rec;
  const int clusters_a = (int)std::min<int64_t>(units, kListClusters);
  e = launch_cluster_list(sa, dt, plan, kClusterModeList, fa.list_a, fa.counters + 0, clusters_a,
                          stream);
  if (e != cudaSuccess) return e;
  fast_emit_kernel<<<(fa.s.N + 127) / 128, 128, 0, stream>>>(fa);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int clusters_b = std::min(fa.s.N, kListClusters);
  return launch_cluster_list(sa, dt, plan, kClusterModeSample, fa.list_b, fa.counters + 1,
                             clusters_b, stream);
}

}  // namespace

FastLayout fast_layout(int32_t N, int32_t B) {
  FastLayout L;
  const int64_t units = (int64_t)N * (B + 1);
  const int64_t rows = units + (int64_t)N * B;
  size_t off = 0;
  L.rec_off = off;
  off = align256(off + sizeof(UnitRecord) * (size_t)units);
  L.rows_off = off;
  off = align256(off + sizeof(RowRecord) * (size_t)rows);
  L.cand_off = off;
  off = align256(off + sizeof(uint64_t) * (size_t)rows * kCandCap);
  L.counters_off = off;
  off = align256(off + sizeof(int32_t) * kCounters);
  L.list_a_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)units);
  L.list_b_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)N);
  L.wide_rows_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)rows);
  L.wide_units_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)units);
  L.round_rows_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)rows);
  L.round_units_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)units);
  L.active_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)N);
  L.total = off;
  return L;
}

bool fast_path_fits(int32_t N, int32_t B) {
  // row indices travel in 30 bits of a second-pass list entry
  return (int64_t)N * (2 * (int64_t)B + 1) < (int64_t(1) << 30);
}

cudaError_t launch_sampled_fast(const SampledArgs &a, psi_dtype dtype, const SampledPlan &plan,
                                void *workspace, const KernelEvents &ev, cudaStream_t stream) {
  const FastLayout L = fast_layout(a.N, a.B);
  char *ws = static_cast<char *>(workspace);
  FastArgs fa;
  fa.s = a;
  fa.rows = (int64_t)a.N * (a.B + 1) + (int64_t)a.N * a.B;
  fa.coef64 = 1.4426950408889634 / (double)a.temperature;
  fa.coef = (float)fa.coef64;
  // first-pass window: 13 log2 units for top_p <= 0.95, one more unit for
  // every halving of the allowed tail mass beyond 5%, at most the wide window
  double wlog2 = kWindowBaseLog2;
  if (a.top_p < 1.0f && a.top_p > 0.95f) wlog2 += log2(0.05 / (1.0 - (double)a.top_p));
  if (wlog2 > kWindowWideLog2) wlog2 = kWindowWideLog2;
  fa.win_narrow = (float)(wlog2 / fa.coef64);
  fa.win_wide = (float)(kWindowWideLog2 / fa.coef64);
  fa.use_top_p = a.top_p < 1.0f ? 1 : 0;
  fa.pass = 1;
  fa.rec = reinterpret_cast<UnitRecord *>(ws + L.rec_off);
  fa.rowrec = reinterpret_cast<RowRecord *>(ws + L.rows_off);
  fa.cand = reinterpret_cast<uint64_t *>(ws + L.cand_off);
  fa.counters = reinterpret_cast<int32_t *>(ws + L.counters_off);
  fa.list_a = reinterpret_cast<int32_t *>(ws + L.list_a_off);
  fa.list_b = reinterpret_cast<int32_t *>(ws + L.list_b_off);
  fa.wide_rows = reinterpret_cast<int32_t *>(ws + L.wide_rows_off);
  fa.wide_units = reinterpret_cast<int32_t *>(ws + L.wide_units_off);
  fa.round_rows = reinterpret_cast<int32_t *>(ws + L.round_rows_off);
  fa.round_units = reinterpret_cast<int32_t *>(ws + L.round_units_off);
  fa.active = reinterpret_cast<int32_t *>(ws + L.active_off);
  fa.rlist = nullptr;
  fa.rcount = nullptr;
  fa.ulist = nullptr;
  fa.ucount = nullptr;
  fa.s.records = fa.rec;
  // without p / q outputs only the rows up to each sequence's first rejection
  // matter: verify in early-exit rounds
  const bool early_exit = a.out_p == nullptr && a.out_q == nullptr && a.N >= PSI_EARLY_EXIT_MIN_N;
  if (dtype == PSI_DTYPE_BF16) return launch_fast_typed<uint16_t>(fa, plan, early_exit, ev, stream);
  return launch_fast_typed<uint32_t>(fa, plan, early_exit, ev, stream);
}

}  // namespace psi
