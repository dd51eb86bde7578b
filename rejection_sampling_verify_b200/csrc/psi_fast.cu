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
//   row_stats      Persistent CTAs stream every logit row ONCE from HBM
//                  through a 4-stage ring of TMA bulk copies (16 KB each) in
//                  shared memory.  Per row: maximum m and sum of exponentials
//                  Z (online, fp32 for the bulk of the row), and with top-p
//                  the few elements within 2^16 of the running maximum
//                  ("candidates", typically ~1% of the row) kept in shared
//                  memory, re-evaluated in double precision at the end of the
//                  row, and radix-selected on their logit key to find the
//                  top-p threshold tau, the renormaliser Z' and the nucleus
//                  (written out, <= 1024 entries).
//   unit_decide    One CTA per (sequence, row): p(x), q(x), the acceptance
//                  test, and -- with top-p -- the correction or bonus draw
//                  over the nucleus only (max(0, p - q) vanishes outside p's
//                  nucleus), so no logit is read twice.
//   (cluster kernel, list mode)  units the streaming path cannot handle
//                  (candidate overflow, a top-p set wider than the window).
//   fast_emit      First rejected row per sequence; emitted tokens.  Without
//                  top-p the emitting row's draw needs the whole row again:
//                  it is queued for the cluster kernel in sample mode.
#include <algorithm>

#include "psi_internal.h"

namespace psi {

namespace {

constexpr int kStages = 4;
constexpr int kChunkBytes = 16384;
constexpr int kCandCap = 4096;              // candidate buffer (shared memory)
constexpr double kFixD = 1099511627776.0;  // 2^40
// Candidate window, in log2 units below the (running) row maximum: starts at
// 16 (e > 2^-16 of the maximum) and narrows by 2 down to 12 when the buffer
// fills; the final window must hold top_p of the mass, else the unit goes to
// the general path.
constexpr float kWindowLog2 = 16.f;
constexpr float kWindowStepLog2 = 2.f;
constexpr float kWindowMinLog2 = 12.f;
constexpr int kUnitThreads = 256;
constexpr int kListClusters = 16;

struct FastArgs {
  SampledArgs s;
  int64_t rows;          // N*(B+1) AR rows followed by N*B draft rows
  float coef;            // log2(e) / T
  double coef64;
  float win_off;         // initial window width in logit units: 16 / coef
  int use_top_p;
  UnitRecord *rec;       // [N*(B+1)]
  RowRecord *rowrec;     // [rows]
  uint64_t *nuc;         // [rows][kNucCap]
  int32_t *counters;     // [0] list A count, [1] list B count
  int32_t *list_a;       // units for the general path
  int32_t *list_b;       // units whose draw needs the whole row
};

template <typename Bits>
__device__ __forceinline__ const Bits *row_ptr(const FastArgs &a, int64_t r) {
  const int64_t nar = (int64_t)a.s.N * (a.s.B + 1);
  if (r < nar) return static_cast<const Bits *>(a.s.ar) + r * a.s.ar_stride;
  return static_cast<const Bits *>(a.s.draft) + (r - nar) * a.s.draft_stride;
}

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

// Block-wide sum (fixed order), broadcast to every thread.
template <typename T>
__device__ __forceinline__ T block_sum_all(T v, T *scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_any(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  T r = T(0);
#pragma unroll
  for (int w = 0; w < kWarps; ++w) r += scratch[w];
  return r;
}

__device__ __forceinline__ float block_max_all(float v, float *scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  float r = -INFINITY;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) r = fmaxf(r, scratch[w]);
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

// Packed fp32 pairs (sm_100 f32x2 instructions).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2,%3};\n\tmov.b64 rb, {%4,%5};\n\t"
      "mov.b64 rc, {%6,%7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0,%1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2,%3};\n\tmov.b64 rb, {%4,%5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0,%1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// Block-wide compaction of the candidate buffer: entries with logit > thr
// stay (packed to the front, in thread order); the others leave the buffer
// and their mass exp2((x - ref) * coef) is added to zd_t, the thread's
// dropped-mass accumulator, whose reference zd_ref is moved to `ref` first.
// An overflowed buffer (count > capacity) stays marked as overflowed.
template <typename Bits>
__device__ void compact_candidates(unsigned long long *cand, int *s_cand, int *s_keep, float thr,
                                   float ref, float coef, float &zd_t, float &zd_ref) {
  constexpr int PER = kCandCap / kThreads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (zd_ref != ref) {
    zd_t = (zd_ref == -INFINITY) ? 0.f : zd_t * fast_exp2((zd_ref - ref) * coef);
    zd_ref = ref;
  }
  const int count = *s_cand;
  const int n_have = min(count, kCandCap);
  unsigned long long mine[PER];
  uint32_t kept = 0u;  // bit t: entry t of this thread stays
  int keep = 0;
#pragma unroll
  for (int t = 0; t < PER; ++t) {
    const int j = tid * PER + t;
    mine[t] = 0ull;
    if (j < n_have) {
      const unsigned long long e = cand[j];
      const float x = Elem<Bits>::to_float((uint32_t)(e >> 32));
      if (x > thr) {
        mine[t] = e;
        kept |= 1u << t;
        ++keep;
      } else {
        zd_t += fast_exp2((x - ref) * coef);
      }
    }
  }
  int incl = keep;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  __syncthreads();  // every entry has been read
  if (lane == 31) s_keep[warp] = incl;
  __syncthreads();
  int off = incl - keep, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    if (w < warp) off += s_keep[w];
    tot += s_keep[w];
  }
#pragma unroll
  for (int t = 0; t < PER; ++t)
    if (kept & (1u << t)) cand[off++] = mine[t];
  __syncthreads();  // everyone has read the old count and s_keep
  if (threadIdx.x == 0) *s_cand = (count > kCandCap) ? kCandCap + 1 : tot;
  __syncthreads();
}

// Warp-aggregated append of this lane's candidates (bit e of `mask`: element
// e of the vector starting at vocabulary index `base`).  Every lane of the
// warp must call it.  Returns the largest appended logit of this lane.
template <typename Bits>
__device__ __forceinline__ float append_candidates(const uint4 &w, uint32_t mask, int32_t base,
                                                   int *s_cand, unsigned long long *cand) {
  const int lane = threadIdx.x & 31;
  const int cnt = __popc(mask);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  const int tot = __shfl_sync(0xFFFFFFFFu, incl, 31);
  int first = 0;
  if (lane == 31 && tot) first = atomicAdd(s_cand, tot);
  int pos = __shfl_sync(0xFFFFFFFFu, first, 31) + incl - cnt;
  float mx = -INFINITY;
  while (mask) {
    const int e = __ffs(mask) - 1;
    mask &= mask - 1;
    const uint32_t b = vec_elem<Bits>(w, e);
    mx = fmaxf(mx, Elem<Bits>::to_float(b));
    if (pos < kCandCap) cand[pos] = ((unsigned long long)b << 32) | (uint32_t)(base + e);
    ++pos;
  }
  return mx;
}

// The streaming step on one 16-byte vector: elements above the candidate
// threshold are replaced by -inf (their bit set in the returned mask), the
// exponentials of the others are added to the two packed accumulators.
template <typename Bits>
__device__ __forceinline__ uint32_t stream_vec(uint4 w, float thr, float2 c2, float2 s2,
                                               float2 &acc_a, float2 &acc_b) {
  uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  uint32_t mask = 0u;
  if constexpr (sizeof(Bits) == 2) {
    // thr rounded down to bf16: x > thr implies x > thr_b, so the candidate
    // set can only grow; sum and append use this same test.
    const __nv_bfloat162 t2 = __bfloat162bfloat162(__float2bfloat16_rd(thr));
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t m = __hgt2_mask(*reinterpret_cast<const __nv_bfloat162 *>(&ws[q]), t2);
      ws[q] = (ws[q] & ~m) | (0xFF80FF80u & m);
      mask |= ((m & 1u) | ((m >> 15) & 2u)) << (2 * q);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 x = make_float2(__uint_as_float(ws[q] << 16), __uint_as_float(ws[q] & 0xFFFF0000u));
      const float2 t = ffma2(x, c2, s2);
      const float2 e = make_float2(fast_exp2(t.x), fast_exp2(t.y));
      if (q & 1) acc_b = fadd2(acc_b, e);
      else acc_a = fadd2(acc_a, e);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (__uint_as_float(ws[q]) > thr) {
        mask |= 1u << q;
        ws[q] = 0xFF800000u;
      }
#pragma unroll
    for (int q = 0; q < 4; q += 2) {
      const float2 x = make_float2(__uint_as_float(ws[q]), __uint_as_float(ws[q + 1]));
      const float2 t = ffma2(x, c2, s2);
      const float2 e = make_float2(fast_exp2(t.x), fast_exp2(t.y));
      if (q & 2) acc_b = fadd2(acc_b, e);
      else acc_a = fadd2(acc_a, e);
    }
  }
  return mask;
}

template <typename Bits>
__device__ __forceinline__ float candidate_threshold_value(float thr) {
  if constexpr (sizeof(Bits) == 2)
    return __bfloat162float(__float2bfloat16_rd(thr));
  else
    return thr;
}

// ---------------------------------------------------------------------------
// row_stats
// ---------------------------------------------------------------------------
template <typename Bits>
__global__ void __launch_bounds__(kThreads, 2) row_stats_kernel(const FastArgs a) {
  constexpr int VEC = Elem<Bits>::kVec;
  constexpr int CH = kChunkBytes / (int)sizeof(Bits);  // elements per chunk
  constexpr int KEYB = Elem<Bits>::kKeyBits;
  extern __shared__ __align__(128) unsigned char smem[];
  Bits *stages = reinterpret_cast<Bits *>(smem);
  unsigned long long *cand = reinterpret_cast<unsigned long long *>(smem + kStages * kChunkBytes);
  __shared__ __align__(8) uint64_t mbar[kStages];
  __shared__ float s_f[kWarps];
  __shared__ float s_wmax[2][kWarps];
  __shared__ double s_d[kWarps];
  __shared__ unsigned long long s_u[kWarps];
  __shared__ unsigned long long s_bs[2][kWarps];
  __shared__ int s_cand, s_nuc;
  __shared__ int s_keep[kWarps];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t V = a.s.V;
  const int64_t R = a.rows;
  const int32_t nck = (V + CH - 1) / CH;
  const int64_t my_rows = ((int64_t)blockIdx.x < R) ? (R - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int64_t total = my_rows * nck;
  const float coef = a.coef;
  const float2 c2 = make_float2(coef, coef);
  const int max_narrowings = (int)((kWindowLog2 - kWindowMinLog2) / kWindowStepLog2);
  // Without top-p the "window" is empty: candidates are only the elements
  // above the running reference (a few per row), summed exactly at the end.
  const float win0 = a.use_top_p ? a.win_off : 0.f;

  if (blockIdx.x == 0 && tid < 2) a.counters[tid] = 0;  // work lists of this call
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&mbar[s], 1);
    fence_mbar_init();
  }
  __syncthreads();

  auto issue = [&](int64_t g) {  // thread 0: start the copy of chunk g
    if (g >= total) return;
    const int64_t r = blockIdx.x + (g / nck) * (int64_t)gridDim.x;
    const int32_t c0 = (int32_t)(g % nck) * CH;
    const int32_t len = min(CH, V - c0);
    const uint32_t bytes = (uint32_t)(len / VEC) * VEC * (uint32_t)sizeof(Bits);
    uint64_t *bar = &mbar[g % kStages];
    mbar_arrive_expect_tx(bar, bytes);
    if (bytes) bulk_load(stages + (g % kStages) * CH, row_ptr<Bits>(a, r) + c0, bytes, bar);
  };
  if (tid == 0)
    for (int64_t g = 0; g < kStages; ++g) issue(g);

  // m_ref: CTA-uniform lower bound of the row maximum, never below any
  // non-candidate seen so far.  z_t: this thread's sum of exp2((x - m_ref) *
  // coef) over non-candidates (each <= 1, so nothing overflows); zd_t: mass
  // of candidates dropped by a compaction, relative to zd_ref.  off: window
  // width in logit units.
  float z_t = 0.f, m_ref = -INFINITY, shift = -INFINITY;
  float zd_t = 0.f, zd_ref = -INFINITY, off = win0;
  int narrowed = 0;
  bool timed_out = false;
  for (int64_t g = 0; g < total; ++g) {
    const int64_t r = blockIdx.x + (g / nck) * (int64_t)gridDim.x;
    const int32_t k = (int32_t)(g % nck);
    const int32_t c0 = k * CH, len = min(CH, V - c0), nv = len / VEC, tail = len - nv * VEC;
    const Bits *row = row_ptr<Bits>(a, r);
    const uint4 *sv = reinterpret_cast<const uint4 *>(stages + (g % kStages) * CH);
    if (k == 0) {
      z_t = 0.f;
      zd_t = 0.f;
      zd_ref = -INFINITY;
      off = win0;
      narrowed = 0;
      if (tid == 0) s_cand = 0;
      // First reference: the maximum over every chunk of this row already in
      // the ring (up to kStages * 16 KB of the row).
      const int32_t in_ring = min(kStages, nck);
      const int32_t ahead = (total - g < (int64_t)in_ring) ? (int32_t)(total - g) : in_ring;
      float mx = -INFINITY;
      for (int32_t h = 0; h < ahead; ++h) {
        const int64_t gh = g + h;
        timed_out |= !mbar_wait_bounded(&mbar[gh % kStages], (uint32_t)((gh / kStages) & 1));
        const int32_t ch0 = h * CH, chl = min(CH, V - ch0), chv = chl / VEC;
        const uint4 *hv = reinterpret_cast<const uint4 *>(stages + (gh % kStages) * CH);
        for (int32_t j = tid; j < chv; j += kThreads) {
          const float vm = raw_vec_max<Bits>(hv[j]);
          if (vm == vm) mx = fmaxf(mx, vm);
        }
        const int32_t cht = chl - chv * VEC;
        if (tid < cht) {
          const float x = Elem<Bits>::to_float(row[ch0 + chv * VEC + tid]);
          if (x == x) mx = fmaxf(mx, x);
        }
      }
      m_ref = block_max_all(mx, s_f);
      if (!(m_ref < INFINITY)) m_ref = -INFINITY;  // +inf: everything above -inf is a candidate
      shift = (m_ref == -INFINITY) ? -INFINITY : -m_ref * coef;
    }
    timed_out |= !mbar_wait_bounded(&mbar[g % kStages], (uint32_t)((g / kStages) & 1));
    const float thr = m_ref - off;  // candidate iff x > thr (as rounded for the test)
    const float2 s2 = make_float2(shift, shift);
    float2 acc_a = make_float2(0.f, 0.f), acc_b = make_float2(0.f, 0.f);
    float cmx = -INFINITY;
    uint4 neg;
    neg.x = neg.y = neg.z = neg.w = sizeof(Bits) == 2 ? 0xFF80FF80u : 0xFF800000u;
    // Two vectors per lane per iteration; every lane of a warp runs the same
    // number of iterations (the ballot below needs the whole warp).
    for (int32_t j0 = warp * 32; j0 < nv; j0 += 2 * kThreads) {
      const int32_t ja = j0 + lane, jb = j0 + kThreads + lane;
      const uint4 wa = ja < nv ? sv[ja] : neg;
      const uint4 wb = jb < nv ? sv[jb] : neg;
      const uint32_t ma = stream_vec<Bits>(wa, thr, c2, s2, acc_a, acc_b);
      const uint32_t mb = stream_vec<Bits>(wb, thr, c2, s2, acc_a, acc_b);
      if (__ballot_sync(0xFFFFFFFFu, (ma | mb) != 0u)) {
        cmx = fmaxf(cmx, append_candidates<Bits>(wa, ma, c0 + ja * VEC, &s_cand, cand));
        cmx = fmaxf(cmx, append_candidates<Bits>(wb, mb, c0 + jb * VEC, &s_cand, cand));
      }
    }
    z_t += (acc_a.x + acc_a.y) + (acc_b.x + acc_b.y);
    if (tid < tail) {  // ragged end of the row (fewer than one vector)
      const uint32_t b = row[c0 + nv * VEC + tid];
      const float x = Elem<Bits>::to_float(b);
      if (x > candidate_threshold_value<Bits>(thr)) {
        const int slot = atomicAdd(&s_cand, 1);
        if (slot < kCandCap)
          cand[slot] = ((unsigned long long)b << 32) | (uint32_t)(c0 + nv * VEC + tid);
        cmx = fmaxf(cmx, x);
      } else {
        z_t += fast_exp2(fmaf(x, coef, shift));
      }
    }
    cmx = warp_max(cmx);
    if (lane == 0) s_wmax[g & 1][warp] = cmx;
    __syncthreads();  // stage consumed, candidate maxima and count published
    float m_new = m_ref;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) m_new = fmaxf(m_new, s_wmax[g & 1][w]);
    if (!(m_new < INFINITY)) m_new = m_ref;  // a +inf candidate: the row is flagged later
    if (tid == 0) issue(g + kStages);
    if (m_new > m_ref) {
      z_t = (m_ref == -INFINITY) ? 0.f : z_t * fast_exp2((m_ref - m_new) * coef);
      shift = -m_new * coef;
    }
    if (s_cand > kCandCap / 2 &&
        (m_new > m_ref || (a.use_top_p && narrowed < max_narrowings))) {
      // Keep the buffer at most half full: drop what fell below the window
      // (the maximum may have risen), narrowing the window if needed.
      compact_candidates<Bits>(cand, &s_cand, s_keep, m_new - off, m_new, coef, zd_t, zd_ref);
      while (a.use_top_p && s_cand > kCandCap / 2 && s_cand <= kCandCap &&
             narrowed < max_narrowings) {
        ++narrowed;
        off = (kWindowLog2 - kWindowStepLog2 * (float)narrowed) / coef;
        compact_candidates<Bits>(cand, &s_cand, s_keep, m_new - off, m_new, coef, zd_t, zd_ref);
      }
    }
    m_ref = m_new;
    if (k != nck - 1) continue;

    // ---- end of row r ---------------------------------------------------
    // Every element is either a non-candidate (<= m_ref) or a candidate, so
    // the row maximum is the larger of m_ref and the largest candidate.
    float cm = -INFINITY;
    for (int j = tid; j < min(s_cand, kCandCap); j += kThreads)
      cm = fmaxf(cm, Elem<Bits>::to_float((uint32_t)(cand[j] >> 32)));
    const float M = fmaxf(m_ref, block_max_all(cm, s_f));
    int32_t flags = 0;
    const bool overflow = s_cand > kCandCap;
    if (a.use_top_p) {
      // Candidates below the final window leave the buffer (their mass is
      // small: fp32 relative to M); the rest are the only elements that can
      // be at or above the top-p threshold.
      compact_candidates<Bits>(cand, &s_cand, s_keep, M - off, M, coef, zd_t, zd_ref);
    }
    float zl = (m_ref == -INFINITY || !(M < INFINITY)) ? 0.f : z_t * fast_exp2((m_ref - M) * coef);
    if (z_t != z_t) zl = z_t;  // a NaN logit poisons the sum (flagged below)
    if (zd_ref != -INFINITY) zl += zd_t * fast_exp2((zd_ref - M) * coef);
    const double z_light = block_sum_all((double)zl, s_d);
    const int n_in = min(s_cand, kCandCap);
    double Z = z_light, zp = z_light;
    uint32_t tau_bits = Elem<Bits>::kNegInf;
    int n_nuc = 0;
    if (!a.use_top_p) {
      // the few elements that rose above the running reference
      unsigned long long zc = 0ull;
      for (int j = tid; j < n_in; j += kThreads)
        zc += __double2ull_rn(
            exact_exp2d(Elem<Bits>::to_float((uint32_t)(cand[j] >> 32)), M, a.coef64) * kFixD);
      Z = z_light + (double)block_sum_all(zc, s_u) / kFixD;
      zp = Z;
      if (overflow) flags |= kRowNeedGeneral;
    } else if (overflow || n_in > kCandCap / 2 || !(M > -INFINITY)) {
      flags |= kRowNeedGeneral;
    } else {
      // Exact masses (2^-40 fixed point, order-independent sums) into the
      // idle half of the buffer; entries rewritten as (key << 32 | index).
      unsigned long long *cmass = cand + kCandCap / 2;
      unsigned long long zin = 0ull;
      for (int j = tid; j < n_in; j += kThreads) {
        const unsigned long long e = cand[j];
        const uint32_t b = (uint32_t)(e >> 32);
        const unsigned long long fx =
            __double2ull_rn(exact_exp2d(Elem<Bits>::to_float(b), M, a.coef64) * kFixD);
        cmass[j] = fx;
        zin += fx;
        cand[j] = ((unsigned long long)Elem<Bits>::key(b) << 32) | (e & 0xFFFFFFFFull);
      }
      zin = block_sum_all(zin, s_u);  // (its barriers also publish cmass / cand)
      Z = z_light + (double)zin / kFixD;
      zp = Z;
      const unsigned long long target = (unsigned long long)ceil((double)a.s.top_p * Z * kFixD);
      if (zin < target) {
        flags |= kRowNeedGeneral;  // the window holds less than top_p of the mass
      } else {
        // Top-p threshold: the largest key t whose suffix mass S(t) reaches
        // top_p of the total; binary search, one barrier per step.
        uint64_t lo = 0, hi = 1ull << KEYB;
        unsigned long long s_lo = zin;
        int par = 0;
        while (hi - lo > 1) {
          const uint64_t mid = (lo + hi) >> 1;
          unsigned long long part = 0ull;
          for (int j = tid; j < n_in; j += kThreads)
            if ((cand[j] >> 32) >= mid) part += cmass[j];
          part = warp_sum_any(part);
          if (lane == 0) s_bs[par][warp] = part;
          __syncthreads();
          unsigned long long S = 0ull;
#pragma unroll
          for (int w = 0; w < kWarps; ++w) S += s_bs[par][w];
          par ^= 1;
          if (S >= target) {
            lo = mid;
            s_lo = S;
          } else {
            hi = mid;
          }
        }
        zp = (double)s_lo / kFixD;
        tau_bits = key_to_bits<Bits>((uint32_t)lo);
        // the nucleus: every candidate with key >= tau, as (bits << 32 | index)
        if (tid == 0) s_nuc = 0;
        __syncthreads();
        uint64_t *nuc = a.nuc + r * (int64_t)kNucCap;
        for (int j = tid; j < n_in; j += kThreads) {
          const unsigned long long e = cand[j];
          const uint32_t key = (uint32_t)(e >> 32);
          if (key >= (uint32_t)lo) {
            const int slot = atomicAdd(&s_nuc, 1);
            if (slot < kNucCap)
              nuc[slot] = ((unsigned long long)key_to_bits<Bits>(key) << 32) | (e & 0xFFFFFFFFull);
          }
        }
        __syncthreads();
        n_nuc = s_nuc;
        if (n_nuc > kNucCap) flags |= kRowNeedGeneral;
      }
    }
    if (M == -INFINITY || !(fabsf(M * coef) < INFINITY) || !(Z < INFINITY)) flags |= kRowNonfinite;
    if (tid == 0) {
      RowRecord rec;
      rec.m = M;
      rec.flags = flags;
      rec.z = Z;
      rec.zp = zp;
      rec.tau_bits = tau_bits;
      rec.n_nuc = n_nuc;
      a.rowrec[r] = rec;
    }
    __syncthreads();  // candidate buffer and counters free for the next row
  }
  // (NaN / +inf logits surface as non-finite row statistics, reported by
  // unit_decide; a bounded wait that gave up is reported here.)
  const bool any_timeout = __syncthreads_or(timed_out);
  if (tid == 0 && any_timeout && a.s.dev_status) atomicOr(a.s.dev_status, PSI_DEV_TIMEOUT);
}

// ---------------------------------------------------------------------------
// unit_decide
// ---------------------------------------------------------------------------

// In-place ascending bitonic sort of n (a power of two) 64-bit keys.
__device__ void bitonic_sort(unsigned long long *v, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = threadIdx.x; t < n; t += blockDim.x) {
        const int p = t ^ j;
        if (p > t) {
          const bool up = (t & k) == 0;
          const unsigned long long a = v[t], b = v[p];
          if ((a > b) == up) {
            v[t] = b;
            v[p] = a;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Inclusive prefix sums of w[0..n) in index order (deterministic), in place.
__device__ void block_scan(double *w, int n, double *scratch) {
  const int per = (n + kUnitThreads - 1) / kUnitThreads;
  const int b0 = threadIdx.x * per, b1 = min(n, b0 + per);
  double run = 0.0;
  for (int j = b0; j < b1; ++j) {
    run += w[j];
    w[j] = run;
  }
  // exclusive scan of the per-thread totals
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  double off = incl - run;
  for (int w2 = 0; w2 < warp; ++w2) off += scratch[w2];
  for (int j = b0; j < b1; ++j) w[j] += off;
  __syncthreads();
}

template <typename Bits>
__global__ void __launch_bounds__(kUnitThreads) unit_decide_kernel(const FastArgs a) {
  __shared__ unsigned long long ent[kNucCap];
  __shared__ double wv[kNucCap];
  __shared__ double scratch[kUnitThreads / 32];
  __shared__ int s_need;
  const int tid = threadIdx.x;
  const SampledArgs &s = a.s;
  const int32_t B = s.B, N = s.N, V = s.V;
  const int64_t unit = blockIdx.x;
  const int32_t n = (int32_t)(unit / (B + 1)), i = (int32_t)(unit % (B + 1));
  const bool has_q = i < B;
  const int64_t rp_idx = unit;
  const int64_t rq_idx = (int64_t)N * (B + 1) + (int64_t)n * B + i;
  const RowRecord rp = a.rowrec[rp_idx];
  RowRecord rq = rp;
  if (has_q) rq = a.rowrec[rq_idx];
  const bool general = ((rp.flags | (has_q ? rq.flags : 0)) & kRowNeedGeneral) != 0;
  if (general) {  // the cluster kernel verifies this unit (records included)
    if (tid == 0) a.list_a[atomicAdd(&a.counters[0], 1)] = (int32_t)unit;
    return;
  }
  const uint64_t seq = s.seq_ids ? s.seq_ids[n] : (uint64_t)n;
  const Bits *row_p = static_cast<const Bits *>(s.ar) + unit * s.ar_stride;
  const Bits *row_q = has_q ? static_cast<const Bits *>(s.draft) + ((int64_t)n * B + i) * s.draft_stride
                            : nullptr;
  const float tau_p = Elem<Bits>::to_float(rp.tau_bits);
  const float tau_q = Elem<Bits>::to_float(rq.tau_bits);

  if (tid == 0) {
    int need = 1;
    if (has_q) {
      const int32_t x = s.ids[(int64_t)n * B + i];
      double p = 0.0, q = 0.0;
      const bool valid = x >= 0 && x < V;
      if (valid) {
        const float xp = Elem<Bits>::to_float(row_p[x]);
        const float xq = Elem<Bits>::to_float(row_q[x]);
        if (xp >= tau_p && rp.zp > 0.0) p = exact_exp2d(xp, rp.m, a.coef64) / rp.zp;
        if (xq >= tau_q && rq.zp > 0.0) q = exact_exp2d(xq, rq.m, a.coef64) / rq.zp;
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
    if (((rp.flags | (has_q ? rq.flags : 0)) & kRowNonfinite) && s.dev_status)
      atomicOr(s.dev_status, PSI_DEV_NONFINITE);
    s_need = need;
  }
  __syncthreads();
  if (!s_need) return;
  if (!a.use_top_p) {  // the draw needs whole rows: decided after the emit step
    if (tid == 0) a.rec[unit].token = -2;
    return;
  }

  // ---- correction / bonus draw over p's nucleus ----------------------------
  const int nn = rp.n_nuc;
  int np2 = 1;
  while (np2 < nn) np2 <<= 1;
  const uint64_t *nuc = a.nuc + rp_idx * (int64_t)kNucCap;
  for (int t = tid; t < np2; t += kUnitThreads) {
    if (t < nn) {
      const uint64_t e = nuc[t];  // (bits << 32) | index  ->  (index << 32) | bits
      ent[t] = ((e & 0xFFFFFFFFull) << 32) | (e >> 32);
    } else {
      ent[t] = ~0ull;
    }
  }
  __syncthreads();
  bitonic_sort(ent, np2);  // vocabulary order
  for (int pass = 0; pass < 2; ++pass) {
    const bool p_only = !has_q || pass == 1;
    for (int t = tid; t < nn; t += kUnitThreads) {
      const int32_t v = (int32_t)(ent[t] >> 32);
      const float xp = Elem<Bits>::to_float((uint32_t)(ent[t] & 0xFFFFFFFFull));
      double w = exact_exp2d(xp, rp.m, a.coef64) / rp.zp;
      if (!p_only) {
        const float xq = Elem<Bits>::to_float(row_q[v]);
        const double q = (xq >= tau_q && rq.zp > 0.0) ? exact_exp2d(xq, rq.m, a.coef64) / rq.zp : 0.0;
        w = w > q ? w - q : 0.0;
      }
      wv[t] = w;
    }
    __syncthreads();
    block_scan(wv, nn, scratch);
    const double W = nn > 0 ? wv[nn - 1] : 0.0;
    if (W > 0.0 || p_only) {
      if (tid == 0) {
        int32_t token = 0;
        if (W > 0.0) {
          const double u2 = (double)uniform24(s.seed, seq, s.step, (uint64_t)i, PSI_PURPOSE_RESID);
          const double t = u2 * W;
          int lo = 0, hi = nn;  // first j with wv[j] > t
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (wv[mid] > t) hi = mid;
            else lo = mid + 1;
          }
          if (lo >= nn) {  // rounding: the last entry with positive weight
            lo = nn - 1;
            while (lo > 0 && !(wv[lo] > wv[lo - 1])) --lo;
          }
          token = (int32_t)(ent[lo] >> 32);
        }
        a.rec[unit].token = token;
      }
      break;
    }
    __syncthreads();  // residual vanished: draw from p itself
  }
}

// ---------------------------------------------------------------------------
// fast_emit: one thread per sequence.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) fast_emit_kernel(const FastArgs a) {
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

int sm_count() {
  static int count = 0;
  if (count == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        count <= 0)
      count = 148;
  }
  return count;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

template <typename Bits>
cudaError_t launch_fast_typed(const FastArgs &fa, const SampledPlan &plan, const KernelEvents &ev,
                              cudaStream_t stream) {
  const size_t smem = (size_t)kStages * kChunkBytes + sizeof(unsigned long long) * kCandCap;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(row_stats_kernel<Bits>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int64_t grid1 = std::min<int64_t>(fa.rows, (int64_t)sm_count() * 2);
  cudaError_t e;
  if (ev.before && (e = cudaEventRecord(ev.before, stream)) != cudaSuccess) return e;
  row_stats_kernel<Bits><<<(unsigned)grid1, kThreads, smem, stream>>>(fa);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (ev.after && (e = cudaEventRecord(ev.after, stream)) != cudaSuccess) return e;
  const int64_t units = (int64_t)fa.s.N * (fa.s.B + 1);
  unit_decide_kernel<Bits><<<(unsigned)units, kUnitThreads, 0, stream>>>(fa);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const psi_dtype dt = sizeof(Bits) == 2 ? PSI_DTYPE_BF16 : PSI_DTYPE_F32;
  SampledArgs sa = fa.s;
  sa.records = fa.rec;
  const int clusters_a = (int)std::min<int64_t>(units, kListClusters);
  e = launch_cluster_list(sa, dt, plan, 1, fa.list_a, fa.counters + 0, clusters_a, stream);
  if (e != cudaSuccess) return e;
  fast_emit_kernel<<<(fa.s.N + 127) / 128, 128, 0, stream>>>(fa);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int clusters_b = std::min(fa.s.N, kListClusters);
  return launch_cluster_list(sa, dt, plan, 2, fa.list_b, fa.counters + 1, clusters_b, stream);
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
  L.nuc_off = off;
  off = align256(off + sizeof(uint64_t) * (size_t)rows * kNucCap);
  L.counters_off = off;
  off = align256(off + sizeof(int32_t) * 4);
  L.list_a_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)units);
  L.list_b_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)N);
  L.total = off;
  return L;
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
  fa.win_off = kWindowLog2 / fa.coef;
  fa.use_top_p = a.top_p < 1.0f ? 1 : 0;
  fa.rec = reinterpret_cast<UnitRecord *>(ws + L.rec_off);
  fa.rowrec = reinterpret_cast<RowRecord *>(ws + L.rows_off);
  fa.nuc = reinterpret_cast<uint64_t *>(ws + L.nuc_off);
  fa.counters = reinterpret_cast<int32_t *>(ws + L.counters_off);
  fa.list_a = reinterpret_cast<int32_t *>(ws + L.list_a_off);
  fa.list_b = reinterpret_cast<int32_t *>(ws + L.list_b_off);
  fa.s.records = fa.rec;
  if (dtype == PSI_DTYPE_BF16) return launch_fast_typed<uint16_t>(fa, plan, ev, stream);
  return launch_fast_typed<uint32_t>(fa, plan, ev, stream);
}

}  // namespace psi
