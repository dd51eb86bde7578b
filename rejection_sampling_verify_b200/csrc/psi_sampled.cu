// psi_sampled.cu - linear verify with temperature > 0 (speculative rejection
// sampling with optional top-p).
//
// Sources (page title, section):
//  "Uno Psi-Spec 是什麼？Diffusion-Augmented LLM 如何保留 AR 分布、一次驗證多個
//  Token" (alphalab.site), "Uno Psi-Spec 怎麼運作？完整走一次四個 Token": step 3
//  (the frozen AR scores the block and applies the rejection rule keeping the
//  longest accepted prefix), step 4 (the first rejected position is replaced
//  by a draw from the corrected residual), and the following paragraph (a
//  bonus token from the block-end logits when every draft passes);
//  "想跑 Uno：先確認官方程式需要的環境" (temperature and top-p are sampler
//  settings on the run card).  "Uno / Psi-Spec - 같은 모델 안에서 초안 뽑고 AR로
//  도장 찍기" (lanes-ecd.pages.dev), "어디서 왔나": the rule is the draft ->
//  verify -> correct construction of Leviathan et al. (2023).
//
// Design.  One thread-block cluster of C CTAs handles one (sequence, row)
// unit: AR row i with draft row i (i < B), or the bonus AR row B alone.  CTA
// k of the cluster brings its 1/C slice of both rows into its own shared
// memory ONCE (bulk copies, no multicast, when the slice starts on a 16-byte
// boundary; element loads otherwise); every later pass (max, sum of exponentials,
// top-p radix select, the correction / bonus draw) reads shared memory, and
// the cluster combines per-CTA partials through distributed shared memory.
// Each unit decides its own draft (accept or reject) redundantly in every
// CTA, and a rejected row (or the bonus row) draws its correction while the
// row pair is still on chip, so no logit is read from HBM twice.  A small
// second kernel finds the first rejected row of each sequence and emits.
//
// Probabilities: e(v) = 2^((x_v - m) * log2(e)/T) with m the row maximum,
// p(v) = e(v) / Z.  Top-p: the threshold is a logit value tau found by a
// most-significant-digit radix select over the order-preserving integer key
// of the logit (bf16: 9 + 7 bits), weighted by e(v) in 2^-40 fixed point
// (exact integer sums, independent of summation order).  Only elements with
// e(v) > (1 - top_p) / (2V) can be at or above the threshold, so only those
// are histogrammed.
#include "psi_internal.h"

namespace psi {

namespace {

constexpr int kBins = 512;                         // radix bins per level (9 bits)
constexpr int kModeGrid = 0;    // one unit per cluster, units in grid order
// (kClusterModeList / kClusterModeSample: the list modes, see psi_internal.h)
constexpr int kModeSample = kClusterModeSample;
constexpr float kFixScale = 1099511627776.0f;      // 2^40
constexpr double kFixScaleD = 1099511627776.0;     // 2^40
constexpr double kFixInv = 1.0 / 1099511627776.0;  // 2^-40
// Relative to the row maximum, elements with e > 2^-12 carry most of the
// mass; with top-p their e(v) is re-evaluated in double precision so that
// the threshold decision agrees with an exact computation to ~1e-9.
constexpr float kExactAbove = 2.44140625e-04f;     // 2^-12
// First, narrow top-p window: elements with e > 2^-16 (usually ~1% of the
// vocabulary).  It is used whenever its mass alone reaches top_p.
constexpr float kNarrowWindow = 1.52587890625e-05f;  // 2^-16

template <typename Bits>
struct RadixLevels;
template <>
struct RadixLevels<uint16_t> {
  static constexpr int kCount = 2;
  __device__ static constexpr int bits(int l) { return l == 0 ? 9 : 7; }
};
template <>
struct RadixLevels<uint32_t> {
  static constexpr int kCount = 4;
  __device__ static constexpr int bits(int l) { return l < 3 ? 9 : 5; }
};

// Values other CTAs of the cluster read through DSMEM.  Every field is
// written once per kernel, before the cluster barrier that publishes it.
struct Xchg {
  float max_part[2];
  float zlo_part[2];                   // fp32 part of the sum of exponentials
  double zhi_part[2];                  // double part (top-p only)
  unsigned long long zwin_part[2];     // fixed-point mass inside the narrow window
  unsigned long long block_sum[4][2];  // radix level, row
  unsigned long long w_part[2];        // [0] first draw, [1] fallback draw (fixed point)
};

struct Broadcast {  // CTA-local results shared after __syncthreads
  float m[2];
  double z[2];
  float window[2];  // top-p histogram window for this row
  double zp[2];    // normaliser after top-p (Z without top-p)
  float tau[2];    // keep v iff logit >= tau (-inf: keep all)
  unsigned long long above[2];
  unsigned long long target[2];
  uint32_t prefix[2];
  int need_sample;
  int cross_rank;
  unsigned long long t_local;
  unsigned long long w_total;
  int use_p_only;
};

// Fixed-point (2^-40) mass of one element for the top-p histograms: the
// fp32 value, or for the heavy elements the double-precision one.  Every
// pass uses this same function, so bins of different levels add up exactly.
__device__ __forceinline__ double exact_exp2(float x, float m, double coef64) {
  return exp2(((double)x - (double)m) * coef64);
}

__device__ __forceinline__ unsigned long long fixed_mass(float x, float e, float m,
                                                         double coef64) {
  if (e > kExactAbove) return __double2ull_rn(exact_exp2(x, m, coef64) * kFixScaleD);
  return __float2ull_rn(e * kFixScale);
}

template <typename T>
__device__ __forceinline__ T warp_sum_t(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Sum over the CTA (any arithmetic type); result valid in warp 0.
template <typename T>
__device__ __forceinline__ T block_sum_t(T v, T *scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_t(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  T r = T(0);
  if (warp == 0) r = warp_sum_t(lane < kWarps ? scratch[lane] : T(0));
  return r;
}

__device__ __forceinline__ float block_max(float v, float *scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  float r = -INFINITY;
  if (warp == 0) {
    r = lane < kWarps ? scratch[lane] : -INFINITY;
    r = warp_max(r);
  }
  return r;
}

// Largest finite-or-(-inf) value in a 16-byte vector; NaN/+inf set `bad`.
template <typename Bits>
__device__ __forceinline__ float vec_max(const uint4 &w, bool &bad) {
  float vm;
  if constexpr (sizeof(Bits) == 2) {
    const __nv_bfloat162 m = __hmax2_nan(
        __hmax2_nan(*reinterpret_cast<const __nv_bfloat162 *>(&w.x),
                    *reinterpret_cast<const __nv_bfloat162 *>(&w.y)),
        __hmax2_nan(*reinterpret_cast<const __nv_bfloat162 *>(&w.z),
                    *reinterpret_cast<const __nv_bfloat162 *>(&w.w)));
    vm = __bfloat162float(__hmax_nan(__low2bfloat16(m), __high2bfloat16(m)));
  } else {
    const float a = __uint_as_float(w.x), b = __uint_as_float(w.y);
    const float c = __uint_as_float(w.z), d = __uint_as_float(w.w);
    vm = (a != a || b != b || c != c || d != d) ? NAN : fmaxf(fmaxf(a, b), fmaxf(c, d));
  }
  if (!(vm < INFINITY)) {
    vm = -INFINITY;
#pragma unroll
    for (int k = 0; k < Elem<Bits>::kVec; ++k) {
      const uint32_t b = vec_elem<Bits>(w, k);
      bad |= Elem<Bits>::bad(b);
      vm = fmaxf(vm, Elem<Bits>::to_float(b));  // fmaxf skips NaN
    }
  }
  return vm;
}

// The radix crossing search for one row, run by one full warp.
//   level_bits   bins at this level = 1 << level_bits
//   hist_owned   this CTA's owner-reduced bins (same layout in every CTA)
// Updates bc->above / bc->prefix; on the last level sets bc->zp, bc->tau.
template <typename Bits>
__device__ void radix_crossing(int r, int level, int level_bits, bool last, uint32_t C,
                               Xchg *xc, unsigned long long *owned, int per,
                               Broadcast *bc) {
  const int lane = threadIdx.x & 31;
  const unsigned long long target = bc->target[r];
  unsigned long long above = bc->above[r];
  const unsigned long long bs =
      (uint32_t)lane < C ? dsmem_ld_u64(dsmem_map(&xc->block_sum[level][r], lane)) : 0ull;
  // suffix sums over ranks: suf_k = sum_{k' >= k} bs_k'
  unsigned long long suf = bs;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long t = __shfl_down_sync(0xFFFFFFFFu, suf, o);
    if (lane + o < 32) suf += t;
  }
  const unsigned crossing = __ballot_sync(0xFFFFFFFFu, (uint32_t)lane < C && above + suf >= target);
  int kstar;
  bool fallback = false;
  if (crossing) {
    kstar = 31 - __clz(crossing);
  } else {  // rounding left the target out of reach: keep every in-window bin
    const unsigned nz = __ballot_sync(0xFFFFFFFFu, (uint32_t)lane < C && bs != 0ull);
    kstar = nz ? __ffs(nz) - 1 : 0;
    fallback = true;
  }
  const unsigned long long suf_k = __shfl_sync(0xFFFFFFFFu, suf, kstar);
  const unsigned long long bs_k = __shfl_sync(0xFFFFFFFFu, bs, kstar);
  const int nbins = 1 << level_bits;
  const int b_lo = kstar * per;
  const int b_hi = min(nbins, b_lo + per);  // exclusive
  unsigned long long run = above + (suf_k - bs_k);  // mass of all higher ranks
  int bstar = b_lo;
  unsigned long long mass_b = 0;
  if (!fallback) {
    for (int top = b_hi; top > b_lo; top -= 32) {
      const int b = top - 1 - lane;
      const unsigned long long v =
          b >= b_lo ? dsmem_ld_u64(dsmem_map(&owned[r * per + (b - b_lo)], kstar)) : 0ull;
      unsigned long long pre = v;  // inclusive prefix from the highest bin down
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long t = __shfl_up_sync(0xFFFFFFFFu, pre, o);
        if (lane >= o) pre += t;
      }
      const unsigned hit = __ballot_sync(0xFFFFFFFFu, b >= b_lo && run + pre >= target);
      if (hit) {
        const int l = __ffs(hit) - 1;
        bstar = top - 1 - l;
        const unsigned long long pre_l = __shfl_sync(0xFFFFFFFFu, pre, l);
        mass_b = __shfl_sync(0xFFFFFFFFu, v, l);
        run = run + pre_l - mass_b;
        break;
      }
      run += __shfl_sync(0xFFFFFFFFu, pre, 31);
    }
    // Integer sums are exact, so the crossing always lies inside rank kstar.
  } else {
    // lowest non-empty bin of rank kstar; everything above it is kept
    bool found = false;
    for (int base = b_lo; base < b_hi && !found; base += 32) {
      const int b = base + lane;
      const unsigned long long v =
          b < b_hi ? dsmem_ld_u64(dsmem_map(&owned[r * per + (b - b_lo)], kstar)) : 0ull;
      const unsigned nz = __ballot_sync(0xFFFFFFFFu, v != 0ull);
      if (nz) {
        const int l = __ffs(nz) - 1;
        bstar = base + l;
        mass_b = __shfl_sync(0xFFFFFFFFu, v, l);
        found = true;
      }
    }
    // mass above the kept bin: everything in the window except that bin
    unsigned long long all = __shfl_sync(0xFFFFFFFFu, suf, 0);
    run = above + all - mass_b;
  }
  if (lane == 0) {
    bc->above[r] = run;
    bc->prefix[r] = (bc->prefix[r] << level_bits) | (uint32_t)bstar;
    if (last) {
      bc->zp[r] = (double)(run + mass_b) * kFixInv;
      // threshold logit: the value whose key is the full prefix
      const uint32_t key = bc->prefix[r];
      uint32_t bits;
      if constexpr (sizeof(Bits) == 2) {
        bits = (key & 0x8000u) ? (key & 0x7FFFu) : (~key & 0xFFFFu);
        bc->tau[r] = __uint_as_float(bits << 16);
      } else {
        bits = (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
        bc->tau[r] = __uint_as_float(bits);
      }
    }
  }
  __syncwarp();
}

}  // namespace

template <typename Bits>
__global__ void __launch_bounds__(kThreads) sampled_unit_kernel(SampledArgs a, SampledPlan plan,
                                                                 float coef, double coef64,
                                                                 float w_min, float w_narrow,
                                                                 int use_top_p, int mode,
                                                                 const int32_t *work_list,
                                                                 const int32_t *work_count) {
  pdl_wait();  // the previous kernel's results are visible
  pdl_trigger();
  constexpr int VEC = Elem<Bits>::kVec;
  extern __shared__ __align__(128) unsigned char dyn_smem[];
  __shared__ Xchg xc;
  __shared__ Broadcast bc;
  __shared__ __align__(8) uint64_t mbar;
  __shared__ float scratch[kWarps];
  __shared__ float scratch2[kWarps];
  __shared__ double scratch_d[kWarps];
  __shared__ unsigned long long scratch_u[kWarps];
  __shared__ uint32_t s_x_bits[2];
  __shared__ int32_t s_x;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_rank();
  const uint32_t C = cluster_size();
  const int32_t B = a.B, V = a.V;
  if (tid == 0) {
    mbar_init(&mbar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // kModeGrid: cluster k handles unit k.  kModeList / kModeSample: the
  // clusters of a small persistent grid walk a device-side list of units.
  const int64_t n_items = mode == kModeGrid ? (int64_t)a.N * (B + 1) : (int64_t)*work_count;
  const int64_t first = blockIdx.x / C, stride = gridDim.x / C;
  uint32_t parity = 0;
  for (int64_t item = first; item < n_items; item += stride, parity ^= 1u) {
  const int64_t unit = mode == kModeGrid ? item : (int64_t)work_list[item];
  const int32_t n = (int32_t)(unit / (B + 1));
  const int32_t i = (int32_t)(unit % (B + 1));
  const bool has_q = i < B;
  const Bits *row_p = static_cast<const Bits *>(a.ar) + ((int64_t)n * (B + 1) + i) * a.ar_stride;
  const Bits *row_q =
      has_q ? static_cast<const Bits *>(a.draft) + ((int64_t)n * B + i) * a.draft_stride : nullptr;
  const int32_t S = plan.slice;
  const int32_t c0 = (int32_t)rank * S;
  const int32_t len = max(0, min(V, c0 + S) - c0);
  const int32_t nvp = plan.nvec_pad;
  const int32_t nchunks = nvp / 32;
  const uint64_t seq = a.seq_ids ? a.seq_ids[n] : (uint64_t)n;

  Bits *buf_p = reinterpret_cast<Bits *>(dyn_smem);
  Bits *buf_q = buf_p + (size_t)nvp * VEC;
  unsigned long long *hist = reinterpret_cast<unsigned long long *>(buf_q + (size_t)nvp * VEC);
  const int per_max = (kBins + (int)C - 1) / (int)C;
  unsigned long long *owned = hist + 2 * kBins;
  unsigned long long *chunk_sum = owned + 2 * per_max;

  // ---- 1. one bulk copy per row slice into shared memory -------------------
  const bool aligned = ((reinterpret_cast<uintptr_t>(row_p + c0) & 15u) == 0) &&
                       (!has_q || (reinterpret_cast<uintptr_t>(row_q + c0) & 15u) == 0);
  const int32_t bulk = aligned ? (len / VEC) * VEC : 0;
  if (tid == 0) {  // completes this item's phase (at once when nothing is copied)
    const uint32_t bytes = (uint32_t)bulk * sizeof(Bits);
    mbar_arrive_expect_tx(&mbar, bytes * (has_q ? 2u : 1u));
    for (uint32_t off = 0; off < bytes; off += 32768u) {
      const uint32_t piece = min(32768u, bytes - off);
      bulk_load(reinterpret_cast<char *>(buf_p) + off,
                reinterpret_cast<const char *>(row_p + c0) + off, piece, &mbar);
      if (has_q)
        bulk_load(reinterpret_cast<char *>(buf_q) + off,
                  reinterpret_cast<const char *>(row_q + c0) + off, piece, &mbar);
    }
  }
  // the drafted id and its two logits, needed for the decision (warp 1)
  if (tid == 32) {
    int32_t x = -1;
    uint32_t bp = 0, bq = 0;
    if (has_q) {
      x = a.ids[(int64_t)n * B + i];
      if (x >= 0 && x < V) {
        bp = row_p[x];
        bq = row_q[x];
      }
    }
    s_x = x;
    s_x_bits[0] = bp;
    s_x_bits[1] = bq;
  }
  // ragged tail of the slice and -inf padding up to whole warp chunks
  for (int32_t v = bulk + tid; v < nvp * VEC; v += kThreads) {
    buf_p[v] = v < len ? row_p[c0 + v] : (Bits)Elem<Bits>::kNegInf;
    if (has_q) buf_q[v] = v < len ? row_q[c0 + v] : (Bits)Elem<Bits>::kNegInf;
  }
  if (use_top_p)
    for (int t = tid; t < 2 * kBins; t += kThreads) hist[t] = 0ull;
  __syncthreads();
  bool timed_out = false;
  timed_out = !mbar_wait_bounded(&mbar, parity);

  const uint4 *vp = reinterpret_cast<const uint4 *>(buf_p);
  const uint4 *vq = reinterpret_cast<const uint4 *>(buf_q);

  // ---- 2. row maxima ------------------------------------------------------
  bool bad = false;
  {
    float mp = -INFINITY, mq = -INFINITY;
    for (int32_t j = tid; j < nvp; j += kThreads) {
      mp = fmaxf(mp, vec_max<Bits>(vp[j], bad));
      if (has_q) mq = fmaxf(mq, vec_max<Bits>(vq[j], bad));
    }
    mp = block_max(mp, scratch);
    mq = block_max(mq, scratch2);
    if (tid == 0) {
      xc.max_part[0] = mp;
      xc.max_part[1] = mq;
    }
  }
  cluster_sync();
  if (warp == 0) {
    float mp = (uint32_t)lane < C ? dsmem_ld_f32(dsmem_map(&xc.max_part[0], lane)) : -INFINITY;
    float mq = (uint32_t)lane < C ? dsmem_ld_f32(dsmem_map(&xc.max_part[1], lane)) : -INFINITY;
    mp = warp_max(mp);
    mq = warp_max(mq);
    if (lane == 0) {
      bc.m[0] = mp;
      bc.m[1] = mq;
    }
  }
  __syncthreads();
  const int nrows = has_q ? 2 : 1;
  // -m * coef per row, with an all -inf row mapped to probability 0
  const float shift_p = bc.m[0] == -INFINITY ? -INFINITY : -bc.m[0] * coef;
  const float shift_q = bc.m[1] == -INFINITY ? -INFINITY : -bc.m[1] * coef;
  for (int r = 0; r < nrows; ++r) {
    const float m = bc.m[r];
    if (m == -INFINITY || !(fabsf(m * coef) < INFINITY)) bad = true;
  }

  // ---- 3. sum of exponentials (+ level-1 top-p histogram) ------------------
  const int shift1 = Elem<Bits>::kKeyBits - RadixLevels<Bits>::bits(0);
  for (int r = 0; r < nrows; ++r) {
    const uint4 *src = r == 0 ? vp : vq;
    const float m = bc.m[r];
    float zlo = 0.f;
    double zhi = 0.0;
    unsigned long long zwin = 0ull;
    if (!use_top_p) {
      // without top-p, Z normalises the whole-row draw: fp32 exponentials,
      // summed in fp32 per vector and in double per thread (the streaming
      // path's Z has the same fp32 accuracy)
      if (m > -INFINITY)
        for (int32_t j = tid; j < nvp; j += kThreads) {
          const uint4 w = src[j];
          float part = 0.f;
#pragma unroll
          for (int k = 0; k < VEC; ++k)
            part += fast_exp2(fmaf(Elem<Bits>::to_float(vec_elem<Bits>(w, k)), coef,
                                   r == 0 ? shift_p : shift_q));
          zhi += (double)part;
        }
    } else {
      for (int32_t j = tid; j < nvp; j += kThreads) {
        const uint4 w = src[j];
        float part = 0.f;
#pragma unroll
        for (int k = 0; k < VEC; ++k) {
          const uint32_t b = vec_elem<Bits>(w, k);
          const float x = Elem<Bits>::to_float(b);
          const float e = fast_exp2(fmaf(x, coef, (r == 0 ? shift_p : shift_q)));
          if (e > w_narrow) {
            const unsigned long long fx = fixed_mass(x, e, m, coef64);
            if (e > kExactAbove) zhi += exact_exp2(x, m, coef64);
            else part += e;
            atomicAdd(&hist[r * kBins + (Elem<Bits>::key(b) >> shift1)], fx);
            zwin += fx;
          } else {
            part += e;
          }
        }
        zlo += part;
      }
    }
    zlo = block_sum_t(zlo, scratch);
    zhi = block_sum_t(zhi, scratch_d);
    zwin = block_sum_t(zwin, scratch_u);
    if (tid == 0) {
      xc.zlo_part[r] = zlo;
      xc.zhi_part[r] = zhi;
      xc.zwin_part[r] = zwin;
    }
  }
  __syncthreads();  // level-1 histograms complete
  cluster_sync();
  if (warp < 2) {  // warp r reduces row r
    const int r = warp;
    const bool on = (uint32_t)lane < C && r < nrows;
    double z = on ? (double)dsmem_ld_f32(dsmem_map(&xc.zlo_part[r], lane)) : 0.0;
    double zh = on ? dsmem_ld_f64(dsmem_map(&xc.zhi_part[r], lane)) : 0.0;
    unsigned long long zw = on ? dsmem_ld_u64(dsmem_map(&xc.zwin_part[r], lane)) : 0ull;
    z = warp_sum_t(z) + warp_sum_t(zh);
    zw = warp_sum_t(zw);
    if (lane == 0) {
      bc.z[r] = z;
      bc.zp[r] = z;
      bc.tau[r] = -INFINITY;
      bc.above[r] = 0ull;
      bc.prefix[r] = 0u;
      // smallest fixed-point mass that reaches top_p of the total
      const unsigned long long target = (unsigned long long)ceil((double)a.top_p * z * kFixScaleD);
      bc.target[r] = target;
      bc.window[r] = (zw >= target || !(r < nrows)) ? w_narrow : w_min;
    }
  }
  __syncthreads();

  // Rows whose narrow window cannot reach top_p rebuild their level-1
  // histogram over the wide window (same decision in every CTA).
  if (use_top_p && (bc.window[0] < w_narrow || bc.window[1] < w_narrow)) {
    for (int r = 0; r < nrows; ++r) {
      if (!(bc.window[r] < w_narrow)) continue;
      for (int t = tid; t < kBins; t += kThreads) hist[r * kBins + t] = 0ull;
      __syncthreads();
      const uint4 *src = r == 0 ? vp : vq;
      const float m = bc.m[r];
      for (int32_t j = tid; j < nvp; j += kThreads) {
        const uint4 w = src[j];
#pragma unroll
        for (int k = 0; k < VEC; ++k) {
          const uint32_t b = vec_elem<Bits>(w, k);
          const float x = Elem<Bits>::to_float(b);
          const float e = fast_exp2(fmaf(x, coef, (r == 0 ? shift_p : shift_q)));
          if (e > w_min)
            atomicAdd(&hist[r * kBins + (Elem<Bits>::key(b) >> shift1)],
                      fixed_mass(x, e, m, coef64));
        }
      }
    }
    __syncthreads();
    cluster_sync();
  }

  // ---- 4. top-p threshold: MSD radix select over the logit key -------------
  if (use_top_p) {
    int consumed = 0;
    for (int level = 0; level < RadixLevels<Bits>::kCount; ++level) {
      const int lbits = RadixLevels<Bits>::bits(level);
      const int nb = 1 << lbits;
      const bool last = level == RadixLevels<Bits>::kCount - 1;
      if (level > 0) {
        // histogram of the elements whose key matches the prefix so far
        for (int t = tid; t < 2 * kBins; t += kThreads) hist[t] = 0ull;
        __syncthreads();
        const int shift_prev = Elem<Bits>::kKeyBits - consumed;
        const int shift_here = shift_prev - lbits;
        for (int r = 0; r < nrows; ++r) {
          const uint4 *src = r == 0 ? vp : vq;
          const uint32_t want = bc.prefix[r];
          const float window = bc.window[r];
          for (int32_t j = tid; j < nvp; j += kThreads) {
            const uint4 w = src[j];
#pragma unroll
            for (int k = 0; k < VEC; ++k) {
              const uint32_t b = vec_elem<Bits>(w, k);
              const uint32_t key = Elem<Bits>::key(b);
              if ((key >> shift_prev) == want) {
                const float x = Elem<Bits>::to_float(b);
                const float e = fast_exp2(fmaf(x, coef, (r == 0 ? shift_p : shift_q)));
                if (e > window)
                  atomicAdd(&hist[r * kBins + ((key >> shift_here) & (uint32_t)(nb - 1))],
                            fixed_mass(x, e, bc.m[r], coef64));
              }
            }
          }
        }
        __syncthreads();
        cluster_sync();
      }
      // (level 0: the histograms were complete before the barrier that
      // published the sums of exponentials)
      // owner reduction: CTA `rank` sums bins [rank*per, rank*per + per)
      const int per = (nb + (int)C - 1) / (int)C;
      for (int t = tid; t < nrows * per; t += kThreads) {
        const int r = t / per, b = (int)rank * per + t % per;
        unsigned long long s = 0ull;
        if (b < nb)
          for (uint32_t k = 0; k < C; ++k) s += dsmem_ld_u64(dsmem_map(&hist[r * kBins + b], k));
        owned[r * per + t % per] = s;
      }
      __syncthreads();
      if (warp < nrows) {
        unsigned long long s = 0ull;
        for (int t = lane; t < per; t += 32) s += owned[warp * per + t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
        if (lane == 0) xc.block_sum[level][warp] = s;
      }
      __syncthreads();
      cluster_sync();
      if (warp < nrows) radix_crossing<Bits>(warp, level, lbits, last, C, &xc, owned, per, &bc);
      __syncthreads();
      consumed += lbits;
    }
  }

  // ---- 5. accept / reject the drafted token (every CTA, same result) -------
  const double zp_p = bc.zp[0], zp_q = bc.zp[1];
  const float tau_p = bc.tau[0], tau_q = bc.tau[1];
  const float m_p = bc.m[0], m_q = bc.m[1];
  if (tid == 0) {
    int need = 1;
    if (has_q) {
      const int32_t x = s_x;
      double p = 0.0, q = 0.0;
      const bool valid = x >= 0 && x < V;
      if (valid) {
        const float xp = Elem<Bits>::to_float(s_x_bits[0]);
        const float xq = Elem<Bits>::to_float(s_x_bits[1]);
        if (xp >= tau_p && zp_p > 0.0) p = exact_exp2(xp, m_p, coef64) / zp_p;
        if (xq >= tau_q && zp_q > 0.0) q = exact_exp2(xq, m_q, coef64) / zp_q;
      }
      const double u = uniform24(a.seed, seq, a.step, (uint64_t)i, PSI_PURPOSE_ACCEPT);
      const int accept = (u * q < p) ? 1 : 0;
      need = (mode == kModeSample) ? 1 : !accept;
      if (rank == 0 && mode != kModeSample) {
        const int64_t o = (int64_t)n * B + i;
        if (a.out_p) a.out_p[o] = (float)p;
        if (a.out_q) a.out_q[o] = (float)q;
        a.records[unit].accept = accept;
        if (accept) a.records[unit].token = -1;
        if (!valid && a.dev_status) atomicOr(a.dev_status, PSI_DEV_BAD_TOKEN_ID);
      }
    } else if (rank == 0 && mode != kModeSample) {
      a.records[unit].accept = 1;  // the bonus row always draws
    }
    bc.need_sample = need;
    bc.use_p_only = has_q ? 0 : 1;
  }
  const bool any_bad = __syncthreads_or(bad || timed_out);
  if (tid == 0 && any_bad && a.dev_status)
    atomicOr(a.dev_status, (bad ? PSI_DEV_NONFINITE : 0u) | (timed_out ? PSI_DEV_TIMEOUT : 0u));

  // ---- 6. correction (rejected row) or bonus (row B) draw -------------------
  // Weights w(v) = max(0, p(v) - q(v)) or p(v), from fp32 exponentials (the
  // draw's CDF is then within ~1e-7 of the exact one, far inside the
  // near-tie margin), in 2^40 fixed point (exact integer sums in any
  // order); inverse CDF in vocabulary order: the first v whose running sum
  // exceeds t = floor(u' * sum(w)).  Every pass uses this same function.
  const float inv_zp = zp_p > 0.0 ? (float)(1.0 / zp_p) : 0.f;
  const float inv_zq = zp_q > 0.0 ? (float)(1.0 / zp_q) : 0.f;
  auto weight = [&](uint32_t bp, uint32_t bq, bool p_only) -> unsigned long long {
    const float xp = Elem<Bits>::to_float(bp);
    if (!(xp >= tau_p) || !(zp_p > 0.0)) return 0ull;
    float pv = fast_exp2(fmaf(xp, coef, shift_p)) * inv_zp;
    if (!p_only) {
      const float xq = Elem<Bits>::to_float(bq);
      const float qv = (xq >= tau_q) ? fast_exp2(fmaf(xq, coef, shift_q)) * inv_zq : 0.f;
      pv = pv - qv;
    }
    return pv > 0.f ? __float2ull_rn(fminf(pv, 1.f) * kFixScale) : 0ull;
  };
  if (bc.need_sample) {
    for (int attempt = 0; attempt < 2; ++attempt) {
      const bool p_only = bc.use_p_only != 0;
      // per warp-chunk sums (a chunk = 32 consecutive vectors, in order)
      for (int32_t j = tid; j < nvp; j += kThreads) {
        const uint4 w = vp[j];
        const uint4 u = p_only ? w : vq[j];
        unsigned long long part = 0ull;
#pragma unroll
        for (int k = 0; k < VEC; ++k)
          part += weight(vec_elem<Bits>(w, k), vec_elem<Bits>(u, k), p_only);
        part = warp_sum_t(part);
        if (lane == 0) chunk_sum[j >> 5] = part;
      }
      __syncthreads();
      if (tid == 0) {
        unsigned long long s = 0ull;
        for (int c = 0; c < nchunks; ++c) s += chunk_sum[c];
        xc.w_part[attempt] = s;
      }
      cluster_sync();
      if (warp == 0) {
        const unsigned long long wk =
            (uint32_t)lane < C ? dsmem_ld_u64(dsmem_map(&xc.w_part[attempt], lane)) : 0ull;
        // inclusive prefix over ranks in rank (= vocabulary) order
        unsigned long long pre = wk;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long t = __shfl_up_sync(0xFFFFFFFFu, pre, o);
          if (lane >= o) pre += t;
        }
        const unsigned long long total = __shfl_sync(0xFFFFFFFFu, pre, 31);
        if (lane == 0) bc.w_total = total;
        if (total > 0ull) {
          const float u2 = uniform24(a.seed, seq, a.step, (uint64_t)i, PSI_PURPOSE_RESID);
          const unsigned long long k = (unsigned long long)(u2 * 16777216.0f);  // u' = k / 2^24
          const unsigned long long t = (__umul64hi(k, total) << 40) | ((k * total) >> 24);
          const unsigned hit = __ballot_sync(0xFFFFFFFFu, (uint32_t)lane < C && pre > t);
          const int kstar = __ffs(hit) - 1;  // exact sums: t < total, so some rank hits
          const unsigned long long before = __shfl_sync(0xFFFFFFFFu, pre - wk, kstar);
          if (lane == 0) {
            bc.cross_rank = kstar;
            bc.t_local = t - before;
          }
        }
      }
      __syncthreads();
      if (bc.w_total > 0ull || p_only) break;
      // the residual vanished (q_L(x_L) was 0): draw from p_L instead
      if (tid == 0) bc.use_p_only = 1;
      __syncthreads();
    }

    if (bc.w_total > 0ull && (int)rank == bc.cross_rank && warp == 0) {
      const bool p_only = bc.use_p_only != 0;
      const unsigned long long t = bc.t_local;
      // the chunk holding the crossing (same order as the CTA total)
      int cstar = 0;
      unsigned long long before = 0ull;
      for (int c = 0; c < nchunks; ++c) {
        const unsigned long long nxt = before + chunk_sum[c];
        if (nxt > t) {
          cstar = c;
          break;
        }
        before = nxt;
      }
      const int32_t j = cstar * 32 + lane;  // this lane's vector in the chunk
      const uint4 w = vp[j];
      const uint4 u = p_only ? w : vq[j];
      unsigned long long wv[VEC];
      unsigned long long part = 0ull;
#pragma unroll
      for (int k = 0; k < VEC; ++k) {
        wv[k] = weight(vec_elem<Bits>(w, k), vec_elem<Bits>(u, k), p_only);
        part += wv[k];
      }
      unsigned long long pre = part;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long tt = __shfl_up_sync(0xFFFFFFFFu, pre, o);
        if (lane >= o) pre += tt;
      }
      const unsigned hit = __ballot_sync(0xFFFFFFFFu, before + pre > t);
      const int l = hit ? __ffs(hit) - 1 : 31;
      int32_t token = c0 + j * VEC;
      if (lane == l) {
        unsigned long long run = before + pre - part;
        int kk = VEC - 1;
        for (int k = 0; k < VEC; ++k) {
          run += wv[k];
          if (run > t) {
            kk = k;
            break;
          }
        }
        token = c0 + j * VEC + kk;
      }
      token = __shfl_sync(0xFFFFFFFFu, token, l);
      if (lane == 0) {
        if (mode == kModeSample) a.out_tokens[unit] = token;
        else a.records[unit].token = token;
      }
    }
  }
  if (bc.need_sample && bc.w_total == 0ull && rank == 0 && tid == 0) {
    // no positive weight anywhere (degenerate row)
    if (mode == kModeSample) a.out_tokens[unit] = 0;
    else a.records[unit].token = 0;
  }

  // keep this CTA's shared memory alive until every peer is done reading it
  // (and the buffers free for the next item)
  cluster_sync();
  }  // work items
}

// One thread per sequence: first rejected row -> emitted tokens.
__global__ void __launch_bounds__(128) sampled_emit_kernel(const UnitRecord *__restrict__ rec,
                                                           const int32_t *__restrict__ ids,
                                                           int32_t N, int32_t B,
                                                           int32_t *__restrict__ out_tokens,
                                                           int32_t *__restrict__ out_n) {
  const int32_t n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const UnitRecord *r = rec + (int64_t)n * (B + 1);
  int32_t L = B;
  for (int32_t i = 0; i < B; ++i)
    if (!r[i].accept) {
      L = i;
      break;
    }
  int32_t *tok = out_tokens + (int64_t)n * (B + 1);
  for (int32_t i = 0; i < L; ++i) tok[i] = ids[(int64_t)n * B + i];
  tok[L] = r[L].token;
  for (int32_t i = L + 1; i <= B; ++i) tok[i] = -1;
  out_n[n] = L + 1;
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
bool plan_sampled(int32_t V, int elem_bytes, SampledPlan *plan) {
  const int vec = 16 / elem_bytes;
  const int64_t pref = 24576 / elem_bytes;  // preferred elements per row per CTA
  const int64_t hard = 49152 / elem_bytes;  // largest slice that still fits
  int C = 1;
  while (C < 16 && ((int64_t)V + C - 1) / C > pref) C *= 2;
  int64_t S = ((int64_t)V + C - 1) / C;
  S = (S + vec - 1) / vec * vec;
  if (S > hard) return false;
  const int64_t nvec = S / vec;
  const int64_t nvp = (nvec + 31) / 32 * 32;
  const int per_max = (kBins + C - 1) / C;
  plan->cluster = C;
  plan->slice = (int32_t)S;
  plan->nvec_pad = (int32_t)nvp;
  plan->smem = (size_t)2 * nvp * 16 + sizeof(unsigned long long) * (2 * kBins + 2 * per_max) +
               sizeof(unsigned long long) * (size_t)(nvp / 32);
  return true;
}

struct ClusterParams {
  float coef;
  double coef64;
  float w_min, w_narrow;
  int use_top_p;
};

static ClusterParams cluster_params(const SampledArgs &a) {
  ClusterParams c;
  c.coef64 = 1.4426950408889634 / (double)a.temperature;  // log2(e) / T
  c.coef = (float)c.coef64;
  c.use_top_p = a.top_p < 1.0f ? 1 : 0;
  // Only e(v) above (1 - top_p) / V can reach the threshold (the mass below
  // the threshold key exceeds (1 - top_p) * Z >= 1 - top_p and is spread over
  // at most V tokens); half of it leaves room for rounding.
  c.w_min = c.use_top_p ? (float)(0.5 * (1.0 - (double)a.top_p) / (double)a.V) : 0.f;
  c.w_narrow = fmaxf(kNarrowWindow, c.w_min);
  return c;
}

template <typename Bits>
static cudaError_t launch_cluster_kernel(const SampledArgs &a, const SampledPlan &plan, int mode,
                                         const int32_t *list, const int32_t *count,
                                         int64_t n_clusters, const KernelEvents *ev,
                                         cudaStream_t stream) {
  auto kernel = sampled_unit_kernel<Bits>;
  // the largest shared memory set so far, per device
  static std::atomic<int> configured_smem[PerDevice::kMax] = {};
  const int dev = PerDevice::current();
  const bool slot = dev >= 0 && dev < PerDevice::kMax;
  if (!slot || (int)plan.smem > configured_smem[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)plan.smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    if ((e = prefer_max_shared(kernel)) != cudaSuccess) return e;
    if (slot) {
      int cur = configured_smem[dev].load(std::memory_order_relaxed);
      while ((int)plan.smem > cur &&
             !configured_smem[dev].compare_exchange_weak(cur, (int)plan.smem)) {
      }
    }
  }
  const int64_t grid = n_clusters * plan.cluster;
  if (grid > 0x7FFFFFFFLL || grid < 1) return cudaErrorInvalidConfiguration;
  const ClusterParams c = cluster_params(a);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)plan.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_pdl
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e;
  if (ev && ev->before && (e = cudaEventRecord(ev->before, stream)) != cudaSuccess) return e;
  e = cudaLaunchKernelEx(&cfg, kernel, a, plan, c.coef, c.coef64, c.w_min, c.w_narrow,
                         c.use_top_p, mode, list, count);
  if (e != cudaSuccess) return e;
  if (ev && ev->after && (e = cudaEventRecord(ev->after, stream)) != cudaSuccess) return e;
  return cudaSuccess;
}

cudaError_t launch_sampled(const SampledArgs &a, psi_dtype dtype, const SampledPlan &plan,
                           const KernelEvents &ev, cudaStream_t stream) {
  const int64_t units = (int64_t)a.N * (a.B + 1);
  cudaError_t e =
      dtype == PSI_DTYPE_BF16
          ? launch_cluster_kernel<uint16_t>(a, plan, kModeGrid, nullptr, nullptr, units, &ev, stream)
          : launch_cluster_kernel<uint32_t>(a, plan, kModeGrid, nullptr, nullptr, units, &ev, stream);
  if (e != cudaSuccess) return e;
  sampled_emit_kernel<<<(a.N + 127) / 128, 128, 0, stream>>>(a.records, a.ids, a.N, a.B,
                                                             a.out_tokens, a.out_n);
  return cudaGetLastError();
}

cudaError_t launch_sampled_emit(const SampledArgs &a, cudaStream_t stream) {
  sampled_emit_kernel<<<(a.N + 127) / 128, 128, 0, stream>>>(a.records, a.ids, a.N, a.B,
                                                             a.out_tokens, a.out_n);
  return cudaGetLastError();
}

cudaError_t launch_cluster_list(const SampledArgs &a, psi_dtype dtype, const SampledPlan &plan,
                                int mode, const int32_t *list, const int32_t *count,
                                int max_clusters, cudaStream_t stream) {
  if (dtype == PSI_DTYPE_BF16)
    return launch_cluster_kernel<uint16_t>(a, plan, mode, list, count, max_clusters, nullptr, stream);
  return launch_cluster_kernel<uint32_t>(a, plan, mode, list, count, max_clusters, nullptr, stream);
}

}  // namespace psi
