// psi_finish.cuh - the finish of one logit row of the streaming path (row
// maximum, normaliser, top-p / top-k threshold) from the scan's slice
// records and set-aside lists, by one warp (the row_finish kernel of the
// linear verify and of the sampled tree walk).
//
// Sources (page title, section): "Uno Psi-Spec 是什麼？Diffusion-Augmented LLM
// 如何保留 AR 分布、一次驗證多個 Token" (alphalab.site), "想跑 Uno：先確認官方程式
// 需要的環境" (temperature and top-p on the run card).
#pragma once

#include "psi_internal.h"

namespace psi {

// A finished row, as the row_finish kernel leaves it for the unit kernel.
// The row's candidates (x above its final threshold), as raw list entries
// (bits << 32) | vocabulary index, are compacted in place at the front of
// the row's set-aside area.
struct RowFin {
  float m;            // row maximum
  int32_t status;     // kFin* bits
  double zp;          // normaliser after top-p (Z without top-p)
  uint32_t tau_bits;  // top-p threshold (raw bits): keep x >= tau
  uint32_t tau_key;   // its order-preserving key (0 without top-p)
  int32_t n;          // candidates at the front of the row's area
  int32_t pad;
};

namespace finish {

template <typename T>
__device__ __forceinline__ T warp_sum_any(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
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
constexpr int kFinTopK = 8;       // the candidates do not hold the row's top-k set

constexpr int kLoadChunk = 16;           // global loads per lane in flight together
constexpr int kQChunk = 16;              // q loads per lane in flight together
constexpr int kRegCand = 16;             // candidates per lane a search keeps in registers
// Masses and draw weights (each <= 1) are summed in 2^52 fixed point: the sum
// of up to kCandCap of them fits 64 bits, and integer sums do not depend on
// the order of the candidates.
constexpr double kFix52 = 4503599627370496.0;  // 2^52

struct WarpScratch {
  uint32_t key[kFinishCap];  // candidate keys (order-preserving image of the logit)
  uint32_t idx[kFinishCap];  // vocabulary indices; later the nucleus indices
  uint64_t m[kFinishCap];    // 2^52 fixed-point masses exp2((x - M) * log2(e)/T) (double);
                           // later the nucleus masses, compacted; in the q row's
                           // scratch, the draw weights
};

// A mass or weight in [0, 1] in 2^52 fixed point.
__device__ __forceinline__ uint64_t fixed52(double m) { return __double2ull_rn(m * kFix52); }

// floor(m * 2^52) of an fp32 m in [0, 1], from its bits (integer shifts
// only): m = (2^23 + frac) * 2^(e - 150), so m * 2^52 = (2^23 + frac) << (e - 98).
__device__ __forceinline__ uint64_t fixed52_f32(float m) {
  const uint32_t b = __float_as_uint(m);
  const int sh = (int)(b >> 23) - 98;
  const uint64_t mant = (uint64_t)((b & 0x7FFFFFu) | 0x800000u);
  if (sh <= -24) return 0ull;  // below 2^-52, zero and subnormals included
  return sh >= 0 ? (mant << sh) : (mant >> (-sh));
}

// ---------------------------------------------------------------------------
// The row finish: one CTA of kFinWarps warps per row, results to global
// memory (the row_finish kernel of the linear verify and the tree walk).
// ---------------------------------------------------------------------------
constexpr int kFinWarps = 4;
constexpr int kFinThreads = 32 * kFinWarps;
constexpr int kFinChunk = 8;  // list entries per lane and chunk (loads in flight together)

struct FinShared {
  unsigned long long e[kFinishCap];  // the candidates' list entries (bits << 32 | index)
  unsigned long long m[kFinishCap];  // their exact masses, 2^52 fixed point
  unsigned long long red[kFinWarps][2];
  uint32_t kred[kFinWarps][2];
  unsigned long long sv[kFinWarps];  // search: the pivots' values
  uint32_t sp[kFinWarps];            // search: the pivots
  int n;                             // candidates found so far
};

// Largest t in [lo, hi) with F(t) >= target, for F non-increasing and
// F(lo) = f_lo >= target, by a 4-ary search: warps 1..3 each evaluate F at one
// pivot per round (`eval(t)`: the warp's value of F(t), the same in every
// lane).  Every thread of the CTA takes part; f_lo returns F(t).
template <typename Eval>
__device__ uint32_t cta_search(uint32_t lo, uint32_t hi, unsigned long long target,
                               unsigned long long &f_lo, FinShared &sh, Eval eval) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  while (hi - lo > 1u) {
    if (warp >= 1) {
      const uint32_t piv = lo + (uint32_t)(((uint64_t)(hi - lo) * (uint64_t)warp) / kFinWarps);
      const bool valid = piv > lo;
      const unsigned long long v = valid ? eval(piv) : 0ull;
      if (lane == 0) {
        sh.sv[warp] = v;
        sh.sp[warp] = valid ? piv : 0u;
      }
    }
    __syncthreads();
    uint32_t nlo = lo, nhi = hi;
    unsigned long long nf = f_lo;
    for (int w = 1; w < kFinWarps; ++w) {  // pivots ascend, F descends
      const uint32_t piv = sh.sp[w];
      if (piv == 0u || piv <= nlo) continue;
      if (sh.sv[w] >= target) {
        nlo = piv;
        nf = sh.sv[w];
      } else {
        nhi = piv;
        break;
      }
    }
    lo = nlo;
    hi = nhi;
    f_lo = nf;
    __syncthreads();  // the pivots' slots are written again next round
  }
  return lo;
}

// Row maximum, Z, top-p (and top-k) threshold tau and renormaliser Z' of
// row r from its slice records and set-aside lists, by one CTA.  M is the
// largest slice maximum; Z is the slices' sums rescaled to M plus the
// set-aside masses.  The set-aside elements above the row's final threshold
// (M - window, rounded as the scan rounds) are the candidates: every element
// the top-p cut (or a top-k cut that they hold) can keep.  Their masses are
// exact (double precision, 2^52 fixed point); they are gathered in shared
// memory and then written, compacted, to the front of the row's set-aside
// area, where the draws read them.  The other set-aside masses (with top-p
// each under 2^-13 of the maximum's) are taken in fp32, like the slices'
// sums, and join Z in fixed point; integer sums keep the result independent
// of the lists' order (and of the order in which the warps gather).  tau is
// the largest key t whose suffix mass S(t) (every candidate with key >= t)
// reaches top_p * Z, found by a search on exact integer sums; with top-k, the
// k-th largest key t_k comes first (the same search on counts) and top-p
// then cuts the set at or above t_k, whose mass replaces Z.
template <typename Bits>
__device__ RowFin finish_row_cta(const FastArgs &a, int64_t r, FinShared &sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  RowFin out;
  out.m = -INFINITY;
  out.zp = 0.0;
  out.tau_bits = Elem<Bits>::kNegInf;
  out.tau_key = 0u;
  out.n = 0;
  out.status = 0;
  out.pad = 0;
  const int C = a.g.slices;
  const SliceRecord *sr = a.srec + r * kMaxSlices;
  float M = -INFINITY;
  bool lost = false;
  int nc[kMaxSlices] = {};
  for (int c = 0; c < C; ++c) {
    M = fmaxf(M, sr[c].m);
    lost |= (sr[c].flags & kRowLost) != 0 || sr[c].n_cand > a.g.cap;
    nc[c] = sr[c].n_cand;
  }
  out.m = M;
  if (lost) {
    out.status = kFinOverflow;
    return out;
  }
  double Z = 0.0;
  for (int c = 0; c < C; ++c)
    if (sr[c].m > -INFINITY) Z += sr[c].z * exp2(((double)sr[c].m - (double)M) * a.coef64);
  if (!(M > -INFINITY) || !(fabsf(M * a.coef) < INFINITY) || Z != Z) {
    out.status = kFinNonfinite;
    return out;
  }
  const float thr = a.use_window ? threshold_value<Bits>(M - sr[0].off) : INFINITY;
  unsigned long long *area = reinterpret_cast<unsigned long long *>(a.cand + r * (int64_t)kCandCap);
  if (tid == 0) sh.n = 0;
  __syncthreads();
  // ---- sort the lists: chunks of 32 * kFinChunk entries, dealt to the warps
  constexpr int kChunkEntries = 32 * kFinChunk;
  const int q0 = (nc[0] + kChunkEntries - 1) / kChunkEntries;
  const int q1 = C > 1 ? (nc[1] + kChunkEntries - 1) / kChunkEntries : 0;
  unsigned long long zrest = 0ull;
  for (int q = warp; q < q0 + q1; q += kFinWarps) {
    const int c = q < q0 ? 0 : 1;
    const int base = (q < q0 ? q : q - q0) * kChunkEntries;
    const unsigned long long *src = area + (int64_t)c * a.g.cap;
    unsigned long long e[kFinChunk];
#pragma unroll
    for (int h = 0; h < kFinChunk; ++h) {
      const int j = base + 32 * h + lane;
      e[h] = j < nc[c] ? __ldcg(src + j) : 0ull;
    }
    uint32_t cmask = 0u;  // bit h: entry h is a candidate
#pragma unroll
    for (int h = 0; h < kFinChunk; ++h) {
      const int j = base + 32 * h + lane;
      const float x = Elem<Bits>::to_float((uint32_t)(e[h] >> 32));
      const bool live = j < nc[c];
      const bool cand = live && x > thr;
      cmask |= (cand ? 1u : 0u) << h;
      const float mf = (live && !cand) ? fast_exp2((x - M) * a.coef) : 0.f;  // <= 1
      zrest += fixed52_f32(mf);
    }
    const int cnt = __popc(cmask);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    int base_d = 0;
    if (lane == 31) base_d = atomicAdd(&sh.n, incl);
    int d = __shfl_sync(0xFFFFFFFFu, base_d, 31) + incl - cnt;
#pragma unroll
    for (int h = 0; h < kFinChunk; ++h)
      if ((cmask >> h) & 1u) {
        if (d < kFinishCap) sh.e[d] = e[h];
        ++d;
      }
  }
  __syncthreads();
  const int n = sh.n;
  // ---- the candidates: exact masses, the compacted list to the area (every
  // list entry has been read), key range
  unsigned long long zin = 0ull;
  uint32_t kmax = 0u, kmin_inv = 0u;
  if (n <= kFinishCap) {
    for (int j = tid; j < n; j += kFinThreads) {
      const unsigned long long ej = sh.e[j];
      const uint32_t b = (uint32_t)(ej >> 32);
      const unsigned long long m52 = fixed52(exact_exp2d(Elem<Bits>::to_float(b), M, a.coef64));
      sh.m[j] = m52;
      zin += m52;
      area[j] = ej;
      const uint32_t key = Elem<Bits>::key(b);
      kmax = max(kmax, key);
      kmin_inv = max(kmin_inv, ~key);
    }
  }
  zin = warp_sum_any(zin);
  zrest = warp_sum_any(zrest);
  kmax = warp_max_u32(kmax);
  kmin_inv = warp_max_u32(kmin_inv);
  if (lane == 0) {
    sh.red[warp][0] = zin;
    sh.red[warp][1] = zrest;
    sh.kred[warp][0] = kmax;
    sh.kred[warp][1] = kmin_inv;
  }
  __syncthreads();
  zin = zrest = 0ull;
  kmax = kmin_inv = 0u;
#pragma unroll
  for (int w = 0; w < kFinWarps; ++w) {
    zin += sh.red[w][0];
    zrest += sh.red[w][1];
    kmax = max(kmax, sh.kred[w][0]);
    kmin_inv = max(kmin_inv, sh.kred[w][1]);
  }
  if (n > kFinishCap) {  // more candidates than the area holds: rescan, then the general path
    out.status = kFinOverflow;
    return out;
  }
  out.n = n;
  Z += ((double)zin + (double)zrest) / kFix52;
  out.zp = Z;
  if (!(Z < INFINITY)) {
    out.status = kFinNonfinite;
    return out;
  }
  if (!a.use_window) return out;
  const uint32_t kmin = ~kmin_inv;
  // the warp's suffix mass (or count) at key t
  auto mass_from = [&](uint32_t t) -> unsigned long long {
    unsigned long long part = 0ull;
    for (int j = lane; j < n; j += 32)
      if (Elem<Bits>::key((uint32_t)(sh.e[j] >> 32)) >= t) part += sh.m[j];
    return warp_sum_any(part);
  };
  auto count_from = [&](uint32_t t) -> unsigned long long {
    int cnt = 0;
    for (int j = lane; j < n; j += 32)
      cnt += Elem<Bits>::key((uint32_t)(sh.e[j] >> 32)) >= t ? 1 : 0;
    return (unsigned long long)__reduce_add_sync(0xFFFFFFFFu, cnt);
  };
  if (a.top_k > 0) {
    // top-k: the k-th largest key among the candidates is the row's when
    // they number at least k (every other element lies below them); else
    // the whole-row top-k path takes the unit
    if (n < a.top_k) {
      out.status = kFinTopK;
      return out;
    }
    unsigned long long cnt_lo = (unsigned long long)n;
    const uint32_t tk =
        cta_search(kmin, kmax + 1u, (unsigned long long)a.top_k, cnt_lo, sh, count_from);
    // the mass of the top-k set
    unsigned long long zk = 0ull;
    for (int j = tid; j < n; j += kFinThreads)
      if (Elem<Bits>::key((uint32_t)(sh.e[j] >> 32)) >= tk) zk += sh.m[j];
    zk = warp_sum_any(zk);
    __syncthreads();
    if (lane == 0) sh.red[warp][0] = zk;
    __syncthreads();
    zk = 0ull;
#pragma unroll
    for (int w = 0; w < kFinWarps; ++w) zk += sh.red[w][0];
    uint32_t t = tk;
    unsigned long long s_at = zk;
    if (a.use_top_p) {  // top-p of the renormalised top-k distribution
      unsigned long long target = (unsigned long long)ceil((double)a.s.top_p * (double)zk);
      if (target == 0ull) target = 1ull;
      t = cta_search(tk, kmax + 1u, target, s_at, sh, mass_from);
    }
    out.zp = (double)s_at / kFix52;
    out.tau_key = t;
    out.tau_bits = key_to_bits<Bits>(t);
    return out;
  }
  const double target_d = ceil((double)a.s.top_p * Z * kFix52);
  if (!(target_d < 9.2e18) || (double)zin < target_d) {  // (zin < 2^63)
    out.status = kFinCoverage;
    return out;
  }
  const unsigned long long target = (unsigned long long)target_d;
  if (zin < target) {
    out.status = kFinCoverage;
    return out;
  }
  // search over [kmin, kmax]: S(kmin) = zin reaches the target
  unsigned long long s_at = zin;
  const uint32_t t = cta_search(kmin, kmax + 1u, target, s_at, sh, mass_from);
  out.zp = (double)s_at / kFix52;
  out.tau_key = t;
  out.tau_bits = key_to_bits<Bits>(t);
  return out;
}

}  // namespace finish
}  // namespace psi
