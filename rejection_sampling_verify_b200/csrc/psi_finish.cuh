// psi_finish.cuh - the finish of one logit row of the streaming path (row
// maximum, normaliser, top-p threshold) from the scan's slice records and
// candidate lists, by one warp.  Shared by the linear verify's unit kernel
// and the sampled tree walk.
//
// Sources (page title, section): "Uno Psi-Spec 是什麼？Diffusion-Augmented LLM
// 如何保留 AR 分布、一次驗證多個 Token" (alphalab.site), "想跑 Uno：先確認官方程式
// 需要的環境" (temperature and top-p on the run card).
#pragma once

#include "psi_internal.h"

namespace psi {
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

// Row maximum, Z, top-p threshold tau and renormaliser Z' of row r from its
// slice records and set-aside lists, by one warp.  M is the largest slice
// reference; the set-aside elements above the row's final threshold
// (M - window, rounded as the scan rounds) are the candidates, the others
// join Z with the slices' sums (rescaled to M), every mass in double
// precision and 2^52 fixed point.  The top-p threshold is the largest logit
// key t whose suffix mass S(t) (every x with key >= t) reaches top_p * Z: a
// binary search over the candidates' key range on exact integer sums
// (independent of the order of the lists).  Only candidates can be at or
// above tau when they hold at least top_p of the mass.  The lists stay
// unchanged, so a second pass may finish the row again.
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
  const int C = a.g.slices;
  const SliceRecord *sr = a.srec + r * kMaxSlices;
  float M = -INFINITY;
  bool lost = false;
  for (int c = 0; c < C; ++c) {
    M = fmaxf(M, sr[c].m);
    lost |= (sr[c].flags & kRowLost) != 0 || sr[c].n_cand > a.g.cap;
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
  const float thr = a.use_top_p ? threshold_value<Bits>(M - sr[0].off) : INFINITY;
  // sort the set-aside elements: candidates to the scratch, the rest to Z
  const unsigned below = (1u << lane) - 1u;
  int n = 0;
  unsigned long long zin = 0ull, zrest = 0ull;
  uint32_t kmax = 0u, kmin_inv = 0u;
  for (int c = 0; c < C; ++c) {
    const int nc = sr[c].n_cand;
    const unsigned long long *src = reinterpret_cast<const unsigned long long *>(
        a.cand + r * (int64_t)kCandCap + (int64_t)c * a.g.cap);
    for (int base = 0; base < nc; base += 32 * kLoadChunk) {
      unsigned long long e[kLoadChunk];
#pragma unroll
      for (int h = 0; h < kLoadChunk; ++h) {
        const int j = base + 32 * h + lane;
        e[h] = j < nc ? __ldcg(src + j) : 0ull;
      }
#pragma unroll
      for (int h = 0; h < kLoadChunk; ++h) {
        const int j = base + 32 * h + lane;
        const uint32_t b = (uint32_t)(e[h] >> 32);
        const float x = Elem<Bits>::to_float(b);
        const bool live = j < nc;
        const bool cand = live && x > thr;
        const double mass = live ? exact_exp2d(x, M, a.coef64) : 0.0;
        if (live && !cand && mass > 0.0) zrest += fixed52(mass);
        const unsigned bal = __ballot_sync(0xFFFFFFFFu, cand);
        const int d = n + __popc(bal & below);
        if (cand && d < kFinishCap) {
          const uint32_t key = Elem<Bits>::key(b);
          const uint64_t m52 = fixed52(mass);
          ws->key[d] = key;
          ws->idx[d] = (uint32_t)e[h];
          ws->m[d] = m52;
          zin += m52;
          kmax = max(kmax, key);
          kmin_inv = max(kmin_inv, ~key);
        }
        n += __popc(bal);
      }
    }
  }
  if (n > kFinishCap) {  // more candidates than the finish holds: rescan, then the general path
    out.status = kFinOverflow;
    return out;
  }
  out.n = n;
  kmax = warp_max_u32(kmax);
  kmin_inv = warp_max_u32(kmin_inv);
  zin = warp_sum_any(zin);
  zrest = warp_sum_any(zrest);
  __syncwarp();
  Z += ((double)zin + (double)zrest) / kFix52;
  out.zp = Z;
  if (!(Z < INFINITY)) {
    out.status = kFinNonfinite;
    return out;
  }
  if (!a.use_top_p) return out;
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
  // binary search over [kmin, kmax] with exact integer sums (order-free):
  // S(kmin) = zin reaches the target
  uint32_t lo = ~kmin_inv, hi = kmax + 1u;
  unsigned long long s_lo = zin;
  if (n <= 32 * kRegCand) {
    uint32_t kr[kRegCand];  // the row's candidates in registers
    uint64_t mr[kRegCand];
#pragma unroll
    for (int c = 0; c < kRegCand; ++c) {
      const int j = lane + 32 * c;
      kr[c] = j < n ? ws->key[j] : 0u;
      mr[c] = j < n ? ws->m[j] : 0ull;
    }
    while (hi - lo > 1u) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      unsigned long long part = 0ull;
#pragma unroll
      for (int c = 0; c < kRegCand; ++c) part += kr[c] >= mid ? mr[c] : 0ull;
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
  out.zp = (double)s_lo / kFix52;
  out.tau_key = lo;
  out.tau_bits = key_to_bits<Bits>(lo);
  return out;
}

}  // namespace finish
}  // namespace psi
