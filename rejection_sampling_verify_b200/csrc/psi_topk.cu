// psi_topk.cu - the linear verify's whole-row path for top-k (one CTA per
// (sequence, position) unit): units whose candidate window does not hold
// their rows' top-k sets, and every unit when the streaming path does not
// apply.
//
// Sources (page title, section): "想跑 Uno：先確認官方程式需要的環境" (the run
// card names top-k beside top-p and temperature); "Uno Psi-Spec 怎麼運作？
// 完整走一次四個 Token", steps 3-4 and the bonus paragraph (accept while
// u < p/q, residual correction, bonus token).  Reading of the order: top-k is
// taken on the temperature softmax, its kept mass renormalised, and top-p
// then cuts that distribution; ties with the k-th probability stay.
//
// Per row (p, then q), by the whole CTA, reading the row from global memory:
//   1. the row maximum M (and non-finite logits flagged);
//   2. t_k, the k-th largest order-preserving key: a most-significant-digit
//      radix select on counts, 8 bits per level;
//   3. Z_k = the mass of the elements with key >= t_k, each exp2((x - M) *
//      log2(e) / T) in double and 2^52 fixed point (order-free sums);
//   4. with top-p, tau = the largest key whose suffix mass within the top-k
//      set reaches top_p * Z_k: the same radix select on those masses;
//      without, tau = t_k.  zp = the suffix mass at tau.
// Then p(x) and q(x) of the drafted token decide the unit, and a rejected (or
// bonus) unit draws from the residual max(0, p - q) (or p) over the whole
// row in vocabulary order: each thread sums a contiguous chunk, a block scan
// places the draw's point t = floor(u' * W), and the chunk that holds it is
// walked element by element.
#include "psi_internal.h"

namespace psi {

namespace {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr double kFix52 = 4503599627370496.0;  // 2^52

struct TopkShared {
  unsigned long long hist[256];  // radix counts or masses of one level
  unsigned long long wsum[kTopkWarps];
  uint32_t wkey[kTopkWarps];
  uint32_t prefix;               // radix prefix so far
  unsigned long long need;       // counts: elements still to pass; masses: target
  unsigned long long above;      // mass above the prefix's range
  unsigned long long at;         // mass at the chosen bin
  int bad;
};

struct TopkRow {
  float m;                // row maximum
  uint32_t tau_key;       // keep x with key >= tau_key
  unsigned long long zp;  // kept mass in 2^52 fixed point
};

__device__ __forceinline__ double mass_d(float x, float m, double coef64) {
  return exp2(((double)x - (double)m) * coef64);
}

__device__ __forceinline__ unsigned long long fix52(double v) { return __double2ull_rn(v * kFix52); }

template <typename T>
__device__ __forceinline__ T warp_add(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Block sum (every thread gets it).
__device__ unsigned long long block_add(unsigned long long v, TopkShared &sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_add(v);
  if (lane == 0) sh.wsum[warp] = v;
  __syncthreads();
  unsigned long long t = 0ull;
#pragma unroll
  for (int w = 0; w < kTopkWarps; ++w) t += sh.wsum[w];
  __syncthreads();
  return t;
}

// One radix level: thread 0 walks the 256 bins from the top and keeps the bin
// where the running total (on top of sh.above) first reaches sh.need.
__device__ void pick_bin_from_top(TopkShared &sh, int nb) {
  if (threadIdx.x == 0) {
    unsigned long long run = sh.above;
    int bstar = 0;
    for (int b = (1 << nb) - 1; b >= 0; --b) {
      if (run + sh.hist[b] >= sh.need) {
        bstar = b;
        break;
      }
      run += sh.hist[b];
    }
    sh.at = sh.hist[bstar];
    sh.above = run;
    sh.prefix = (sh.prefix << nb) | (uint32_t)bstar;
  }
  __syncthreads();
}

template <typename Bits>
__device__ TopkRow topk_row_stats(const Bits *row, int32_t V, int32_t K, float top_p,
                                  double coef64, TopkShared &sh, uint32_t *dev_status) {
  constexpr int KB = 8 * (int)sizeof(Bits);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // ---- 1. maximum (largest key) and non-finite logits
  uint32_t kmax = 0u;
  int bad = 0;
  for (int32_t v = tid; v < V; v += kTopkThreads) {
    const uint32_t b = (uint32_t)row[v];
    bad |= Elem<Bits>::bad(b) ? 1 : 0;
    kmax = max(kmax, Elem<Bits>::key(b));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) kmax = max(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, o));
  bad = __any_sync(0xFFFFFFFFu, bad);
  if (lane == 0) sh.wkey[warp] = kmax;
  if (tid == 0) sh.bad = 0;
  __syncthreads();
  if (lane == 0 && bad) sh.bad = 1;
  uint32_t km = 0u;
#pragma unroll
  for (int w = 0; w < kTopkWarps; ++w) km = max(km, sh.wkey[w]);
  __syncthreads();
  if (tid == 0 && sh.bad && dev_status) atomicOr(dev_status, PSI_DEV_NONFINITE);
  TopkRow out;
  out.m = Elem<Bits>::to_float(sizeof(Bits) == 2 ? ((km & 0x8000u) ? (km & 0x7FFFu) : (~km & 0xFFFFu))
                                                 : ((km & 0x80000000u) ? (km & 0x7FFFFFFFu) : ~km));
  const float M = out.m;
  // ---- 2. t_k: the K-th largest key, 8 bits per level from the top
  if (tid == 0) {
    sh.prefix = 0u;
    sh.need = (unsigned long long)K;
    sh.above = 0ull;
  }
  for (int low = KB; low > 0; low -= 8) {
    const int shift = low - 8;
    for (int b = tid; b < 256; b += kTopkThreads) sh.hist[b] = 0ull;
    __syncthreads();
    const uint32_t pre = sh.prefix;
    for (int32_t v = tid; v < V; v += kTopkThreads) {
      const uint32_t key = Elem<Bits>::key((uint32_t)row[v]);
      if ((low >= 32 ? 0u : (key >> low)) == pre)
        atomicAdd(&sh.hist[(key >> shift) & 255u], 1ull);
    }
    __syncthreads();
    pick_bin_from_top(sh, 8);
  }
  const uint32_t tk = sh.prefix;
  // ---- 3. Z_k, the mass of the top-k set
  unsigned long long zk = 0ull;
  for (int32_t v = tid; v < V; v += kTopkThreads) {
    const uint32_t b = (uint32_t)row[v];
    if (Elem<Bits>::key(b) >= tk) zk += fix52(mass_d(Elem<Bits>::to_float(b), M, coef64));
  }
  zk = block_add(zk, sh);
  out.tau_key = tk;
  out.zp = zk;
  if (!(top_p < 1.0f) || zk == 0ull) return out;
  // ---- 4. top-p within the top-k set: suffix mass radix select
  if (tid == 0) {
    sh.prefix = 0u;
    sh.need = (unsigned long long)ceil((double)top_p * (double)zk);
    if (sh.need == 0ull) sh.need = 1ull;
    sh.above = 0ull;
  }
  __syncthreads();
  for (int low = KB; low > 0; low -= 8) {
    const int shift = low - 8;
    for (int b = tid; b < 256; b += kTopkThreads) sh.hist[b] = 0ull;
    __syncthreads();
    const uint32_t pre = sh.prefix;
    for (int32_t v = tid; v < V; v += kTopkThreads) {
      const uint32_t b = (uint32_t)row[v];
      const uint32_t key = Elem<Bits>::key(b);
      if (key >= tk && (low >= 32 ? 0u : (key >> low)) == pre)
        atomicAdd(&sh.hist[(key >> shift) & 255u], fix52(mass_d(Elem<Bits>::to_float(b), M, coef64)));
    }
    __syncthreads();
    pick_bin_from_top(sh, 8);
  }
  out.tau_key = sh.prefix;
  out.zp = sh.above + sh.at;
  __syncthreads();
  return out;
}

template <typename Bits>
__global__ void __launch_bounds__(kTopkThreads) topk_unit_kernel(SampledArgs a, double coef64,
                                                                const int32_t *list,
                                                                const int32_t *count) {
  pdl_wait();  // the previous kernel's results are visible
  pdl_trigger();
  __shared__ TopkShared sh;
  const int tid = threadIdx.x;
  const int32_t B = a.B, N = a.N, V = a.V;
  const int64_t n_items = list ? (int64_t)*count : (int64_t)N * (B + 1);
  for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int64_t unit = list ? (int64_t)list[item] : item;
    const int32_t n = (int32_t)(unit / (B + 1)), i = (int32_t)(unit % (B + 1));
    const bool has_q = i < B;
    const Bits *row_p = static_cast<const Bits *>(a.ar) + unit * a.ar_stride;
    const Bits *row_q =
        has_q ? static_cast<const Bits *>(a.draft) + ((int64_t)n * B + i) * a.draft_stride : nullptr;
    const TopkRow fp = topk_row_stats<Bits>(row_p, V, a.top_k, a.top_p, coef64, sh, a.dev_status);
    TopkRow fq;
    fq.m = -INFINITY;
    fq.tau_key = 0xFFFFFFFFu;
    fq.zp = 0ull;
    if (has_q) fq = topk_row_stats<Bits>(row_q, V, a.top_k, a.top_p, coef64, sh, a.dev_status);
    const uint64_t seq = a.seq_ids ? a.seq_ids[n] : (uint64_t)n;
    // p(v), q(v) after top-k and top-p
    auto pv_of = [&](uint32_t b) -> double {
      return (Elem<Bits>::key(b) >= fp.tau_key && fp.zp > 0ull)
                 ? mass_d(Elem<Bits>::to_float(b), fp.m, coef64) * kFix52 / (double)fp.zp
                 : 0.0;
    };
    auto qv_of = [&](uint32_t b) -> double {
      return (Elem<Bits>::key(b) >= fq.tau_key && fq.zp > 0ull)
                 ? mass_d(Elem<Bits>::to_float(b), fq.m, coef64) * kFix52 / (double)fq.zp
                 : 0.0;
    };
    // ---- decide
    int need = 1;
    if (has_q) {
      const int32_t x = a.ids[(int64_t)n * B + i];
      const bool valid = x >= 0 && x < V;
      const double p = valid ? pv_of((uint32_t)row_p[x]) : 0.0;
      const double q = valid ? qv_of((uint32_t)row_q[x]) : 0.0;
      const double u = (double)uniform24(a.seed, seq, a.step, (uint64_t)i, PSI_PURPOSE_ACCEPT);
      const int accept = (u * q < p) ? 1 : 0;
      need = !accept;
      if (tid == 0) {
        if (a.out_p) a.out_p[(int64_t)n * B + i] = (float)p;
        if (a.out_q) a.out_q[(int64_t)n * B + i] = (float)q;
        a.records[unit].accept = accept;
        if (accept) a.records[unit].token = -1;
        if (!valid && a.dev_status) atomicOr(a.dev_status, PSI_DEV_BAD_TOKEN_ID);
      }
    } else if (tid == 0) {
      a.records[unit].accept = 1;
    }
    if (need) {
      // ---- draw over the whole row in vocabulary order: the residual, or p
      // itself when the residual has no mass (or for the bonus row)
      const int32_t chunk = (V + kTopkThreads - 1) / kTopkThreads;
      const int32_t v0 = min(V, tid * chunk), v1 = min(V, v0 + chunk);
      int32_t token = 0;
      for (int pass = has_q ? 0 : 1; pass < 2; ++pass) {
        auto weight = [&](int32_t v) -> unsigned long long {
          const double pv = pv_of((uint32_t)row_p[v]);
          if (pass == 1) return fix52(pv);
          if (pv <= 0.0) return 0ull;
          const double qv = qv_of((uint32_t)row_q[v]);
          return pv > qv ? fix52(fmin(pv - qv, 1.0)) : 0ull;
        };
        unsigned long long wc = 0ull;
        for (int32_t v = v0; v < v1; ++v) wc += weight(v);
        // exclusive scan of the chunk sums over the block
        const int lane = tid & 31, warp = tid >> 5;
        unsigned long long incl = wc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += t;
        }
        if (lane == 31) sh.wsum[warp] = incl;
        __syncthreads();
        unsigned long long before = 0ull, W = 0ull;
#pragma unroll
        for (int w = 0; w < kTopkWarps; ++w) {
          if (w < warp) before += sh.wsum[w];
          W += sh.wsum[w];
        }
        before += incl - wc;
        __syncthreads();
        if (W == 0ull) continue;  // no residual mass: draw from p
        const float u2 = uniform24(a.seed, seq, a.step, (uint64_t)i, PSI_PURPOSE_RESID);
        const unsigned long long k = (unsigned long long)(u2 * 16777216.0f);
        const unsigned long long t = (__umul64hi(k, W) << 40) | ((k * W) >> 24);
        if (tid == 0) sh.prefix = 0u;
        __syncthreads();
        if (before <= t && t < before + wc) {  // exactly one thread's chunk holds t
          unsigned long long run = before;
          for (int32_t v = v0; v < v1; ++v) {
            run += weight(v);
            if (run > t) {
              sh.prefix = (uint32_t)v;
              break;
            }
          }
        }
        __syncthreads();
        token = (int32_t)sh.prefix;
        __syncthreads();
        break;
      }
      if (tid == 0) a.records[unit].token = token;
    }
    __syncthreads();  // shared memory free for the next unit
  }
}

template <typename Bits>
cudaError_t launch_topk_typed(const SampledArgs &a, const int32_t *list, const int32_t *count,
                              int64_t grid, cudaStream_t stream) {
  const double coef64 = 1.4426950408889634 / (double)a.temperature;
  return launch_pdl(topk_unit_kernel<Bits>, dim3((unsigned)grid), dim3(kTopkThreads), 0, stream, a,
                    coef64, list, count);
}

}  // namespace

cudaError_t launch_topk_units(const SampledArgs &a, psi_dtype dtype, const int32_t *list,
                              const int32_t *count, int64_t max_ctas, cudaStream_t stream) {
  const int64_t grid = std::max<int64_t>(1, max_ctas);
  if (dtype == PSI_DTYPE_BF16) return launch_topk_typed<uint16_t>(a, list, count, grid, stream);
  return launch_topk_typed<uint32_t>(a, list, count, grid, stream);
}

}  // namespace psi
