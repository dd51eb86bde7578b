// psi_tree.cu - sampled (T > 0) verify of a draft tree per sequence.
//
// Sources (page title, section): "Uno Psi-Spec 是什麼？Diffusion-Augmented LLM
// 如何保留 AR 分布、一次驗證多個 Token" (alphalab.site), "Linear 與 Tree sampler"
// (several candidates per position kept in a finite prefix tree and verified
// in one pass) and "Uno Psi-Spec 怎麼運作？完整走一次四個 Token" (the rejection
// rule and the residual draw that a tree generalises); "想跑 Uno：先確認官方程式
// 需要的環境" (temperature, top-p).
//
// The pages give no sampled rule for the tree; the one taken is recursive
// rejection over the children of each reached node (the multi-candidate
// speculative sampling of SpecInfer, Miao et al., ASPLOS 2024), every child
// being its own point-mass proposal.  At a node whose AR row gives the target
// P (tempered, top-p cut), the valid children are tried in ascending index:
// child k with token x is accepted iff u_k * R < w(x), where w is what
// remains of P (a rejected token's mass is removed, so a later duplicate has
// none) and R = sum(w); u_k = U(seed, seq, step, k + 1, ACCEPT).  An accepted
// child becomes the next node.  When none is accepted (or the node is a
// leaf) the step ends with an inverse-CDF draw in vocabulary order from w (from
// P if nothing remains) at u' = U(seed, seq, step, row, RESID), row being the
// node's row (0 for the root).
//
// Kernels: the streaming row scan over every node row (psi_scan.cu) leaves
// each row's maximum, sum and candidates; the row finish (psi_finish.cuh, one
// warp per row, all rows at once) turns them into the row's maximum, top-p
// threshold and renormaliser (exact double masses, integer searches); then
// one CTA per tree walks the path, evaluates the children in double
// precision, and draws over the nucleus.  A row whose top-p set the candidate list cannot settle, and the
// draw when top-p is off (the whole vocabulary), take an exact whole-row path:
// the CTA re-reads the row (usually from L2) with double-precision masses in
// 2^40 fixed point (order-free integer sums).
#include <algorithm>

#include "psi_finish.cuh"

namespace psi {

namespace {

using namespace finish;

constexpr int kTreeThreads = 256;
constexpr int kTreeWarps = kTreeThreads / 32;
constexpr int kRemovedCap = PSI_MAX_TREE_NODES;   // rejected tokens at one node
constexpr double kFix40 = 1099511627776.0;        // 2^40: whole-row masses (V * 2^40 < 2^64)

struct TreeShared {
  WarpScratch ws;                       // the visited row's candidates (warp 0)
  int32_t removed[kRemovedCap];         // tokens rejected at the current node
  unsigned long long red[kTreeWarps];   // CTA reductions
  unsigned long long scan[kTreeThreads];
  RowFinal fin;                         // the visited row, as warp 0 finished it
  int next;                             // accepted child, or -1
  int n_removed;
  int token;
  uint32_t tau_key;                     // top-p threshold of the exact path
  double zp;                            // its nucleus mass (fixed-point units / 2^40)
};

// Sum over the CTA of one value per thread (every thread gets the total).
__device__ __forceinline__ unsigned long long cta_sum(unsigned long long v,
                                                      unsigned long long *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_u64(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  unsigned long long t = 0ull;
#pragma unroll
  for (int w = 0; w < kTreeWarps; ++w) t += red[w];
  return t;
}

__device__ __forceinline__ bool is_removed(const int32_t *removed, int n, int32_t v) {
  for (int j = 0; j < n; ++j)
    if (removed[j] == v) return true;
  return false;
}

// 2^40 fixed-point mass exp2((x - M) * coef) of one element if its key is at
// least key_lo and it is not excluded, else 0.
template <typename Bits>
__device__ __forceinline__ unsigned long long whole_row_mass(uint32_t bits, float M, double coef64,
                                                             uint32_t key_lo) {
  if (Elem<Bits>::key(bits) < key_lo) return 0ull;
  const double e = exact_exp2d(Elem<Bits>::to_float(bits), M, coef64);
  return e > 0.0 ? __double2ull_rn(fmin(e, 1.0) * kFix40) : 0ull;
}

// The contiguous range of elements thread t covers in a whole-row pass.
__device__ __forceinline__ void thread_range(int32_t V, int32_t &v0, int32_t &v1) {
  const int32_t ch = (V + kTreeThreads - 1) / kTreeThreads;
  v0 = min(V, (int32_t)threadIdx.x * ch);
  v1 = min(V, v0 + ch);
}

// CTA: sum of whole_row_mass over the row (excluding removed tokens if asked).
template <typename Bits>
__device__ unsigned long long whole_row_sum(const Bits *row, int32_t V, float M, double coef64,
                                            uint32_t key_lo, const int32_t *removed,
                                            int n_removed, unsigned long long *red) {
  int32_t v0, v1;
  thread_range(V, v0, v1);
  unsigned long long s = 0ull;
  for (int32_t v = v0; v < v1; ++v) {
    const unsigned long long m = whole_row_mass<Bits>((uint32_t)row[v], M, coef64, key_lo);
    if (m && !(n_removed && is_removed(removed, n_removed, v))) s += m;
  }
  return cta_sum(s, red);
}

// CTA: inverse-CDF draw in vocabulary order over the whole row with weights
// whole_row_mass (minus the removed tokens if any weight remains): the first v
// whose running sum exceeds floor(u' * W).  Returns the token (0 if no weight).
template <typename Bits>
__device__ int32_t whole_row_draw(const Bits *row, int32_t V, float M, double coef64,
                                  uint32_t key_lo, const int32_t *removed, int n_removed,
                                  float u2, TreeShared &sh) {
  int32_t v0, v1;
  thread_range(V, v0, v1);
  for (int attempt = 0; attempt < 2; ++attempt) {
    const int nr = attempt == 0 ? n_removed : 0;
    unsigned long long s = 0ull;
    for (int32_t v = v0; v < v1; ++v) {
      const unsigned long long m = whole_row_mass<Bits>((uint32_t)row[v], M, coef64, key_lo);
      if (m && !(nr && is_removed(removed, nr, v))) s += m;
    }
    // exclusive prefix over the threads, in vocabulary order
    sh.scan[threadIdx.x] = s;
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      unsigned long long carry = 0ull;
      for (int base = 0; base < kTreeThreads; base += 32) {
        const unsigned long long x = sh.scan[base + lane];
        unsigned long long incl = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += y;
        }
        sh.scan[base + lane] = carry + incl - x;
        carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
      }
      if (lane == 0) sh.red[0] = carry;
    }
    __syncthreads();
    const unsigned long long W = sh.red[0];
    if (W == 0ull) {
      __syncthreads();
      if (attempt == 0 && nr > 0) continue;  // nothing remains: draw from P itself
      return 0;
    }
    const unsigned long long k = (unsigned long long)(u2 * 16777216.0f);  // u' = k / 2^24
    const unsigned long long t = (__umul64hi(k, W) << 40) | ((k * W) >> 24);
    const unsigned long long before = sh.scan[threadIdx.x];
    if (threadIdx.x == 0) sh.token = 0;
    __syncthreads();
    if (before <= t && t < before + s) {  // exactly one thread holds the crossing
      unsigned long long run = before;
      for (int32_t v = v0; v < v1; ++v) {
        const unsigned long long m = whole_row_mass<Bits>((uint32_t)row[v], M, coef64, key_lo);
        if (!m || (nr && is_removed(removed, nr, v))) continue;
        run += m;
        if (run > t) {
          sh.token = v;
          break;
        }
      }
    }
    __syncthreads();
    return sh.token;
  }
  return 0;
}

template <typename Bits>
__global__ void __launch_bounds__(kTreeThreads) tree_sampled_kernel(
    const __grid_constant__ FastArgs a, const int32_t *__restrict__ tok,
    const int32_t *__restrict__ par, int32_t M, int32_t *__restrict__ out_path,
    int32_t *__restrict__ out_len, int32_t *__restrict__ out_tokens, int scanned) {
  pdl_wait();  // the previous kernel's results are visible
  pdl_trigger();
  extern __shared__ __align__(16) unsigned char tree_smem[];
  TreeShared &sh = *reinterpret_cast<TreeShared *>(tree_smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t n = blockIdx.x, V = a.s.V;
  const uint64_t seq = a.s.seq_ids ? a.s.seq_ids[n] : (uint64_t)n;
  const int32_t *tk = tok + (int64_t)n * M;
  const int32_t *pr = par + (int64_t)n * M;
  int32_t *path = out_path + (int64_t)n * M;
  int32_t *toks = out_tokens + (int64_t)n * (M + 1);

  // every node is checked (as the greedy tree does), reached or not
  uint32_t st = 0u;
  for (int32_t k = tid; k < M; k += kTreeThreads) {
    const int32_t p = pr[k];
    if (p < -1 || p >= k) st |= PSI_DEV_BAD_PARENT;
    else if (tk[k] < 0 || tk[k] >= V) st |= PSI_DEV_BAD_TOKEN_ID;
    path[k] = -1;
    toks[k] = -1;
  }
  if (tid == 0) toks[M] = -1;
  st = __reduce_or_sync(0xFFFFFFFFu, st);
  if (lane == 0 && st && a.s.dev_status) atomicOr(a.s.dev_status, st);
  __syncthreads();

  int32_t node = -1, depth = 0, token = 0;
  for (int32_t hop = 0; hop <= M; ++hop) {
    const int64_t r = (int64_t)n * (M + 1) + node + 1;
    const Bits *row = static_cast<const Bits *>(a.s.ar) + r * a.s.ar_stride;
    if (scanned) {
      if (tid == 0) {
        const RowFin rf = a.rfin[r];
        RowFinal f;
        f.m = rf.m;
        f.zp = rf.zp;
        f.tau_bits = rf.tau_bits;
        f.tau_key = rf.tau_key;
        f.n = rf.n;
        f.status = rf.status;
        sh.fin = f;
      }
    } else {  // rows that could not be scanned: the maximum by a whole-row pass
      int32_t v0, v1;
      thread_range(V, v0, v1);
      float m = -INFINITY;
      bool bad = false;
      for (int32_t v = v0; v < v1; ++v) {
        const uint32_t b = (uint32_t)row[v];
        bad |= Elem<Bits>::bad(b);
        m = fmaxf(m, Elem<Bits>::to_float(b));
      }
      m = warp_max(m);
      bad = __syncthreads_or(bad);
      if (lane == 0) sh.red[warp] = __float_as_uint(m);
      __syncthreads();
      if (tid == 0) {
        float mm = -INFINITY;
        for (int w = 0; w < kTreeWarps; ++w) mm = fmaxf(mm, __uint_as_float((uint32_t)sh.red[w]));
        RowFinal f;
        f.m = mm;
        f.zp = 0.0;
        f.tau_bits = Elem<Bits>::kNegInf;
        f.tau_key = 0u;
        f.n = 0;
        f.status = (bad || !(mm > -INFINITY) || !(fabsf(mm * a.coef) < INFINITY))
                       ? kFinNonfinite
                       : kFinOverflow;  // settled on the exact path below
        sh.fin = f;
      }
    }
    __syncthreads();
    const RowFinal fin = sh.fin;
    if (fin.status & kFinNonfinite) {  // undefined sequence: flagged, the walk stops
      if (tid == 0 && a.s.dev_status) atomicOr(a.s.dev_status, PSI_DEV_NONFINITE);
      token = 0;
      break;
    }
    // the row's target P: exact path when its top-p set did not fit the
    // candidates (the threshold by an integer search over the key range)
    const bool exact = (a.use_top_p || !scanned) && (fin.status & (kFinOverflow | kFinCoverage));
    uint32_t tau_key = fin.tau_key;
    double zp = fin.zp;  // P(x) = exp2((x - M) * coef) / zp
    if (exact && !a.use_top_p) {  // unscanned row without top-p: Z by a whole-row pass
      zp = (double)whole_row_sum<Bits>(row, V, fin.m, a.coef64, 0u, nullptr, 0, sh.red) / kFix40;
    } else if (exact) {
      const unsigned long long z = whole_row_sum<Bits>(row, V, fin.m, a.coef64, 0u, nullptr, 0,
                                                        sh.red);
      const double target = ceil((double)a.s.top_p * (double)z);
      uint32_t lo = 0u, hi = sizeof(Bits) == 2 ? 0x10000u : 0xFFFFFFFFu;  // S(lo) >= target
      unsigned long long s_lo = z;
      while (hi - lo > 1u) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        const unsigned long long s = whole_row_sum<Bits>(row, V, fin.m, a.coef64, mid, nullptr, 0,
                                                          sh.red);
        if ((double)s >= target) {
          lo = mid;
          s_lo = s;
        } else {
          hi = mid;
        }
      }
      tau_key = lo;
      zp = (double)s_lo / kFix40;
    }
    // children of the node in ascending index (warp 0): every lane loads its
    // child's logit and uniform at once, then the warp walks the children in
    // order with the same values in every lane (the tests are sequential)
    if (warp == 0) {
      double R = 1.0;  // mass of P not yet removed
      int nrem = 0, next = -1;
      for (int32_t base = node + 1; base < M && next < 0; base += 32) {
        const int32_t k = base + lane;
        bool child = false;
        int32_t x = 0;
        if (k < M) {
          const int32_t p = pr[k];
          x = tk[k];
          child = p == node && p < k && p >= -1 && x >= 0 && x < V;
        }
        double px = 0.0, u = 0.0;
        if (child) {
          const uint32_t bits = (uint32_t)row[x];
          if (Elem<Bits>::key(bits) >= tau_key && zp > 0.0)
            px = exact_exp2d(Elem<Bits>::to_float(bits), fin.m, a.coef64) / zp;
          u = uniform24(a.s.seed, seq, a.s.step, (uint64_t)(k + 1), PSI_PURPOSE_ACCEPT);
        }
        unsigned bal = __ballot_sync(0xFFFFFFFFu, child);
        while (bal && next < 0) {
          const int c = __ffs(bal) - 1;
          bal &= bal - 1;
          const double pxc = __shfl_sync(0xFFFFFFFFu, px, c);
          const double uc = __shfl_sync(0xFFFFFFFFu, u, c);
          const int32_t xc = __shfl_sync(0xFFFFFFFFu, x, c);
          const bool gone = is_removed(sh.removed, nrem, xc);
          if (uc * R < (gone ? 0.0 : pxc)) {
            next = base + c;
          } else if (!gone) {
            if (nrem < kRemovedCap) {
              if (lane == 0) sh.removed[nrem] = xc;
              ++nrem;
            }
            R -= pxc;
            __syncwarp();  // the removed token is visible to the next test
          }
        }
      }
      if (lane == 0) {
        sh.next = next;
        sh.n_removed = nrem;
      }
    }
    __syncthreads();
    const int next = sh.next;
    if (next >= 0) {
      if (tid == 0) {
        path[depth] = next;
        toks[depth] = tk[next];
      }
      ++depth;
      node = next;
      __syncthreads();
      continue;
    }
    // the draw from what remains of P at this node's row
    const float u2 = uniform24(a.s.seed, seq, a.s.step, (uint64_t)(node + 1), PSI_PURPOSE_RESID);
    const int nrem = sh.n_removed;
    if (!a.use_top_p || exact) {
      token = whole_row_draw<Bits>(row, V, fin.m, a.coef64, a.use_top_p ? tau_key : 0u,
                                   sh.removed, nrem, u2, sh);
    } else if (warp == 0) {
      // over p's nucleus (the row's candidates, compacted at the front of its
      // list area by the row finish, with key >= tau): index and exact mass,
      // remove the rejected tokens, then the integer search
      WarpScratch *ws = &sh.ws;
      const unsigned long long *area =
          reinterpret_cast<const unsigned long long *>(a.cand + r * (int64_t)kCandCap);
      int nn = 0;
      for (int base = 0; base < fin.n; base += 32 * kLoadChunk) {
        unsigned long long e[kLoadChunk];  // loads in flight together
#pragma unroll
        for (int h = 0; h < kLoadChunk; ++h) {
          const int j = base + 32 * h + lane;
          e[h] = j < fin.n ? __ldcg(area + j) : 0ull;
        }
        uint32_t inm = 0u;
#pragma unroll
        for (int h = 0; h < kLoadChunk; ++h) {
          const int j = base + 32 * h + lane;
          const bool in = j < fin.n && Elem<Bits>::key((uint32_t)(e[h] >> 32)) >= tau_key;
          inm |= (in ? 1u : 0u) << h;
        }
        const int cnt = __popc(inm);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += v;
        }
        int d = nn + incl - cnt;
        nn += __shfl_sync(0xFFFFFFFFu, incl, 31);
#pragma unroll
        for (int h = 0; h < kLoadChunk; ++h)
          if ((inm >> h) & 1u) {
            ws->idx[d] = (uint32_t)e[h];
            ws->m[d] = e[h] >> 32;  // the logit's bits until its mass replaces them
            ++d;
          }
      }
      __syncwarp();
      for (int j = lane; j < nn; j += 32)
        ws->m[j] = fixed52(exact_exp2d(Elem<Bits>::to_float((uint32_t)ws->m[j]), fin.m, a.coef64));
      __syncwarp();
      int32_t tkn = 0;
      for (int attempt = 0; attempt < 2; ++attempt) {
        const int nr = attempt == 0 ? nrem : 0;
        unsigned long long part = 0ull;
        for (int j = lane; j < nn; j += 32)
          if (!(nr && is_removed(sh.removed, nr, (int32_t)ws->idx[j]))) part += ws->m[j];
        const unsigned long long W = warp_sum_any(part);
        if (W == 0ull) continue;  // nothing remains: draw from P itself
        const unsigned long long kk = (unsigned long long)(u2 * 16777216.0f);
        const unsigned long long t = (__umul64hi(kk, W) << 40) | ((kk * W) >> 24);
        uint32_t lo = 0u, hi = (uint32_t)V;  // smallest X with C(X) > t; the token is X - 1
        while (hi - lo > 1u) {
          const uint32_t mid = (lo + hi) >> 1;
          unsigned long long cnt = 0ull;
          for (int j = lane; j < nn; j += 32)
            if (ws->idx[j] < mid && !(nr && is_removed(sh.removed, nr, (int32_t)ws->idx[j])))
              cnt += ws->m[j];
          cnt = warp_sum_any(cnt);
          if (cnt > t) hi = mid;
          else lo = mid;
        }
        tkn = (int32_t)lo;
        break;
      }
      if (lane == 0) sh.token = tkn;
    }
    __syncthreads();
    token = sh.token;
    break;
  }
  if (tid == 0) {
    toks[depth] = token;
    out_len[n] = depth;
  }
}

}  // namespace

TreeLayout tree_layout(int32_t N, int32_t M) {
  TreeLayout L;
  const int64_t rows = (int64_t)N * (M + 1);
  size_t off = 0;
  auto align = [](size_t x) { return (x + 255) / 256 * 256; };
  L.srec_off = off;
  off = align(off + sizeof(SliceRecord) * (size_t)rows * kMaxSlices);
  L.cand_off = off;
  off = align(off + sizeof(uint64_t) * (size_t)rows * kCandCap);
  L.known_off = off;
  off = align(off + sizeof(float) * (size_t)rows);
  L.rfin_off = off;
  off = align(off + sizeof(RowFin) * (size_t)rows);
  L.total = off;
  return L;
}

cudaError_t launch_tree_sampled(const void *ar, int64_t ar_stride, psi_dtype dtype,
                                const int32_t *node_tokens, const int32_t *parents, int32_t N,
                                int32_t M, int32_t V, float temperature, float top_p,
                                uint64_t seed, const uint64_t *seq_ids, uint64_t step,
                                int32_t *out_path, int32_t *out_len, int32_t *out_tokens,
                                uint32_t *dev_status, void *workspace, const KernelEvents &ev,
                                cudaStream_t stream) {
  const TreeLayout L = tree_layout(N, M);
  char *ws = static_cast<char *>(workspace);
  const int es = dtype == PSI_DTYPE_BF16 ? 2 : 4;
  FastArgs fa = {};
  fa.s.ar = ar;
  fa.s.ar_stride = ar_stride;
  fa.s.draft = nullptr;  // every scanned row is an AR row (rows < N * (M + 1))
  fa.s.draft_stride = ar_stride;
  fa.s.N = N;
  fa.s.B = M;
  fa.s.V = V;
  fa.s.temperature = temperature;
  fa.s.top_p = top_p;
  fa.s.seed = seed;
  fa.s.seq_ids = seq_ids;
  fa.s.step = step;
  fa.s.dev_status = dev_status;
  fa.g = plan_scan(V, es);
  fa.rows = (int64_t)N * (M + 1);
  fa.coef64 = 1.4426950408889634 / (double)temperature;
  fa.coef = (float)fa.coef64;
  double wlog2 = 13.0;  // the linear path's first-pass window
  if (top_p < 1.0f && top_p > 0.95f) wlog2 += log2(0.05 / (1.0 - (double)top_p));
  if (wlog2 > 20.0) wlog2 = 20.0;
  fa.win_narrow = fa.win_wide = (float)(wlog2 / fa.coef64);
  fa.use_top_p = top_p < 1.0f ? 1 : 0;
  fa.use_window = fa.use_top_p;
  fa.top_k = 0;
  fa.pass = 1;
  fa.srec = reinterpret_cast<SliceRecord *>(ws + L.srec_off);
  fa.cand = reinterpret_cast<uint64_t *>(ws + L.cand_off);
  fa.known_max = reinterpret_cast<float *>(ws + L.known_off);
  fa.rfin = reinterpret_cast<RowFin *>(ws + L.rfin_off);
  cudaError_t e;
  // the row scan streams 16-byte vectors; rows that do not start on a 16-byte
  // boundary are settled by the walk's exact whole-row path instead
  const int scanned = (reinterpret_cast<uintptr_t>(ar) % 16 == 0 &&
                       ((size_t)ar_stride * es) % 16 == 0) ? 1 : 0;
  if (scanned) {
    if (ev.before && (e = cudaEventRecord(ev.before, stream)) != cudaSuccess) return e;
    if ((e = launch_row_scan(fa, dtype, stream)) != cudaSuccess) return e;
    if (ev.after && (e = cudaEventRecord(ev.after, stream)) != cudaSuccess) return e;
    // every node row finished at once (the walk reads the rows it visits)
    if ((e = launch_row_finish(fa, dtype, stream)) != cudaSuccess) return e;
  }
  static DeviceOnce configure_bf16, configure_f32;
  const size_t smem = sizeof(TreeShared);
  if (dtype == PSI_DTYPE_BF16) {
    e = configure_bf16([smem] {
      return cudaFuncSetAttribute(tree_sampled_kernel<uint16_t>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (e != cudaSuccess) return e;
    return launch_pdl(tree_sampled_kernel<uint16_t>, dim3(N), dim3(kTreeThreads), smem, stream, fa,
                      node_tokens, parents, M, out_path, out_len, out_tokens, scanned);
  } else {
    e = configure_f32([smem] {
      return cudaFuncSetAttribute(tree_sampled_kernel<uint32_t>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (e != cudaSuccess) return e;
    return launch_pdl(tree_sampled_kernel<uint32_t>, dim3(N), dim3(kTreeThreads), smem, stream, fa,
                      node_tokens, parents, M, out_path, out_len, out_tokens, scanned);
  }
}

}  // namespace psi
