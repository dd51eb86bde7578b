// psi_greedy.cu - greedy (temperature 0) verify kernels.
//
//  row_argmax_kernel   argmax of every AR row, lowest index on ties.  Rows
//                      are split into chunks handled by separate CTAs; each
//                      CTA streams its chunk with 16-byte non-allocating
//                      loads (the data is consumed once, so it goes straight
//                      to registers) and writes one packed (key, ~index)
//                      word.  HBM-bound: 2 bytes per bf16 logit, no exp.
//  greedy_emit_kernel  linear rule: accept while x_i == argmax_i, emit the
//                      argmax of the first mismatching row (or the bonus row).
//  tree_greedy_walk_kernel  tree rule: node matched when its token is its
//                      parent row's argmax and its parent is matched;
//                      deepest matched node ends the path.  One cluster per
//                      tree reads only the root's and the matched nodes'
//                      rows, level by level.
//
// Sources: "Uno Psi-Spec 是什麼？..." (alphalab.site), section "Linear 與 Tree
// sampler" (tree verify); greedy linear verify is the temperature-0 case of
// the section "Uno Psi-Spec 怎麼運作？完整走一次四個 Token".
#include <algorithm>

#include "psi_internal.h"

namespace psi {

// Packed argmax word: order-preserving key in the high half, complemented
// index in the low half, so the unsigned maximum is the largest value and,
// among equal values, the lowest index.  0 never wins against a real element.
__device__ __forceinline__ uint64_t pack_argmax(uint32_t key, uint32_t idx) {
  return ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - idx);
}

// Running (value, index) maximum of one thread.  Values are compared as
// floats: -0 == +0, NaN never wins (it only raises the status bit).
struct RunMax {
  float val = -INFINITY;
  uint32_t idx = 0xFFFFFFFFu;
  bool bad = false;
};

template <typename Bits>
__device__ __forceinline__ void scan_scalar(uint32_t b, uint32_t idx, RunMax &rm) {
  rm.bad |= Elem<Bits>::bad(b);
  const float x = Elem<Bits>::to_float(b);
  if (x > rm.val || rm.idx == 0xFFFFFFFFu && !(x != x) && x == rm.val) {
    rm.val = x;
    rm.idx = idx;
  }
}

// One 16-byte vector whose first element has index `base`.  Each thread
// visits its indices in increasing order, so "strictly greater" keeps the
// lowest index among equal values.
template <typename Bits>
__device__ __forceinline__ void scan_vec(const uint4 &w, uint32_t base, RunMax &rm) {
  constexpr int VEC = Elem<Bits>::kVec;
  float vm;
  if constexpr (sizeof(Bits) == 2) {
    // packed bf16x2 maxima; the _nan form lets a NaN through so it is seen
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
  if (!(vm < INFINITY)) {  // a NaN or +inf is in this vector: exact path
#pragma unroll
    for (int k = 0; k < VEC; ++k) scan_scalar<Bits>(vec_elem<Bits>(w, k), base + k, rm);
    return;
  }
  if (vm > rm.val || (rm.idx == 0xFFFFFFFFu && vm == rm.val)) {
    uint32_t first = base;
#pragma unroll
    for (int k = VEC - 1; k >= 0; --k)
      if (Elem<Bits>::to_float(vec_elem<Bits>(w, k)) == vm) first = base + k;
    rm.val = vm;
    rm.idx = first;
  }
}

template <typename Bits>
__device__ __forceinline__ uint32_t float_key(float v) {
  if constexpr (sizeof(Bits) == 2)
    return Elem<Bits>::key(__float_as_uint(v) >> 16);
  else
    return Elem<Bits>::key(__float_as_uint(v));
}

// The packed argmax of elements [c0, c1) of row r, over the CTA (every
// thread gets it; 0 when the range is empty); any_bad: a NaN or +inf was
// seen.  `red` (kWarps words) is free again after the caller's next barrier.
// U: 16-byte loads in flight per thread.
template <typename Bits, int U = 4>
__device__ __forceinline__ uint64_t cta_chunk_argmax(const Bits *r, int32_t c0, int32_t c1,
                                                     uint64_t *red, bool &any_bad) {
  constexpr int VEC = Elem<Bits>::kVec;
  RunMax rm;

  // 16-byte aligned middle part [a0, a1), scalar head and tail.
  const uintptr_t addr0 = reinterpret_cast<uintptr_t>(r + c0);
  int32_t a0 = c0 + (int32_t)(((16u - (addr0 & 15u)) & 15u) / sizeof(Bits));
  if ((addr0 % sizeof(Bits)) != 0 || a0 > c1) a0 = c1;  // cannot vectorise
  const int32_t nvec = (c1 - a0) / VEC;
  const int32_t a1 = a0 + nvec * VEC;

  for (int32_t v = c0 + threadIdx.x; v < a0; v += kThreads) scan_scalar<Bits>(r[v], v, rm);

  const uint4 *vp = reinterpret_cast<const uint4 *>(r + a0);
  int32_t j = threadIdx.x;
  for (; j + (U - 1) * kThreads < nvec; j += U * kThreads) {
    uint4 w[U];
#pragma unroll
    for (int u = 0; u < U; ++u) w[u] = ldg_stream(vp + j + u * kThreads);
#pragma unroll
    for (int u = 0; u < U; ++u) scan_vec<Bits>(w[u], (uint32_t)(a0 + (j + u * kThreads) * VEC), rm);
  }
  for (; j < nvec; j += kThreads) scan_vec<Bits>(ldg_stream(vp + j), (uint32_t)(a0 + j * VEC), rm);

  for (int32_t v = a1 + threadIdx.x; v < c1; v += kThreads) scan_scalar<Bits>(r[v], v, rm);

  // A chunk made only of -inf/NaN reports its first index with the key of
  // -inf, so an all -inf row resolves to index 0 like everywhere else.
  uint64_t packed = 0;
  if (rm.idx != 0xFFFFFFFFu) packed = pack_argmax(float_key<Bits>(rm.val), rm.idx);
  else if (c0 < c1) packed = pack_argmax(float_key<Bits>(-INFINITY), (uint32_t)c0);
  packed = warp_max_u64(packed);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) red[warp] = packed;
  any_bad = __syncthreads_or(rm.bad);
  uint64_t x = 0ull;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) x = red[w] > x ? red[w] : x;
  return x;
}

// grid: rows * splits CTAs; CTA (item, s) covers [s*chunk, min(V, (s+1)*chunk))
// of row `item`, or of row rlist[item] for the first *rcount items when a
// row list is given (the other CTAs exit).
template <typename Bits>
__global__ void __launch_bounds__(kThreads) row_argmax_kernel(
    const Bits *__restrict__ logits, int64_t row_stride, int32_t V, int32_t splits,
    int32_t chunk, uint64_t *__restrict__ partial, uint32_t *dev_status,
    const int32_t *__restrict__ rlist, const int32_t *__restrict__ rcount) {
  pdl_wait();  // the previous kernel's results are visible
  pdl_trigger();
  const int64_t item = blockIdx.x / splits;
  const int32_t s = blockIdx.x % splits;
  if (rlist && item >= *rcount) return;
  const int64_t row = rlist ? (int64_t)rlist[item] : item;
  const int32_t c0 = s * chunk;
  __shared__ uint64_t red[kWarps];
  bool any_bad;
  const uint64_t x = cta_chunk_argmax<Bits>(logits + row * row_stride, c0, min(V, c0 + chunk),
                                            red, any_bad);
  if (threadIdx.x == 0) {
    partial[row * splits + s] = x;
    if (any_bad && dev_status) atomicOr(dev_status, PSI_DEV_NONFINITE);
  }
}

__device__ __forceinline__ int32_t argmax_of(const uint64_t *partial, int64_t row,
                                             int32_t splits) {
  uint64_t best = 0;
  for (int32_t s = 0; s < splits; ++s) {
    const uint64_t w = partial[row * splits + s];
    best = w > best ? w : best;
  }
  return (int32_t)(0xFFFFFFFFu - (uint32_t)best);
}

// One warp per sequence, lane i at position i.
static_assert(PSI_MAX_B <= 32, "one lane per drafted position");
__global__ void __launch_bounds__(128) greedy_emit_kernel(
    const uint64_t *__restrict__ partial, int32_t splits, const int32_t *__restrict__ ids,
    int32_t N, int32_t B, int32_t V, int32_t *__restrict__ out_tokens,
    int32_t *__restrict__ out_n, uint32_t *dev_status) {
  pdl_wait();  // the previous kernel's results are visible
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t n = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (n >= N) return;
  const int64_t row0 = n * (B + 1);
  bool bad_id = false, mismatch = false;
  if (lane < B) {
    const int32_t x = ids[n * B + lane];
    bad_id = x < 0 || x >= V;
    // with early exit the rows past a sequence's first mismatch were not
    // read in this call: only the lowest mismatch counts, and every row
    // before it was read
    mismatch = x != argmax_of(partial, row0 + lane, splits);
  }
  const uint32_t mm = __ballot_sync(0xFFFFFFFFu, mismatch);
  const int32_t L = mm ? __ffs(mm) - 1 : B;
  const int32_t am = argmax_of(partial, row0 + L, splits);
  int32_t *tok = out_tokens + n * (B + 1);
  for (int32_t i = lane; i <= B; i += 32) tok[i] = i < L ? ids[n * B + i] : (i == L ? am : -1);
  const bool any_bad = __any_sync(0xFFFFFFFFu, bad_id);
  if (lane == 0) {
    out_n[n] = L + 1;
    if (any_bad && dev_status) atomicOr(dev_status, PSI_DEV_BAD_TOKEN_ID);
  }
}

// Greedy tree, level by level: one cluster of C CTAs per tree (C = the
// cluster size, 1 to 8).  Only the rows that the rule needs are read: the
// root's and each matched node's.  A row's argmax is reduced over the
// cluster: CTA c scans elements [c * chunk, (c + 1) * chunk) and the C CTA
// maxima meet in distributed shared memory.  The matched children of a read
// row are queued in index order, so every CTA of the cluster reads the same
// rows in the same order and takes the same decisions.
constexpr int kWalkLoads = 8;       // 16-byte loads in flight per thread of the walk
constexpr int kWalkMaxCluster = 8;  // CTAs per tree at most

template <typename Bits>
__global__ void __launch_bounds__(kThreads) tree_greedy_walk_kernel(
    const Bits *__restrict__ logits, int64_t row_stride, int32_t V, int32_t chunk,
    const int32_t *__restrict__ node_tokens, const int32_t *__restrict__ parents, int32_t M,
    int32_t *__restrict__ out_path_nodes, int32_t *__restrict__ out_path_len,
    int32_t *__restrict__ out_tokens, uint32_t *dev_status) {
  pdl_wait();  // the previous kernel's results are visible
  pdl_trigger();
  extern __shared__ int32_t sm[];
  int32_t *par = sm;              // [M] parent; -2 for an invalid node
  int32_t *tok = par + M;         // [M]
  int32_t *depth = tok + M;       // [M] 0 = not matched
  int32_t *path = depth + M;      // [M]
  int32_t *queue = path + M;      // [M+1] rows to read, in order
  int32_t *am = queue + (M + 1);  // [M+1] argmax of each row read
  __shared__ uint64_t red[kWarps];
  // every CTA's maximum of the current row, slot[b][c] from CTA c (two buffers)
  __shared__ uint64_t slot[2][kWalkMaxCluster];
  __shared__ int32_t wcnt[kWarps];
  __shared__ uint32_t bad_nodes;
  __shared__ int32_t s_best, s_len;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t C = cluster_size(), rank = cluster_rank();
  const int64_t n = blockIdx.x / C;

  if (tid == 0) bad_nodes = 0u;
  __syncthreads();
  uint32_t st = 0u;
  for (int32_t k = tid; k < M; k += kThreads) {
    const int32_t p = parents[n * M + k], t = node_tokens[n * M + k];
    bool ok = true;
    if (p < -1 || p >= k) {
      st |= PSI_DEV_BAD_PARENT;
      ok = false;
    } else if (t < 0 || t >= V) {
      st |= PSI_DEV_BAD_TOKEN_ID;
      ok = false;
    }
    par[k] = ok ? p : -2;
    tok[k] = t;
    depth[k] = 0;
  }
  if (st) atomicOr(&bad_nodes, st);
  if (tid == 0) queue[0] = 0;  // the root's row
  __syncthreads();

  const Bits *rows = logits + n * (int64_t)(M + 1) * row_stride;
  const int32_t c0 = min(V, (int32_t)rank * chunk), c1 = min(V, c0 + chunk);
  bool bad_rows = false;
  int32_t qn = 1;  // rows queued (the same in every thread of the cluster)
  for (int32_t qi = 0; qi < qn; ++qi) {
    const int32_t row = queue[qi];
    bool bad;
    const uint64_t x =
        cta_chunk_argmax<Bits, kWalkLoads>(rows + row * row_stride, c0, c1, red, bad);
    bad_rows |= bad;
    if (tid < (int)C) dsmem_st_u64(dsmem_map(&slot[qi & 1][rank], (uint32_t)tid), x);
    // every CTA's maximum of the row has reached every CTA; `red` and the
    // other slot buffer are free (their readers are past this barrier)
    cluster_sync();
    uint64_t best = 0ull;
    for (uint32_t c = 0; c < C; ++c) best = slot[qi & 1][c] > best ? slot[qi & 1][c] : best;
    const int32_t a = (int32_t)(0xFFFFFFFFu - (uint32_t)best);
    if (tid == 0) am[row] = a;
    const int32_t pd = row == 0 ? 0 : depth[row - 1];
    // the row's node's children whose token is the argmax: matched, queued
    // in index order
    for (int32_t base = 0; base < M; base += kThreads) {
      const int32_t k = base + tid;
      const bool hit = k < M && par[k] == row - 1 && tok[k] == a;
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, hit);
      if (lane == 0) wcnt[warp] = __popc(bal);
      __syncthreads();
      int32_t off = qn, total = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        off += w < warp ? wcnt[w] : 0;
        total += wcnt[w];
      }
      if (hit) {
        depth[k] = pd + 1;
        queue[off + __popc(bal & ((1u << lane) - 1u))] = k + 1;
      }
      qn += total;
      __syncthreads();  // the queue and depths are visible; wcnt is free
    }
  }
  if (tid == 0 && bad_rows && dev_status) atomicOr(dev_status, PSI_DEV_NONFINITE);
  cluster_sync();  // no CTA leaves while another may still write its slots
  if (rank != 0) return;

  // the deepest matched node (lowest index among equals) ends the path
  if (tid == 0) {
    int32_t best = -1, best_depth = 0;
    for (int32_t k = 0; k < M; ++k)
      if (depth[k] > best_depth) {
        best_depth = depth[k];
        best = k;
      }
    int32_t d = best_depth;
    for (int32_t k = best; k >= 0; k = par[k]) path[--d] = k;
    s_best = best;
    s_len = best_depth;
    if (bad_nodes && dev_status) atomicOr(dev_status, bad_nodes);
  }
  __syncthreads();
  const int32_t len = s_len;
  for (int32_t k = tid; k < M; k += kThreads) out_path_nodes[n * M + k] = k < len ? path[k] : -1;
  for (int32_t k = tid; k <= M; k += kThreads) {
    int32_t v = -1;
    if (k < len) v = tok[path[k]];
    else if (k == len) v = am[s_best + 1];
    out_tokens[n * (M + 1) + k] = v;
  }
  if (tid == 0) out_path_len[n] = len;
}

// ---------------------------------------------------------------------------
// Host launchers.
// ---------------------------------------------------------------------------
size_t round_up256(size_t x) { return (x + 255) / 256 * 256; }

ArgmaxPlan plan_argmax(int64_t rows, int32_t V, int elem_bytes) {
  ArgmaxPlan p;
  const int vec = 16 / elem_bytes;
  // Aim for about 8 waves of 4 resident CTAs on each of a B200's 148 SMs, but
  // keep chunks >= 16 KB.  The split tunes speed only: the packed maxima make
  // the result the same for any split.
  const int64_t want_ctas = 148LL * 8 * 4;
  int64_t splits = (want_ctas + rows - 1) / rows;
  const int64_t min_chunk = 16384 / elem_bytes;
  const int64_t max_splits = (V + min_chunk - 1) / min_chunk;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  int64_t chunk = (V + splits - 1) / splits;
  chunk = (chunk + vec - 1) / vec * vec;
  splits = (V + chunk - 1) / chunk;
  p.splits = (int32_t)splits;
  p.chunk = (int32_t)chunk;
  return p;
}

cudaError_t launch_row_argmax(const void *logits, int64_t row_stride, psi_dtype dtype,
                              int64_t rows, int32_t V, const ArgmaxPlan &plan,
                              uint64_t *partial, uint32_t *dev_status, cudaStream_t stream) {
  const int64_t grid = rows * plan.splits;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  const int32_t *no_list = nullptr;
  if (dtype == PSI_DTYPE_BF16)
    return launch_pdl(row_argmax_kernel<uint16_t>, dim3((unsigned)grid), dim3(kThreads), 0, stream,
                      static_cast<const uint16_t *>(logits), row_stride, V, plan.splits,
                      plan.chunk, partial, dev_status, no_list, no_list);
  return launch_pdl(row_argmax_kernel<uint32_t>, dim3((unsigned)grid), dim3(kThreads), 0, stream,
                    static_cast<const uint32_t *>(logits), row_stride, V, plan.splits, plan.chunk,
                    partial, dev_status, no_list, no_list);
}

GreedyLayout greedy_layout(int32_t N, int32_t B, int32_t V, int elem_bytes) {
  GreedyLayout L;
  const int64_t rows = (int64_t)N * (B + 1);
  L.plan = plan_argmax((int64_t)N * std::min(B + 1, PSI_GREEDY_ROUND_POSITIONS), V, elem_bytes);
  size_t off = 0;
  L.partial_off = off;
  off = round_up256(off + sizeof(uint64_t) * (size_t)rows * L.plan.splits);
  L.rows_off = off;
  off = round_up256(off + sizeof(int32_t) * (size_t)N * (B + 1));
  L.counters_off = off;
  off = round_up256(off + sizeof(int32_t) * 4);
  L.active_off = off;
  off = round_up256(off + sizeof(int32_t) * (size_t)N);
  L.total = off;
  return L;
}

// One thread per sequence: the AR rows of early-exit round k (positions
// [greedy_round_begin(k), greedy_round_begin(k + 1)) of B + 1).  A sequence
// takes part when every draft of the earlier rounds matched its row's argmax.
__global__ void __launch_bounds__(128) greedy_advance_kernel(
    const uint64_t *__restrict__ partial, int32_t splits, const int32_t *__restrict__ ids,
    int32_t N, int32_t B, int k, int32_t *active, int32_t *round_rows, int32_t *counters) {
  pdl_wait();  // the previous kernel's results are visible
  pdl_trigger();
  const int32_t n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n == 0) counters[(k + 1) & 1] = 0;  // the next round's list
  if (n >= N) return;
  const int32_t i0 = greedy_round_begin(k, B);
  const int32_t i1 = greedy_round_begin(k + 1, B);
  const int64_t row0 = (int64_t)n * (B + 1);
  int act = 1;
  if (k > 0) {
    act = active[n];
    for (int32_t i = greedy_round_begin(k - 1, B); act && i < i0; ++i)
      if (i < B && ids[(int64_t)n * B + i] != argmax_of(partial, row0 + i, splits)) act = 0;
  }
  active[n] = act;
  if (!act || i0 >= i1) return;
  const int32_t at = atomicAdd(&counters[k & 1], i1 - i0);
  for (int32_t i = i0; i < i1; ++i) round_rows[at + (i - i0)] = (int32_t)(row0 + i);
}

cudaError_t launch_greedy_early_exit(const void *logits, int64_t row_stride, psi_dtype dtype,
                                     const int32_t *ids, int32_t N, int32_t B, int32_t V,
                                     void *workspace, int32_t *out_tokens, int32_t *out_n,
                                     uint32_t *dev_status, const KernelEvents &ev,
                                     cudaStream_t stream) {
  const GreedyLayout L = greedy_layout(N, B, V, dtype == PSI_DTYPE_F32 ? 4 : 2);
  char *ws = static_cast<char *>(workspace);
  uint64_t *partial = reinterpret_cast<uint64_t *>(ws + L.partial_off);
  int32_t *rows = reinterpret_cast<int32_t *>(ws + L.rows_off);
  int32_t *counters = reinterpret_cast<int32_t *>(ws + L.counters_off);
  int32_t *active = reinterpret_cast<int32_t *>(ws + L.active_off);
  if ((int64_t)N * (B + 1) * L.plan.splits > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  cudaError_t e;
  if ((e = cudaMemsetAsync(counters, 0, 4 * sizeof(int32_t), stream)) != cudaSuccess) return e;
  const int rounds = round_count(B, PSI_GREEDY_SHORT_ROUNDS, PSI_GREEDY_ROUND_POSITIONS);
  for (int k = 0; k < rounds; ++k) {
    const int64_t grid = (int64_t)N *
                         (greedy_round_begin(k + 1, B) - greedy_round_begin(k, B)) *
                         L.plan.splits;
    if ((e = launch_pdl(greedy_advance_kernel, dim3((N + 127) / 128), dim3(128), 0, stream,
                        static_cast<const uint64_t *>(partial), L.plan.splits, ids, N, B, k,
                        active, rows, counters)) != cudaSuccess)
      return e;
    if (k == 0 && ev.before && (e = cudaEventRecord(ev.before, stream)) != cudaSuccess) return e;
    const int32_t *rl = rows, *rc = counters + (k & 1);
    if (dtype == PSI_DTYPE_BF16)
      e = launch_pdl(row_argmax_kernel<uint16_t>, dim3((unsigned)grid), dim3(kThreads), 0, stream,
                     static_cast<const uint16_t *>(logits), row_stride, V, L.plan.splits,
                     L.plan.chunk, partial, dev_status, rl, rc);
    else
      e = launch_pdl(row_argmax_kernel<uint32_t>, dim3((unsigned)grid), dim3(kThreads), 0, stream,
                     static_cast<const uint32_t *>(logits), row_stride, V, L.plan.splits,
                     L.plan.chunk, partial, dev_status, rl, rc);
    if (e != cudaSuccess) return e;
    if (k == 0 && ev.after && (e = cudaEventRecord(ev.after, stream)) != cudaSuccess) return e;
  }
  return launch_greedy_emit(partial, L.plan.splits, ids, N, B, V, out_tokens, out_n, dev_status,
                            stream);
}

cudaError_t launch_greedy_emit(const uint64_t *partial, int32_t splits, const int32_t *ids,
                               int32_t N, int32_t B, int32_t V, int32_t *out_tokens,
                               int32_t *out_n, uint32_t *dev_status, cudaStream_t stream) {
  return launch_pdl(greedy_emit_kernel, dim3((N + 3) / 4), dim3(128), 0, stream, partial,
                    splits, ids, N, B, V, out_tokens, out_n, dev_status);
}

template <typename Bits>
cudaError_t launch_tree_walk_typed(const Bits *logits, int64_t row_stride,
                                   const int32_t *node_tokens, const int32_t *parents, int32_t N,
                                   int32_t M, int32_t V, int32_t *out_path_nodes,
                                   int32_t *out_path_len, int32_t *out_tokens,
                                   uint32_t *dev_status, const KernelEvents &ev,
                                   cudaStream_t stream) {
  // the cluster spreads a tree's rows over up to 8 SMs while the trees
  // leave SMs idle
  int C = kWalkMaxCluster;
  while (C > 1 && (int64_t)N * C > 2LL * device_sm_count()) C >>= 1;
  if ((int64_t)N * C > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  constexpr int VEC = Elem<Bits>::kVec;
  const int32_t chunk = ((V + C - 1) / C + VEC - 1) / VEC * VEC;
  const size_t smem = sizeof(int32_t) * (size_t)(6 * M + 2);
  static DeviceOnce configure;  // opt in to > 48 KB once per device (only large M needs it)
  const cudaError_t ce = configure([] {
    return cudaFuncSetAttribute(tree_greedy_walk_kernel<Bits>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(6 * PSI_MAX_TREE_NODES + 2) * 4);
  });
  if (ce != cudaSuccess) return ce;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(N * C), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_pdl
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e;
  if (ev.before && (e = cudaEventRecord(ev.before, stream)) != cudaSuccess) return e;
  e = cudaLaunchKernelEx(&cfg, tree_greedy_walk_kernel<Bits>, logits, row_stride, V, chunk,
                         node_tokens, parents, M, out_path_nodes, out_path_len, out_tokens,
                         dev_status);
  if (e != cudaSuccess) return e;
  if (ev.after && (e = cudaEventRecord(ev.after, stream)) != cudaSuccess) return e;
  return cudaSuccess;
}

cudaError_t launch_tree_walk(const void *logits, int64_t row_stride, psi_dtype dtype,
                             const int32_t *node_tokens, const int32_t *parents, int32_t N,
                             int32_t M, int32_t V, int32_t *out_path_nodes,
                             int32_t *out_path_len, int32_t *out_tokens, uint32_t *dev_status,
                             const KernelEvents &ev, cudaStream_t stream) {
  if (dtype == PSI_DTYPE_BF16)
    return launch_tree_walk_typed(static_cast<const uint16_t *>(logits), row_stride, node_tokens,
                                  parents, N, M, V, out_path_nodes, out_path_len, out_tokens,
                                  dev_status, ev, stream);
  return launch_tree_walk_typed(static_cast<const uint32_t *>(logits), row_stride, node_tokens,
                                parents, N, M, V, out_path_nodes, out_path_len, out_tokens,
                                dev_status, ev, stream);
}

}  // namespace psi
