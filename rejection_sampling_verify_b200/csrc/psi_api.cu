// psi_api.cu - the C ABI: argument validation, workspace sizing, dispatch,
// and the counter-RNG kernel.  Declarations and documentation are in
// include/psi_verify.h.
#include <math.h>
#include <mutex>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "psi_internal.h"

namespace psi {

// out[s][r] = U(seed, seq, step, r, purpose)
__global__ void __launch_bounds__(256) rng_uniforms_kernel(uint64_t seed,
                                                           const uint64_t *__restrict__ seq_ids,
                                                           int32_t n_seq, uint64_t step,
                                                           int32_t n_rows, uint32_t purpose,
                                                           float *__restrict__ out) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (int64_t)n_seq * n_rows) return;
  const int64_t s = t / n_rows;
  const int32_t r = (int32_t)(t % n_rows);
  const uint64_t seq = seq_ids ? seq_ids[s] : (uint64_t)s;
  out[t] = uniform24(seed, seq, step, (uint64_t)r, purpose);
}

cudaError_t launch_rng_uniforms(uint64_t seed, const uint64_t *seq_ids, int32_t n_seq,
                                uint64_t step, int32_t n_rows, uint32_t purpose, float *out,
                                cudaStream_t stream) {
  const int64_t total = (int64_t)n_seq * n_rows;
  const int64_t blocks = (total + 255) / 256;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  rng_uniforms_kernel<<<(unsigned)blocks, 256, 0, stream>>>(seed, seq_ids, n_seq, step, n_rows,
                                                            purpose, out);
  return cudaGetLastError();
}

}  // namespace psi

namespace {

thread_local char g_last_error[256] = "";
thread_local psi::KernelEvents g_events;

psi_status fail(psi_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return st;
}

psi_status cuda_fail(cudaError_t e, const char *where) {
  return fail(PSI_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

int elem_bytes(psi_dtype dt) { return dt == PSI_DTYPE_F32 ? 4 : 2; }

bool valid_dtype(psi_dtype dt) { return dt == PSI_DTYPE_F32 || dt == PSI_DTYPE_BF16; }

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Largest vocabulary per element size that the shared-memory-resident
// sampled design holds (16 CTAs x 48 KB per row).
int32_t max_v(psi_dtype dt) { return dt == PSI_DTYPE_F32 ? PSI_MAX_V / 2 : PSI_MAX_V; }

bool aligned_to(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" {

const char *psi_status_string(psi_status status) {
  switch (status) {
    case PSI_OK: return "PSI_OK";
    case PSI_ERR_INVALID_ARG: return "PSI_ERR_INVALID_ARG";
    case PSI_ERR_MISALIGNED: return "PSI_ERR_MISALIGNED";
    case PSI_ERR_UNSUPPORTED: return "PSI_ERR_UNSUPPORTED";
    case PSI_ERR_CUDA: return "PSI_ERR_CUDA";
    case PSI_ERR_WORKSPACE: return "PSI_ERR_WORKSPACE";
    case PSI_ERR_TIMEOUT: return "PSI_ERR_TIMEOUT";
  }
  return "PSI_ERR_UNKNOWN";
}

const char *psi_last_error(void) { return g_last_error; }

size_t psi_verify_linear_workspace_bytes(int32_t N, int32_t B, int32_t V, psi_dtype dtype,
                                         float temperature, float top_p) {
  (void)top_p;
  if (N < 1 || B < 1 || B > PSI_MAX_B || V < 1 || !valid_dtype(dtype) || V > max_v(dtype))
    return 0;
  if (!(temperature >= 0.f) || !isfinite(temperature)) return 0;
  const int64_t rows = (int64_t)N * (B + 1);
  if (temperature == 0.f) {  // the every-row plan or the early-exit rounds, whichever is larger
    const psi::ArgmaxPlan plan = psi::plan_argmax(rows, V, elem_bytes(dtype));
    const size_t full = round256(sizeof(uint64_t) * (size_t)rows * plan.splits);
    const size_t rounds = round256(psi::greedy_layout(N, B, V, elem_bytes(dtype)).total);
    return full > rounds ? full : rounds;
  }
  (void)rows;
  return round256(psi::fast_layout(N, B).total);
}

static psi_status verify_linear(const void *ar_logits, int64_t ar_row_stride,
                             const void *draft_logits, int64_t draft_row_stride,
                             psi_dtype dtype, const int32_t *draft_ids, int32_t N, int32_t B,
                             int32_t V, float temperature, float top_p, int32_t top_k, uint64_t seed,
                             const uint64_t *seq_ids, uint64_t step, int32_t *out_tokens,
                             int32_t *out_n_emitted, float *out_p_draft, float *out_q_draft,
                             uint32_t *dev_status, void *workspace, size_t workspace_bytes,
                             psi_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!valid_dtype(dtype)) return fail(PSI_ERR_INVALID_ARG, "dtype %d", (int)dtype);
  if (N < 1 || B < 1 || B > PSI_MAX_B || V < 1)
    return fail(PSI_ERR_INVALID_ARG, "sizes N=%d B=%d V=%d (need N>=1, 1<=B<=%d, V>=1)", N, B, V,
                PSI_MAX_B);
  if (V > max_v(dtype))
    return fail(PSI_ERR_UNSUPPORTED, "V=%d above the supported %d for this dtype", V,
                max_v(dtype));
  if (!(temperature >= 0.f) || !isfinite(temperature))
    return fail(PSI_ERR_INVALID_ARG, "temperature %g (need finite, >= 0)", (double)temperature);
  const bool greedy = temperature == 0.f;
  if (!greedy && !(top_p > 0.f && top_p <= 1.f))
    return fail(PSI_ERR_INVALID_ARG, "top_p %g (need 0 < top_p <= 1)", (double)top_p);
  if (!ar_logits || !draft_ids || !out_tokens || !out_n_emitted || (!greedy && !draft_logits))
    return fail(PSI_ERR_INVALID_ARG, "null pointer argument");
  if (ar_row_stride < V || (!greedy && draft_row_stride < V))
    return fail(PSI_ERR_INVALID_ARG, "row stride below V");
  const size_t es = (size_t)elem_bytes(dtype);
  if (!aligned_to(ar_logits, es) || (!greedy && !aligned_to(draft_logits, es)) ||
      !aligned_to(draft_ids, 4) || !aligned_to(out_tokens, 4) || !aligned_to(out_n_emitted, 4) ||
      (seq_ids && !aligned_to(seq_ids, 8)) || (out_p_draft && !aligned_to(out_p_draft, 4)) ||
      (out_q_draft && !aligned_to(out_q_draft, 4)) || (dev_status && !aligned_to(dev_status, 4)))
    return fail(PSI_ERR_MISALIGNED, "pointer not aligned to its element type");
  const size_t need = psi_verify_linear_workspace_bytes(N, B, V, dtype, temperature, top_p);
  if (!workspace || workspace_bytes < need || !aligned_to(workspace, 16))
    return fail(PSI_ERR_WORKSPACE, "workspace %zu bytes at %p, need %zu (16-byte aligned)",
                workspace_bytes, workspace, need);

  const int64_t rows = (int64_t)N * (B + 1);
  cudaError_t e;
  if (greedy && !out_p_draft && !out_q_draft && N >= PSI_EARLY_EXIT_MIN_N) {
    // tokens only: rows after a sequence's first mismatch are never read
    e = psi::launch_greedy_early_exit(ar_logits, ar_row_stride, dtype, draft_ids, N, B, V,
                                      workspace, out_tokens, out_n_emitted, dev_status, g_events,
                                      stream);
    if (e != cudaSuccess) return cuda_fail(e, "greedy verify launch");
    return PSI_OK;
  }
  if (greedy) {
    const psi::ArgmaxPlan plan = psi::plan_argmax(rows, V, (int)es);
    uint64_t *partial = static_cast<uint64_t *>(workspace);
    if (g_events.before && (e = cudaEventRecord(g_events.before, stream)) != cudaSuccess)
      return cuda_fail(e, "event record");
    e = psi::launch_row_argmax(ar_logits, ar_row_stride, dtype, rows, V, plan, partial,
                               dev_status, stream);
    if (e != cudaSuccess) return cuda_fail(e, "row_argmax launch");
    if (g_events.after && (e = cudaEventRecord(g_events.after, stream)) != cudaSuccess)
      return cuda_fail(e, "event record");
    e = psi::launch_greedy_emit(partial, plan.splits, draft_ids, N, B, V, out_tokens,
                                out_n_emitted, dev_status, stream);
    if (e != cudaSuccess) return cuda_fail(e, "greedy_emit launch");
    return PSI_OK;
  }
  psi::SampledPlan plan;
  if (!psi::plan_sampled(V, (int)es, &plan))
    return fail(PSI_ERR_UNSUPPORTED, "V=%d does not fit the shared-memory plan", V);
  psi::SampledArgs a;
  a.ar = ar_logits;
  a.ar_stride = ar_row_stride;
  a.draft = draft_logits;
  a.draft_stride = draft_row_stride;
  a.ids = draft_ids;
  a.N = N;
  a.B = B;
  a.V = V;
  a.temperature = temperature;
  a.top_p = top_p;
  a.top_k = (top_k > 0 && top_k < V) ? top_k : 0;  // k >= V keeps every token
  a.seed = seed;
  a.seq_ids = seq_ids;
  a.step = step;
  a.out_tokens = out_tokens;
  a.out_n = out_n_emitted;
  a.out_p = out_p_draft;
  a.out_q = out_q_draft;
  a.dev_status = dev_status;
  a.records = static_cast<psi::UnitRecord *>(workspace);
  // The streaming path needs every row to start on a 16-byte boundary (its
  // loads are 16-byte vectors); other rows go to one cluster per unit, which
  // bulk-copies the aligned part of each row slice and loads the rest
  // element by element.
  const bool rows_aligned = aligned_to(ar_logits, 16) && aligned_to(draft_logits, 16) &&
                            ((size_t)ar_row_stride * es) % 16 == 0 &&
                            ((size_t)draft_row_stride * es) % 16 == 0;
  if (rows_aligned && psi::fast_path_fits(N, B)) {
    e = psi::launch_sampled_fast(a, dtype, plan, workspace, g_events, stream);
  } else if (a.top_k > 0) {  // the whole-row top-k path for every unit
    e = psi::launch_topk_units(a, dtype, nullptr, nullptr, (int64_t)N * (B + 1), stream);
    if (e == cudaSuccess) e = psi::launch_sampled_emit(a, stream);
  } else {
    e = psi::launch_sampled(a, dtype, plan, g_events, stream);
  }
  if (e != cudaSuccess) return cuda_fail(e, "sampled verify launch");
  return PSI_OK;
}

psi_status psi_verify_linear(const void *ar_logits, int64_t ar_row_stride,
                             const void *draft_logits, int64_t draft_row_stride,
                             psi_dtype dtype, const int32_t *draft_ids, int32_t N, int32_t B,
                             int32_t V, float temperature, float top_p, uint64_t seed,
                             const uint64_t *seq_ids, uint64_t step, int32_t *out_tokens,
                             int32_t *out_n_emitted, float *out_p_draft, float *out_q_draft,
                             uint32_t *dev_status, void *workspace, size_t workspace_bytes,
                             psi_stream_t stream) {
  return verify_linear(ar_logits, ar_row_stride, draft_logits, draft_row_stride, dtype, draft_ids,
                       N, B, V, temperature, top_p, 0, seed, seq_ids, step, out_tokens,
                       out_n_emitted, out_p_draft, out_q_draft, dev_status, workspace,
                       workspace_bytes, stream);
}

size_t psi_verify_linear_topk_workspace_bytes(int32_t N, int32_t B, int32_t V, psi_dtype dtype,
                                              float temperature, float top_p, int32_t top_k) {
  (void)top_k;
  return psi_verify_linear_workspace_bytes(N, B, V, dtype, temperature, top_p);
}

psi_status psi_verify_linear_topk(const void *ar_logits, int64_t ar_row_stride,
                                  const void *draft_logits, int64_t draft_row_stride,
                                  psi_dtype dtype, const int32_t *draft_ids, int32_t N, int32_t B,
                                  int32_t V, float temperature, float top_p, int32_t top_k,
                                  uint64_t seed, const uint64_t *seq_ids, uint64_t step,
                                  int32_t *out_tokens, int32_t *out_n_emitted, float *out_p_draft,
                                  float *out_q_draft, uint32_t *dev_status, void *workspace,
                                  size_t workspace_bytes, psi_stream_t stream) {
  if (top_k < 0) return fail(PSI_ERR_INVALID_ARG, "top_k %d (need >= 0; 0 = off)", (int)top_k);
  return verify_linear(ar_logits, ar_row_stride, draft_logits, draft_row_stride, dtype, draft_ids,
                       N, B, V, temperature, top_p, top_k, seed, seq_ids, step, out_tokens,
                       out_n_emitted, out_p_draft, out_q_draft, dev_status, workspace,
                       workspace_bytes, stream);
}

size_t psi_verify_tree_greedy_workspace_bytes(int32_t N, int32_t M, int32_t V, psi_dtype dtype) {
  if (N < 1 || M < 1 || M > PSI_MAX_TREE_NODES || V < 1 || !valid_dtype(dtype) ||
      V > max_v(dtype))
    return 0;
  return 256;  // the walk keeps its state in shared memory; any buffer will do
}

psi_status psi_verify_tree_greedy(const void *ar_logits, int64_t ar_row_stride, psi_dtype dtype,
                                  const int32_t *node_tokens, const int32_t *parents, int32_t N,
                                  int32_t M, int32_t V, int32_t *out_path_nodes,
                                  int32_t *out_path_len, int32_t *out_tokens,
                                  uint32_t *dev_status, void *workspace, size_t workspace_bytes,
                                  psi_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!valid_dtype(dtype)) return fail(PSI_ERR_INVALID_ARG, "dtype %d", (int)dtype);
  if (N < 1 || M < 1 || M > PSI_MAX_TREE_NODES || V < 1)
    return fail(PSI_ERR_INVALID_ARG, "sizes N=%d M=%d V=%d (need N>=1, 1<=M<=%d, V>=1)", N, M,
                V, PSI_MAX_TREE_NODES);
  if (V > max_v(dtype))
    return fail(PSI_ERR_UNSUPPORTED, "V=%d above the supported %d", V, max_v(dtype));
  if (!ar_logits || !node_tokens || !parents || !out_path_nodes || !out_path_len || !out_tokens)
    return fail(PSI_ERR_INVALID_ARG, "null pointer argument");
  if (ar_row_stride < V) return fail(PSI_ERR_INVALID_ARG, "row stride below V");
  const size_t es = (size_t)elem_bytes(dtype);
  if (!aligned_to(ar_logits, es) || !aligned_to(node_tokens, 4) || !aligned_to(parents, 4) ||
      !aligned_to(out_path_nodes, 4) || !aligned_to(out_path_len, 4) ||
      !aligned_to(out_tokens, 4) || (dev_status && !aligned_to(dev_status, 4)))
    return fail(PSI_ERR_MISALIGNED, "pointer not aligned to its element type");
  const size_t need = psi_verify_tree_greedy_workspace_bytes(N, M, V, dtype);
  if (!workspace || workspace_bytes < need || !aligned_to(workspace, 16))
    return fail(PSI_ERR_WORKSPACE, "workspace %zu bytes, need %zu", workspace_bytes, need);
  const cudaError_t e =
      psi::launch_tree_walk(ar_logits, ar_row_stride, dtype, node_tokens, parents, N, M, V,
                            out_path_nodes, out_path_len, out_tokens, dev_status, g_events,
                            stream);
  if (e != cudaSuccess) return cuda_fail(e, "tree_walk launch");
  return PSI_OK;
}

size_t psi_verify_tree_sampled_workspace_bytes(int32_t N, int32_t M, int32_t V, psi_dtype dtype,
                                               float temperature, float top_p) {
  (void)top_p;
  if (!(temperature >= 0.f) || !isfinite(temperature)) return 0;
  if (temperature == 0.f) return psi_verify_tree_greedy_workspace_bytes(N, M, V, dtype);
  if (N < 1 || M < 1 || M > PSI_MAX_TREE_NODES || V < 1 || !valid_dtype(dtype) ||
      V > max_v(dtype))
    return 0;
  return round256(psi::tree_layout(N, M).total);
}

psi_status psi_verify_tree_sampled(const void *ar_logits, int64_t ar_row_stride, psi_dtype dtype,
                                   const int32_t *node_tokens, const int32_t *parents, int32_t N,
                                   int32_t M, int32_t V, float temperature, float top_p,
                                   uint64_t seed, const uint64_t *seq_ids, uint64_t step,
                                   int32_t *out_path_nodes, int32_t *out_path_len,
                                   int32_t *out_tokens, uint32_t *dev_status, void *workspace,
                                   size_t workspace_bytes, psi_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!(temperature >= 0.f) || !isfinite(temperature))
    return fail(PSI_ERR_INVALID_ARG, "temperature %g (need finite, >= 0)", (double)temperature);
  if (temperature == 0.f)
    return psi_verify_tree_greedy(ar_logits, ar_row_stride, dtype, node_tokens, parents, N, M, V,
                                  out_path_nodes, out_path_len, out_tokens, dev_status,
                                  workspace, workspace_bytes, stream_);
  if (!valid_dtype(dtype)) return fail(PSI_ERR_INVALID_ARG, "dtype %d", (int)dtype);
  if (N < 1 || M < 1 || M > PSI_MAX_TREE_NODES || V < 1)
    return fail(PSI_ERR_INVALID_ARG, "sizes N=%d M=%d V=%d (need N>=1, 1<=M<=%d, V>=1)", N, M,
                V, PSI_MAX_TREE_NODES);
  if (V > max_v(dtype))
    return fail(PSI_ERR_UNSUPPORTED, "V=%d above the supported %d", V, max_v(dtype));
  if (!(top_p > 0.f && top_p <= 1.f))
    return fail(PSI_ERR_INVALID_ARG, "top_p %g (need 0 < top_p <= 1)", (double)top_p);
  if (!ar_logits || !node_tokens || !parents || !out_path_nodes || !out_path_len || !out_tokens)
    return fail(PSI_ERR_INVALID_ARG, "null pointer argument");
  if (ar_row_stride < V) return fail(PSI_ERR_INVALID_ARG, "row stride below V");
  const size_t es = (size_t)elem_bytes(dtype);
  if (!aligned_to(ar_logits, es) || !aligned_to(node_tokens, 4) || !aligned_to(parents, 4) ||
      !aligned_to(out_path_nodes, 4) || !aligned_to(out_path_len, 4) ||
      !aligned_to(out_tokens, 4) || (seq_ids && !aligned_to(seq_ids, 8)) ||
      (dev_status && !aligned_to(dev_status, 4)))
    return fail(PSI_ERR_MISALIGNED, "pointer not aligned to its element type");
  const size_t need = psi_verify_tree_sampled_workspace_bytes(N, M, V, dtype, temperature, top_p);
  if (!workspace || workspace_bytes < need || !aligned_to(workspace, 16))
    return fail(PSI_ERR_WORKSPACE, "workspace %zu bytes, need %zu", workspace_bytes, need);
  cudaError_t e = psi::launch_tree_sampled(ar_logits, ar_row_stride, dtype, node_tokens, parents,
                                           N, M, V, temperature, top_p, seed, seq_ids, step,
                                           out_path_nodes, out_path_len, out_tokens, dev_status,
                                           workspace, g_events, stream);
  if (e != cudaSuccess) return cuda_fail(e, "sampled tree launch");
  return PSI_OK;
}

psi_status psi_rng_uniforms(uint64_t seed, const uint64_t *seq_ids, int32_t n_seq, uint64_t step,
                            int32_t n_rows, uint32_t purpose, float *out, psi_stream_t stream_) {
  if (n_seq < 1 || n_rows < 1 || !out) return fail(PSI_ERR_INVALID_ARG, "n_seq/n_rows/out");
  if (!aligned_to(out, 4) || (seq_ids && !aligned_to(seq_ids, 8)))
    return fail(PSI_ERR_MISALIGNED, "pointer alignment");
  cudaError_t e = psi::launch_rng_uniforms(seed, seq_ids, n_seq, step, n_rows, purpose, out,
                                           reinterpret_cast<cudaStream_t>(stream_));
  if (e != cudaSuccess) return cuda_fail(e, "rng launch");
  return PSI_OK;
}

psi_status psi_profile_main_kernel(psi_event_t before, psi_event_t after) {
  if ((before == nullptr) != (after == nullptr))
    return fail(PSI_ERR_INVALID_ARG, "pass both events or neither");
  g_events.before = reinterpret_cast<cudaEvent_t>(before);
  g_events.after = reinterpret_cast<cudaEvent_t>(after);
  return PSI_OK;
}

// Scratch of psi_verify_linear_noalloc: part of the library's device module
// (one copy per device), so using it allocates nothing.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PSI_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kNoallocDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kNoallocDevices] = {};
}  // namespace

psi_status psi_verify_linear_noalloc(const void *ar_logits, int64_t ar_row_stride,
                                     const void *draft_logits, int64_t draft_row_stride,
                                     psi_dtype dtype, const int32_t *draft_ids, int32_t N,
                                     int32_t B, int32_t V, float temperature, float top_p,
                                     uint64_t seed, const uint64_t *seq_ids, uint64_t step,
                                     int32_t *out_tokens, int32_t *out_n_emitted,
                                     float *out_p_draft, float *out_q_draft,
                                     uint32_t *dev_status, psi_stream_t stream) {
  const size_t need = psi_verify_linear_workspace_bytes(N, B, V, dtype, temperature, top_p);
  if (need == 0)  // invalid sizes: psi_verify_linear reports the precise status
    return psi_verify_linear(ar_logits, ar_row_stride, draft_logits, draft_row_stride, dtype,
                             draft_ids, N, B, V, temperature, top_p, seed, seq_ids, step,
                             out_tokens, out_n_emitted, out_p_draft, out_q_draft, dev_status,
                             nullptr, 0, stream);
  if (need > (size_t)PSI_NOALLOC_SCRATCH_BYTES)
    return fail(PSI_ERR_UNSUPPORTED, "these sizes need %zu bytes of scratch, above the %zu held",
                need, (size_t)PSI_NOALLOC_SCRATCH_BYTES);
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kNoallocDevices)
    return fail(PSI_ERR_UNSUPPORTED, "device %d above the %d this entry point tracks", dev,
                kNoallocDevices);
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {  // once per device, with that device current
      void *p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
      g_noalloc_ptr[dev] = p;
    }
    scratch = g_noalloc_ptr[dev];
  }
  return psi_verify_linear(ar_logits, ar_row_stride, draft_logits, draft_row_stride, dtype,
                           draft_ids, N, B, V, temperature, top_p, seed, seq_ids, step,
                           out_tokens, out_n_emitted, out_p_draft, out_q_draft, dev_status,
                           scratch, (size_t)PSI_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
