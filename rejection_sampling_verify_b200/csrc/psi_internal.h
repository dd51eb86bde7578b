// psi_internal.h - declarations shared by the library's translation units
// (launch plans and launchers).  Not part of the public ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "psi_device.cuh"
#include "psi_verify.h"

namespace psi {

// Host-side settings made once per device (launch attributes, device
// queries): one flag bit per device ordinal below 64; larger ordinals repeat
// the call every time.
struct PerDevice {
  static constexpr int kMax = 64;
  static int current() {
    int dev = 0;
    return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
  }
};

class DeviceOnce {
 public:
  // Runs f() unless it already succeeded on the current device.
  template <typename F>
  cudaError_t operator()(F &&f) {
    const int dev = PerDevice::current();
    const uint64_t bit = (dev >= 0 && dev < PerDevice::kMax) ? (1ull << dev) : 0ull;
    if (bit && (done_.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    const cudaError_t e = f();
    if (e == cudaSuccess && bit) done_.fetch_or(bit, std::memory_order_acq_rel);
    return e;
  }

 private:
  std::atomic<uint64_t> done_{0};
};

// Early-exit round schedule: `short_rounds` rounds of PSI_ROUND_POSITIONS
// positions, then one round with the rest of the B + 1 positions.
__host__ __device__ inline int32_t round_begin(int k, int32_t B, int short_rounds) {
  const int32_t b = k <= short_rounds ? k * PSI_ROUND_POSITIONS : B + 1;
  return b < B + 1 ? b : B + 1;
}
__host__ __device__ inline int round_count(int32_t B, int short_rounds) {
  int k = 0;
  while (round_begin(k, B, short_rounds) < B + 1) ++k;
  return k;
}

// ---- greedy paths ----------------------------------------------------------
struct ArgmaxPlan {
  int32_t splits = 1;  // CTAs per row
  int32_t chunk = 0;   // elements per CTA (multiple of the 16-byte vector)
};

ArgmaxPlan plan_argmax(int64_t rows, int32_t V, int elem_bytes);

cudaError_t launch_row_argmax(const void *logits, int64_t row_stride, psi_dtype dtype,
                              int64_t rows, int32_t V, const ArgmaxPlan &plan,
                              uint64_t *partial, uint32_t *dev_status, cudaStream_t stream);

cudaError_t launch_greedy_emit(const uint64_t *partial, int32_t splits, const int32_t *ids,
                               int32_t N, int32_t B, int32_t V, int32_t *out_tokens,
                               int32_t *out_n, uint32_t *dev_status, cudaStream_t stream);

// Greedy linear verify in early-exit rounds (rows of positions after a
// sequence's first mismatch are not read); workspace carve-up.
struct GreedyLayout {
  ArgmaxPlan plan;
  size_t partial_off, rows_off, counters_off, active_off, total;
};
GreedyLayout greedy_layout(int32_t N, int32_t B, int32_t V, int elem_bytes);
struct KernelEvents;
cudaError_t launch_greedy_early_exit(const void *logits, int64_t row_stride, psi_dtype dtype,
                                     const int32_t *ids, int32_t N, int32_t B, int32_t V,
                                     void *workspace, int32_t *out_tokens, int32_t *out_n,
                                     uint32_t *dev_status, const KernelEvents &ev,
                                     cudaStream_t stream);

cudaError_t launch_tree_walk(const uint64_t *partial, int32_t splits, const int32_t *node_tokens,
                             const int32_t *parents, int32_t N, int32_t M, int32_t V,
                             int32_t *out_path_nodes, int32_t *out_path_len,
                             int32_t *out_tokens, uint32_t *dev_status, cudaStream_t stream);

// ---- sampled linear path -----------------------------------------------------
// Per (sequence, row) record written by the unit kernel, read by the emit
// kernel.
struct UnitRecord {
  int32_t accept;  // row i < B: draft accepted
  int32_t token;   // correction (rejected row) or bonus (row B), else -1
};

struct SampledPlan {
  int32_t cluster = 1;   // CTAs per (sequence, row) unit
  int32_t slice = 0;     // vocabulary elements per CTA (multiple of the vector)
  int32_t nvec_pad = 0;  // 16-byte vectors per row buffer (multiple of 32)
  size_t smem = 0;       // dynamic shared memory per CTA
};

// Returns false if V does not fit the shared-memory-resident design.
bool plan_sampled(int32_t V, int elem_bytes, SampledPlan *plan);

struct SampledArgs {
  const void *ar;
  int64_t ar_stride;
  const void *draft;
  int64_t draft_stride;
  const int32_t *ids;
  int32_t N, B, V;
  float temperature;
  float top_p;
  uint64_t seed;
  const uint64_t *seq_ids;
  uint64_t step;
  int32_t *out_tokens;
  int32_t *out_n;
  float *out_p;
  float *out_q;
  uint32_t *dev_status;
  UnitRecord *records;  // workspace [N][B+1]
};

// Optional events recorded around the main kernel launch (instrumentation).
struct KernelEvents {
  cudaEvent_t before = nullptr;
  cudaEvent_t after = nullptr;
};

// General path: one cluster per unit for every unit, then the emit kernel.
cudaError_t launch_sampled(const SampledArgs &a, psi_dtype dtype, const SampledPlan &plan,
                           const KernelEvents &ev, cudaStream_t stream);

// The cluster kernel over a device-side list of units: full verify of each
// listed unit (kClusterModeList) or only its correction/bonus draw, written
// to out_tokens (kClusterModeSample).  `max_clusters` persistent clusters.
constexpr int kClusterModeList = 1;
constexpr int kClusterModeSample = 2;
cudaError_t launch_cluster_list(const SampledArgs &a, psi_dtype dtype, const SampledPlan &plan,
                                int mode, const int32_t *list, const int32_t *count,
                                int max_clusters, cudaStream_t stream);

// ---- streaming path (rows 16-byte aligned) ------------------------------------
// Per logit row: what the row-scan kernel leaves for the unit kernel.  Every
// element of the row is counted exactly once: in zt (at or below the
// threshold of its batch), in zd (above it, but at or below the row's final
// threshold) or in the row's candidate list (above the final threshold).
struct RowRecord {
  float ref;        // final running reference: the row maximum, unless the row holds +inf
  int32_t n_cand;   // candidates appended (more than the capacity: overflow)
  int32_t flags;    // kRowLost: flagged vectors were dropped (ring overflow)
  int32_t n_parked; // vectors parked by the scan (diagnostics)
  double zt;        // sum of exp2((x - ref) * log2(e) / T) over the unmasked elements
  uint64_t zd;      // 2^31 * the same sum over masked elements that are not candidates
};
constexpr int32_t kRowLost = 1;
constexpr int kCandCap = 2048;     // candidates kept per row (global workspace)

struct FastLayout {  // workspace carve-up of the streaming path
  size_t rec_off, rows_off, cand_off, counters_off, list_a_off, list_b_off, wide_rows_off,
      wide_units_off, round_rows_off, round_units_off, active_off, total;
};
FastLayout fast_layout(int32_t N, int32_t B);
// False when the streaming path's row indices would not fit its lists.
bool fast_path_fits(int32_t N, int32_t B);

cudaError_t launch_sampled_fast(const SampledArgs &a, psi_dtype dtype, const SampledPlan &plan,
                                void *workspace, const KernelEvents &ev, cudaStream_t stream);

cudaError_t launch_rng_uniforms(uint64_t seed, const uint64_t *seq_ids, int32_t n_seq,
                                uint64_t step, int32_t n_rows, uint32_t purpose, float *out,
                                cudaStream_t stream);

}  // namespace psi
