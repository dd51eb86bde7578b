// psi_internal.h - declarations shared by the library's translation units
// (launch plans and launchers).  Not part of the public ABI.
#pragma once

#include <utility>

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

// SM count of the current device (queried once per device).
inline int device_sm_count() {
  static std::atomic<int> cached[PerDevice::kMax] = {};
  const int dev = PerDevice::current();
  const bool slot = dev >= 0 && dev < PerDevice::kMax;
  int n = slot ? cached[dev].load(std::memory_order_relaxed) : 0;
  if (n > 0) return n;
  if (dev < 0 || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n <= 0)
    n = 148;
  if (slot) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

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

// The sampled path alternates kernels of very different shared-memory needs
// (the row scan takes nearly all of an SM's); every one of them asks for the
// largest shared-memory carveout, so that consecutive launches never wait for
// an SM to re-split its L1 / shared storage.
template <typename Kernel>
inline cudaError_t prefer_max_shared(Kernel *k) {
  return cudaFuncSetAttribute(reinterpret_cast<const void *>(k),
                              cudaFuncAttributePreferredSharedMemoryCarveout,
                              (int)cudaSharedmemCarveoutMaxShared);
}

// Early-exit round schedule: `short_rounds` rounds of `positions`
// positions, then one round with the rest of the B + 1 positions.
__host__ __device__ inline int32_t round_begin(int k, int32_t B, int short_rounds, int positions) {
  const int32_t b = k <= short_rounds ? k * positions : B + 1;
  return b < B + 1 ? b : B + 1;
}
__host__ __device__ inline int round_count(int32_t B, int short_rounds, int positions) {
  int k = 0;
  while (round_begin(k, B, short_rounds, positions) < B + 1) ++k;
  return k;
}
__host__ __device__ inline int32_t sampled_round_begin(int k, int32_t B) {
  return round_begin(k, B, PSI_SAMPLED_SHORT_ROUNDS, PSI_SAMPLED_ROUND_POSITIONS);
}
__host__ __device__ inline int32_t greedy_round_begin(int k, int32_t B) {
  return round_begin(k, B, PSI_GREEDY_SHORT_ROUNDS, PSI_GREEDY_ROUND_POSITIONS);
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

cudaError_t launch_tree_walk(const void *logits, int64_t row_stride, psi_dtype dtype,
                             const int32_t *node_tokens, const int32_t *parents, int32_t N,
                             int32_t M, int32_t V, int32_t *out_path_nodes,
                             int32_t *out_path_len, int32_t *out_tokens, uint32_t *dev_status,
                             const KernelEvents &ev, cudaStream_t stream);

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
  int32_t top_k;        // 0: off (else 1 <= top_k < V)
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

// Whole-row top-k path (psi_topk.cu): one CTA per listed unit (list and
// count on the device), or per unit of the batch (list == nullptr), records
// written; `max_ctas` caps the grid.
cudaError_t launch_topk_units(const SampledArgs &a, psi_dtype dtype, const int32_t *list,
                              const int32_t *count, int64_t max_ctas, cudaStream_t stream);
// The emit step of the general path (records -> tokens), one thread per sequence.
cudaError_t launch_sampled_emit(const SampledArgs &a, cudaStream_t stream);

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
// Each logit row is split into `slices` contiguous slices of 16-byte vectors
// (the last one also holds the V % vector-width tail elements), each scanned
// by its own CTA.  Per (row, slice) the scan leaves one record and the list of
// the elements it set aside: every element above the running top-p
// threshold of its stage (and the tail elements).  The row's final threshold
// is known only from all slices, so the finish sorts the set-aside elements
// into candidates (above it: exactly the elements the top-p cut can keep) and
// the rest of the sum.
struct SliceRecord {
  float m;         // reference of z: the slice maximum (or the known row maximum on a rescan)
  int32_t n_cand;  // elements set aside into the slice's list (above its capacity: overflow)
  int32_t flags;   // kRowLost: elements were dropped (the list overflowed)
  float off;       // the row's top-p window below its maximum (logit units) the scan used
  double z;        // sum over the slice's other elements of exp2((x - m) * log2(e) / T)
};
constexpr int32_t kRowLost = 1;
constexpr int kCandCap = 8192;   // set-aside elements kept per row (global workspace), split over slices
constexpr int kFinishCap = 2048; // candidates the finish holds per row
constexpr int kMaxSlices = 2;    // slice records reserved per row (slices per row at most)

// Candidate threshold in the element type: bf16 thresholds are rounded down,
// so rounding can only add candidates.  The scan and the finish round the
// same way.
template <typename Bits>
__device__ __forceinline__ float threshold_value(float thr) {
  if constexpr (sizeof(Bits) == 2)
    return __bfloat162float(__float2bfloat16_rd(thr));
  else
    return thr;
}

// How the scan splits a row (the same for every row of a call; chosen from V
// and the element size only, so per-row results do not depend on N).
struct ScanGeom {
  int32_t nvec;        // whole 16-byte vectors per row
  int32_t tail;        // elements after them (scanned by the last slice)
  int32_t slices;      // slices per row (CTAs per row)
  int32_t stages;      // shared-memory stages per slice
  int32_t stage_vecs;  // vectors per stage (the last stage of a slice may be shorter)
  int32_t cap;         // set-aside list capacity per slice (kCandCap / slices)
};
ScanGeom plan_scan(int32_t V, int elem_bytes);

struct FastLayout {  // workspace carve-up of the streaming path
  size_t rec_off, srec_off, cand_off, known_off, rfin_off, counters_off, list_a_off, list_b_off,
      list_d_off, list_k_off,
      wide_rows_off, wide_units_off, round_rows_off, round_units_off, active_off, total;
};
struct RowFin;  // a finished row (psi_finish.cuh)
FastLayout fast_layout(int32_t N, int32_t B);
// False when the streaming path's row indices would not fit its lists.
bool fast_path_fits(int32_t N, int32_t B);

// Launch with the programmatic-dependent-launch attribute: the kernel may
// start while the previous kernel on the stream drains (its pdl_wait() keeps
// it from reading that kernel's results early).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Everything the streaming path's kernels read.
struct FastArgs {
  SampledArgs s;
  ScanGeom g;
  int64_t rows;        // N*(B+1) AR rows followed by N*B draft rows
  float coef;          // log2(e) / T
  double coef64;
  float win_narrow;    // candidate windows below the row maximum, in logit units
  float win_wide;
  int use_top_p;
  int use_window;      // top-p or top-k: the scan sets elements near the maximum aside
  int32_t top_k;       // 0: off
  int pass;            // 1: a first scan / finish; 2: a rescan of rows that failed
  const int32_t *rlist;   // rows to scan (nullptr: every row); entries may carry kWideBit
  const int32_t *rcount;  // their number
  const int32_t *ulist;   // units to finish (nullptr: every unit)
  const int32_t *ucount;  // their number
  int32_t *active;        // [N] sequence still verifying (early-exit rounds)
  int32_t *round_rows;    // rows of the current round
  int32_t *round_units;   // units of the current round
  UnitRecord *rec;     // [N*(B+1)]
  SliceRecord *srec;   // [rows][kMaxSlices]
  uint64_t *cand;      // [rows][kCandCap]: slice c's set-aside list at c * g.cap;
                       // (bits << 32) | vocabulary index
  float *known_max;    // [rows] row maximum found by a first pass (read by a rescan)
  RowFin *rfin;        // [rows] the row finish's results (streaming linear verify)
  int32_t *counters;   // [0] general units, [1] sample-mode units, [2] wide rows, [3] wide units,
                       // [4 + 2k], [5 + 2k] rows and units of round parity k, [8] draw units,
                       // [9] whole-row top-k units
  int32_t *list_a;     // units for the general path
  int32_t *list_b;     // units whose draw needs the whole row
  int32_t *list_d;     // units whose draw is over their p row's nucleus
  int32_t *list_k;     // units for the whole-row top-k path
  int32_t *wide_rows;  // rows for the second scan (| kWideBit: wide window)
  int32_t *wide_units; // units for the second unit pass
};
constexpr int32_t kWideBit = int32_t(1) << 30;  // second-pass row entry: wide window

// The row scan over the listed rows (or every row): slice records and
// candidate lists.  `clusters_hint` caps the number of clusters launched.
cudaError_t launch_row_scan(const FastArgs &fa, psi_dtype dtype, cudaStream_t stream);

// The row finish over the listed rows (or every row): one warp per row,
// results to fa.rfin, candidates compacted in place (psi_fast.cu).
cudaError_t launch_row_finish(const FastArgs &fa, psi_dtype dtype, cudaStream_t stream);

cudaError_t launch_sampled_fast(const SampledArgs &a, psi_dtype dtype, const SampledPlan &plan,
                                void *workspace, const KernelEvents &ev, cudaStream_t stream);

// ---- sampled tree (psi_tree.cu) -------------------------------------------------
struct TreeLayout {  // workspace: the row scan's records and candidate lists
  size_t srec_off, cand_off, known_off, rfin_off, total;
};
TreeLayout tree_layout(int32_t N, int32_t M);
cudaError_t launch_tree_sampled(const void *ar, int64_t ar_stride, psi_dtype dtype,
                                const int32_t *node_tokens, const int32_t *parents, int32_t N,
                                int32_t M, int32_t V, float temperature, float top_p,
                                uint64_t seed, const uint64_t *seq_ids, uint64_t step,
                                int32_t *out_path, int32_t *out_len, int32_t *out_tokens,
                                uint32_t *dev_status, void *workspace, const KernelEvents &ev,
                                cudaStream_t stream);

cudaError_t launch_rng_uniforms(uint64_t seed, const uint64_t *seq_ids, int32_t n_seq,
                                uint64_t step, int32_t n_rows, uint32_t purpose, float *out,
                                cudaStream_t stream);

}  // namespace psi
