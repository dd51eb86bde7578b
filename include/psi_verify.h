/*
 * psi_verify.h - C ABI of the Psi-Spec verify step on NVIDIA B200 (sm_100a).
 *
 * The verify step of the Psi-Spec sampler: the frozen AR path has scored a
 * block of B drafted tokens (B+1 logit rows, the last one being the bonus
 * row), the diffusion-LoRA draft supplied B logit rows and the drafted ids.
 * Per sequence the step keeps the longest prefix of drafted tokens that
 * passes speculative rejection sampling, then emits one correction token
 * (drawn from the residual at the first rejection) or one bonus token (drawn
 * from the bonus row when every draft passed).
 *
 * Sources (page title, section):
 *  [P1] "Uno / Psi-Spec - 같은 모델 안에서 초안 뽑고 AR로 도장 찍기"
 *       (lanes-ecd.pages.dev): "어디서 왔나" (the Leviathan et al. 2023
 *       draft -> verify -> correct rule), "Psi-Spec이 한 스텝에서 하는 일"
 *       (longest consecutive accepted prefix; lossless).
 *  [P3] "Uno Psi-Spec 是什麼？Diffusion-Augmented LLM 如何保留 AR 分布、
 *       一次驗證多個 Token" (alphalab.site): "Uno Psi-Spec 怎麼運作？完整走一次
 *       四個 Token" (steps 3-4: rejection rule, longest accepted prefix,
 *       residual correction; bonus token from the block-end logits; TPF
 *       bound), "Linear 與 Tree sampler" (tree verify), "想跑 Uno：先確認官方
 *       程式需要的環境" (temperature and top-p on the run card).
 *
 * Conventions shared by every entry point:
 *  - All array arguments are DEVICE pointers owned by the caller.  The
 *    library allocates nothing and keeps no data between calls (only
 *    per-device launch settings, made on a device's first call).
 *  - Calls are asynchronous on `stream` (NULL = the legacy default stream).
 *    After a device's first call, a call only launches work on `stream`, so
 *    it can be captured into a CUDA graph; its scalar arguments (seed, step,
 *    sizes) are then fixed in the graph.
 *  - Argument errors are detected on the host before any launch and
 *    returned as a psi_status; nothing is launched in that case.
 *  - Data errors found on the device (an id outside [0, V), a bad parent
 *    index, a NaN or +inf logit) are OR-ed into *dev_status (a caller-owned
 *    device uint32 that the caller zeroes; NULL = not reported).  The
 *    kernels always run to completion: they never trap, and the only waits
 *    (for bulk copies into shared memory) give up after a time limit.
 *  - Logits are bfloat16 or float32, row-major; `*_row_stride` is the
 *    distance between consecutive rows in ELEMENTS (>= V).  Sampled rows
 *    whose start is 16-byte aligned take the streaming path, others the
 *    cluster path; both give the same results.
 *  - Randomness: the acceptance uniform of row i and the correction/bonus
 *    uniform of the emitting row are a counter-based hash of
 *    (seed, sequence id, step, row, purpose), so a step replays exactly from
 *    its counters and results do not depend on batch composition.
 */
#ifndef PSI_VERIFY_H
#define PSI_VERIFY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *psi_stream_t; /* same type as cudaStream_t */

typedef enum psi_status {
  PSI_OK = 0,
  PSI_ERR_INVALID_ARG = 1, /* null pointer, size or parameter out of range */
  PSI_ERR_MISALIGNED = 2,  /* pointer not aligned to its element type */
  PSI_ERR_UNSUPPORTED = 3, /* valid but beyond this build (e.g. V too large) */
  PSI_ERR_CUDA = 4,        /* a CUDA launch or query failed */
  PSI_ERR_WORKSPACE = 5,   /* workspace NULL or smaller than the query says */
  PSI_ERR_TIMEOUT = 6      /* reserved, not returned: a kernel's wait that
                              gives up sets PSI_DEV_TIMEOUT instead */
} psi_status;

typedef enum psi_dtype { PSI_DTYPE_F32 = 0, PSI_DTYPE_BF16 = 1 } psi_dtype;

/* Bits OR-ed into *dev_status by the kernels. */
#define PSI_DEV_BAD_TOKEN_ID 1u /* drafted or node id outside [0, V): treated
                                   as rejected / unmatched */
#define PSI_DEV_BAD_PARENT 2u   /* parent index >= own index or < -1: node
                                   unmatched */
#define PSI_DEV_NONFINITE 4u    /* a NaN or +inf logit was read (-inf is a
                                   valid logit: probability zero) */
#define PSI_DEV_TIMEOUT 8u      /* a bounded wait inside a kernel gave up;
                                   never expected; outputs are then invalid */

/* RNG purposes (the last hash input). */
#define PSI_PURPOSE_ACCEPT 0u /* u_i of the acceptance test of row i */
#define PSI_PURPOSE_RESID 1u  /* u' of the correction / bonus draw */

/* Largest supported block and vocabulary. */
#define PSI_MAX_B 32
#define PSI_MAX_V 393216
#define PSI_MAX_TREE_NODES 4096
/* Early-exit rounds of the linear verify (see psi_verify_linear): the first
 * PSI_X_SHORT_ROUNDS rounds cover PSI_X_ROUND_POSITIONS positions each, one
 * last round covers the rest of the B + 1 positions (X = SAMPLED for T > 0,
 * GREEDY for T == 0). */
#define PSI_SAMPLED_ROUND_POSITIONS 2
#define PSI_SAMPLED_SHORT_ROUNDS 2
#define PSI_GREEDY_ROUND_POSITIONS 3
#define PSI_GREEDY_SHORT_ROUNDS 3
/* Smallest batch that takes the early-exit rounds (smaller batches are
 * latency-bound: one pass over every row is faster). */
#define PSI_EARLY_EXIT_MIN_N 64

/* Workspace needed by psi_verify_linear for these sizes (bytes, a multiple
 * of 256; 0 on invalid sizes).  The workspace needs no initialisation. */
size_t psi_verify_linear_workspace_bytes(int32_t N, int32_t B, int32_t V,
                                         psi_dtype dtype, float temperature,
                                         float top_p);

/*
 * psi_verify_linear - linear (single-path) verify of N sequences.
 *
 * [P1] "Psi-Spec이 한 스텝에서 하는 일"; [P3] "完整走一次四個 Token" steps
 * 3-4 and the bonus paragraph; temperature / top-p: [P3] run card.
 *
 * For T > 0, per sequence n and row i:
 *   p_i = softmax(ar[n][i] / T), q_i = softmax(draft[n][i] / T); with
 *   top_p < 1 each is cut to its smallest descending-probability set of mass
 *   >= top_p (keeping every token tied with the last one admitted) and
 *   renormalised.  Draft x_i is accepted iff u_i * q_i(x_i) < p_i(x_i) with
 *   u_i = U(seed, seq, step, i, ACCEPT).  L = first rejected row (B if none).
 *   If L < B the correction is the inverse-CDF draw, in vocabulary order,
 *   from max(0, p_L - q_L) at u' = U(seed, seq, step, L, RESID) (from p_L
 *   itself if that residual is all zero, which needs q_L(x_L) = 0); if
 *   L == B the bonus token is drawn from p_B the same way.
 * For T == 0 (greedy): a_i = argmax of ar[n][i] (lowest index on ties);
 *   accept while x_i == a_i; emit a_L.  draft_logits may be NULL and top_p
 *   is ignored.
 *
 * ar_logits     [N][B+1] rows of V logits (row B = bonus row), stride
 *               ar_row_stride elements.
 * draft_logits  [N][B] rows, stride draft_row_stride (ignored if T == 0).
 * draft_ids     int32 [N][B].
 * seq_ids       uint64 [N] sequence ids for the RNG, or NULL (= n).
 * out_tokens    int32 [N][B+1]: x_0..x_{L-1}, then the emitted token, then -1.
 * out_n_emitted int32 [N]: L + 1, in 1..B+1.
 * out_p_draft, out_q_draft  float [N][B] or NULL: p_i(x_i), q_i(x_i) after
 *               top-p (T > 0 only; not written when T == 0).
 * Early exit (both out_p_draft and out_q_draft NULL, N >= PSI_EARLY_EXIT_MIN_N,
 *   any T): rows after a sequence's first rejection (or greedy mismatch) do
 *   not change its result, so positions are verified in rounds
 *   (PSI_SAMPLED_ROUND_POSITIONS positions each for the first
 *   PSI_SAMPLED_SHORT_ROUNDS rounds, PSI_GREEDY_ROUND_POSITIONS for the first
 *   PSI_GREEDY_SHORT_ROUNDS, then the rest), and a sequence takes
 *   part in a round only if every draft of the earlier rounds was accepted.
 *   Tokens and counts are the same as with every row read; the NONFINITE
 *   status bit then covers the rows that were read.  A caller passing p / q
 *   buffers (for T == 0 they are not written) gets every row read.
 * Limits: 1 <= N, 1 <= B <= PSI_MAX_B, 1 <= V <= PSI_MAX_V, T >= 0 and
 *   finite, 0 < top_p <= 1.
 */
psi_status psi_verify_linear(const void *ar_logits, int64_t ar_row_stride,
                             const void *draft_logits,
                             int64_t draft_row_stride, psi_dtype dtype,
                             const int32_t *draft_ids, int32_t N, int32_t B,
                             int32_t V, float temperature, float top_p,
                             uint64_t seed, const uint64_t *seq_ids,
                             uint64_t step, int32_t *out_tokens,
                             int32_t *out_n_emitted, float *out_p_draft,
                             float *out_q_draft, uint32_t *dev_status,
                             void *workspace, size_t workspace_bytes,
                             psi_stream_t stream);

/* Workspace needed by psi_verify_linear_topk (bytes; the same as
 * psi_verify_linear's for these sizes; 0 on invalid sizes). */
size_t psi_verify_linear_topk_workspace_bytes(int32_t N, int32_t B, int32_t V,
                                              psi_dtype dtype, float temperature,
                                              float top_p, int32_t top_k);

/*
 * psi_verify_linear_topk - psi_verify_linear with a top-k cut.
 *
 * Source: the run card ("想跑 Uno：先確認官方程式需要的環境") names top-k
 * beside top-p and temperature as sampler settings.  Reading of the order:
 * top-k is taken on the temperature softmax first (every token whose
 * probability is at least the k-th largest stays, ties with the k-th
 * included), the kept mass is renormalised, and top-p then cuts that
 * distribution as in psi_verify_linear.  It applies to p_i and q_i alike, so
 * the acceptance test, the residual and the bonus draw all use the cut
 * distributions.
 *
 * Arguments, results, layouts and limits as psi_verify_linear, plus
 * top_k: 0 = off; top_k >= V keeps every token (also off); negative values
 *   return PSI_ERR_INVALID_ARG.  Ignored when T == 0 (the argmax is always
 *   kept).
 * With top_k off the call is psi_verify_linear.  Rows whose set-aside
 * candidates (the elements near the maximum that the streaming scan keeps)
 * number at least k are finished from them; the other units (large k, flat
 * rows, or rows that do not start on a 16-byte boundary) go to a slower
 * whole-row path that reads their two rows a few more times.  Results do
 * not depend on which path a unit takes.
 */
psi_status psi_verify_linear_topk(const void *ar_logits, int64_t ar_row_stride,
                                  const void *draft_logits,
                                  int64_t draft_row_stride, psi_dtype dtype,
                                  const int32_t *draft_ids, int32_t N, int32_t B,
                                  int32_t V, float temperature, float top_p,
                                  int32_t top_k, uint64_t seed,
                                  const uint64_t *seq_ids, uint64_t step,
                                  int32_t *out_tokens, int32_t *out_n_emitted,
                                  float *out_p_draft, float *out_q_draft,
                                  uint32_t *dev_status, void *workspace,
                                  size_t workspace_bytes, psi_stream_t stream);

/*
 * psi_verify_linear_noalloc - psi_verify_linear for callers that cannot
 * allocate device memory (no counterpart on the pages: an integration
 * variant, same arithmetic and results as psi_verify_linear).
 *
 * Arguments and results as psi_verify_linear, without the workspace: the
 * call uses a scratch array of PSI_NOALLOC_SCRATCH_BYTES that the library
 * holds in device memory (one per device, created with the library's module;
 * nothing is allocated at run time).  Its address is looked up once per
 * device, on the first call made with that device current; make that first
 * call before capturing the stream into a graph, since it issues a
 * runtime query besides the launches.  The address is kept for the life of
 * the process: it belongs to the device's primary context, so after that
 * context is torn down (cudaDeviceReset) this entry point must not be used
 * on that device again until the library is reloaded.  The scratch needs no initialisation:
 * what the verify needs zeroed it clears itself on every call.
 * Calls that overlap in time on the same device share the scratch and race:
 * the caller serialises them (one stream, or events between streams).
 * Returns PSI_ERR_UNSUPPORTED, without launching anything, when
 * psi_verify_linear_workspace_bytes for these sizes exceeds
 * PSI_NOALLOC_SCRATCH_BYTES (the sampled path needs about 65.7 KB per logit
 * row, N * (2B + 1) rows: e.g. N <= 7 at B = 8; the greedy path far less),
 * and PSI_ERR_CUDA if the scratch address cannot be obtained.
 */
#define PSI_NOALLOC_SCRATCH_BYTES 8388608u /* 8 MiB */
psi_status psi_verify_linear_noalloc(const void *ar_logits, int64_t ar_row_stride,
                                     const void *draft_logits,
                                     int64_t draft_row_stride, psi_dtype dtype,
                                     const int32_t *draft_ids, int32_t N, int32_t B,
                                     int32_t V, float temperature, float top_p,
                                     uint64_t seed, const uint64_t *seq_ids,
                                     uint64_t step, int32_t *out_tokens,
                                     int32_t *out_n_emitted, float *out_p_draft,
                                     float *out_q_draft, uint32_t *dev_status,
                                     psi_stream_t stream);

/* Workspace needed by psi_verify_tree_greedy (bytes; 0 on invalid sizes).
 * The walk keeps its state in shared memory: 256 bytes for any valid sizes. */
size_t psi_verify_tree_greedy_workspace_bytes(int32_t N, int32_t M, int32_t V,
                                              psi_dtype dtype);

/*
 * psi_verify_tree_greedy - greedy (T = 0) verify of a draft tree per sequence.
 *
 * [P3] "Linear 與 Tree sampler": several high-probability candidates per
 * position pruned to a finite prefix tree and verified in one pass.
 *
 * ar_logits    [N][M+1] rows (row 0 = root, row k+1 = node k).
 * node_tokens  int32 [N][M]; parents int32 [N][M] (-1 = child of the root;
 *              otherwise 0 <= parent < own index).
 * Node k is matched iff node_tokens[k] == argmax(row of its parent) and its
 * parent is matched (or is the root).  The deepest matched node (lowest
 * index among equals) ends the accepted path; the bonus token is the
 * argmax of that node's own row (root row when nothing matched).
 * out_path_nodes int32 [N][M]: node indices root-side first, then -1.
 * out_path_len   int32 [N]: number of accepted nodes (0..M).
 * out_tokens     int32 [N][M+1]: accepted tokens, then the bonus, then -1.
 * Rows read: the root's and each matched node's only (level by level, one
 * cluster of CTAs per tree); the NONFINITE status bit covers those rows.
 * Invalid parents and token ids are flagged for every node.
 * Limits: 1 <= N, 1 <= M <= PSI_MAX_TREE_NODES, 1 <= V <= PSI_MAX_V.
 */
psi_status psi_verify_tree_greedy(const void *ar_logits, int64_t ar_row_stride,
                                  psi_dtype dtype, const int32_t *node_tokens,
                                  const int32_t *parents, int32_t N, int32_t M,
                                  int32_t V, int32_t *out_path_nodes,
                                  int32_t *out_path_len, int32_t *out_tokens,
                                  uint32_t *dev_status, void *workspace,
                                  size_t workspace_bytes, psi_stream_t stream);

/* Workspace needed by psi_verify_tree_sampled (bytes, a multiple of 256; 0 on
 * invalid sizes).  The workspace needs no initialisation. */
size_t psi_verify_tree_sampled_workspace_bytes(int32_t N, int32_t M, int32_t V,
                                               psi_dtype dtype, float temperature,
                                               float top_p);

/*
 * psi_verify_tree_sampled - sampled (T > 0) verify of a draft tree per
 * sequence.
 *
 * [P3] "Linear 與 Tree sampler" (a prefix tree of candidates verified in one
 * pass) with the rejection rule and residual draw of [P3] "完整走一次四個
 * Token"; the pages give no sampled tree rule, and the one taken is
 * recursive rejection over each reached node's children (SpecInfer's
 * multi-candidate speculative sampling, Miao et al., ASPLOS 2024), every
 * child being a point-mass proposal:
 *   At a node whose AR row gives the target P (softmax at temperature T,
 *   cut to its top-p set as in psi_verify_linear), the valid children are
 *   tried in ascending index.  Child k with token x is accepted iff
 *   u_k * R < w(x), where w is what remains of P after the node's rejected
 *   tokens lost their mass (a repeated token has none left), R = sum(w) and
 *   u_k = U(seed, seq, step, k + 1, ACCEPT).  An accepted child becomes the
 *   next node.  When no child is accepted (or the node is a leaf) the step
 *   ends with the inverse-CDF draw, in vocabulary order, from w (from P if
 *   nothing remains) at u' = U(seed, seq, step, j, RESID), j being that
 *   node's row (0 = root).  Every emitted token then has the law of its
 *   node's P (lossless).
 * T == 0 is the greedy tree (psi_verify_tree_greedy; top_p ignored).
 * Arguments, layouts, validity rules and outputs as psi_verify_tree_greedy,
 * plus temperature, top_p (0 < top_p <= 1), seed, seq_ids (uint64 [N] or
 * NULL = n) and step as in psi_verify_linear.  out_tokens holds the accepted
 * tokens, then the drawn one, then -1.
 * Limits: as psi_verify_tree_greedy; T >= 0 and finite.
 */
psi_status psi_verify_tree_sampled(const void *ar_logits, int64_t ar_row_stride,
                                   psi_dtype dtype, const int32_t *node_tokens,
                                   const int32_t *parents, int32_t N, int32_t M,
                                   int32_t V, float temperature, float top_p,
                                   uint64_t seed, const uint64_t *seq_ids,
                                   uint64_t step, int32_t *out_path_nodes,
                                   int32_t *out_path_len, int32_t *out_tokens,
                                   uint32_t *dev_status, void *workspace,
                                   size_t workspace_bytes, psi_stream_t stream);

/*
 * psi_rng_uniforms - the uniforms the verify step draws, for inspection and
 * replay: out[s][r] = U(seed, seq_ids ? seq_ids[s] : s, step, r, purpose),
 * a float in [0, 1 - 2^-24] with 24 significant bits.
 * U is the top 24 bits of h = f(f(f(f(f(seed) ^ seq) ^ step) ^ row) ^
 * purpose), f being the SplitMix64 output function (Steele, Lea & Flood,
 * OOPSLA 2014).  out: float [n_seq][n_rows] device memory.
 */
psi_status psi_rng_uniforms(uint64_t seed, const uint64_t *seq_ids,
                            int32_t n_seq, uint64_t step, int32_t n_rows,
                            uint32_t purpose, float *out, psi_stream_t stream);

/*
 * psi_profile_main_kernel - instrumentation for roofline measurements (no
 * counterpart on the pages).  After this call, every verify call made from
 * the same host thread records `before` on its stream immediately before
 * launching its main kernel (the per-row kernel that reads the logits) and
 * `after` immediately after it, so that cudaEventElapsedTime(before, after)
 * is that kernel's duration.  The events are caller-created cudaEvent_t
 * handles, owned by the caller; psi_profile_main_kernel(NULL, NULL) stops
 * recording.  Returns PSI_ERR_INVALID_ARG if exactly one event is NULL.
 */
struct CUevent_st;
typedef struct CUevent_st *psi_event_t; /* same type as cudaEvent_t */
psi_status psi_profile_main_kernel(psi_event_t before, psi_event_t after);

/* Human-readable name of a status code (static string). */
const char *psi_status_string(psi_status status);

/* Detail of the last host-side error on this thread (static buffer). */
const char *psi_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* PSI_VERIFY_H */
