/*
 * psi_oracle.h - plain double-precision CPU oracle of the Psi-Spec verify step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, calls or
 * includes this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant with the
 * CUDA path.
 *
 * Sources (page title, section):
 *   [P1] "Uno / Psi-Spec - 같은 모델 안에서 초안 뽑고 AR로 도장 찍기"
 *        (lanes-ecd.pages.dev), sections "어디서 왔나" (the Leviathan et al.
 *        2023 draft -> verify -> correct lineage) and "Psi-Spec이 한 스텝에서
 *        하는 일" (longest accepted prefix, lossless).
 *   [P3] "Uno Psi-Spec 是什麼？Diffusion-Augmented LLM 如何保留 AR 分布、
 *        一次驗證多個 Token" (alphalab.site), sections
 *        "Uno Psi-Spec 怎麼運作？完整走一次四個 Token" (draft, verify with the
 *        rejection rule, longest accepted prefix, residual correction at the
 *        first rejection, bonus token from the block-end logits, TPF bound),
 *        "為什麼 lossless 不等於答案完全一樣？" (distribution preservation),
 *        "Linear 與 Tree sampler" (tree verify), and
 *        "想跑 Uno：先確認官方程式需要的環境" (temperature and top-p on the
 *        run card).
 *
 * All buffers are HOST memory owned by the caller.  Layouts match the CUDA
 * library's: AR logits [N][B+1][V] (row stride in elements), draft logits
 * [N][B][V], ids [N][B], outputs [N][B+1] padded with -1.
 */
#ifndef PSI_ORACLE_H
#define PSI_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Logit element encodings understood by the oracle. */
#define ORC_F32 0  /* IEEE binary32 */
#define ORC_BF16 1 /* raw bfloat16 bit patterns (uint16) */

/* Status bits (same meaning as the device status word of the CUDA library,
 * defined independently here). */
#define ORC_BAD_TOKEN_ID 1u
#define ORC_BAD_PARENT 2u
#define ORC_NONFINITE 4u

/* RNG purposes. */
#define ORC_PURPOSE_ACCEPT 0u
#define ORC_PURPOSE_RESID 1u

/* One SplitMix64 output step applied to state x (Steele, Lea & Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014). */
uint64_t orc_splitmix64_mix(uint64_t x);
/* Chained counter hash of (seed, seq, step, row, purpose). */
uint64_t orc_counter_hash(uint64_t seed, uint64_t seq, uint64_t step,
                          uint64_t row, uint64_t purpose);
/* 24-bit uniform in [0, 1 - 2^-24] from the counter hash. */
double orc_uniform(uint64_t seed, uint64_t seq, uint64_t step, uint64_t row,
                   uint64_t purpose);

/* Temperature softmax of one logit row, in double, then optional top-k
 * (top_k > 0: keep every token at or above the k-th largest probability,
 * renormalise) and optional top-p (top_p < 1: the smallest descending set
 * of mass >= top_p with the ties of its last token, renormalise).
 * out_prob[V].  Returns status bits.  out_topp_margin (may be NULL) receives
 * the distance of the cumulative mass on either side of the top-p crossing
 * from top_p (+inf when top-p is off). */
uint32_t orc_row_probs(const void *row, int dtype, int32_t V,
                       double temperature, int32_t top_k, double top_p,
                       double *out_prob, double *out_topp_margin);

/* Verify one sequence with explicitly supplied uniforms.
 * u_accept[B]: acceptance uniforms; u_resid[B+1]: residual/bonus uniforms
 * (only u_resid[L] is used).  temperature == 0 selects the greedy rule.
 * out_tokens[B+1], out_n[1], out_p[B], out_q[B] (NULL allowed),
 * out_margin[1] (NULL allowed): smallest distance of any decision from
 * its threshold (acceptance ratio, inverse-CDF crossing, top-p crossing).
 * Returns status bits. */
uint32_t orc_verify_one(const void *ar, int64_t ar_row_stride,
                        const void *draft, int64_t draft_row_stride,
                        int dtype, const int32_t *ids, int32_t B, int32_t V,
                        double temperature, int32_t top_k, double top_p,
                        const double *u_accept, const double *u_resid,
                        int32_t *out_tokens, int32_t *out_n, double *out_p,
                        double *out_q, double *out_margin);

/* Batch verify with the counter RNG: sequence n uses
 * seq = seq_ids ? seq_ids[n] : n.  Returns OR of status bits. */
uint32_t orc_verify_linear(const void *ar, int64_t ar_row_stride,
                           const void *draft, int64_t draft_row_stride,
                           int dtype, const int32_t *ids, int32_t N, int32_t B,
                           int32_t V, double temperature, int32_t top_k,
                           double top_p, uint64_t seed, const uint64_t *seq_ids,
                           uint64_t step, int32_t *out_tokens,
                           int32_t *out_n_emitted, double *out_p_draft,
                           double *out_q_draft, double *out_margin);

/* Greedy tree verify.  AR logits [N][M+1][V] (row 0 = root, row k+1 =
 * node k), node_tokens [N][M], parents [N][M] (-1 = root).
 * Outputs: path_nodes [N][M] (-1 padded), path_len [N],
 * tokens [N][M+1] (-1 padded).  Returns OR of status bits. */
uint32_t orc_verify_tree_greedy(const void *ar, int64_t ar_row_stride,
                                int dtype, const int32_t *node_tokens,
                                const int32_t *parents, int32_t N, int32_t M,
                                int32_t V, int32_t *out_path_nodes,
                                int32_t *out_path_len, int32_t *out_tokens);

/* Sampled tree verify of one sequence with explicitly supplied uniforms.
 * Tree layout as orc_verify_tree_greedy for one sequence.  At each reached
 * node the children (ascending index) are tried in turn: child k, token x,
 * is accepted iff u_accept[k+1] * R < P(x), where P is the node row's
 * tempered (top-p cut) distribution and R the mass of P not yet removed;
 * a rejected child's token is removed from P.  An accepted child becomes the
 * next node; when no child is accepted (or the node is a leaf) the last
 * token is the inverse-CDF draw from what remains of P with u_resid[row].
 * u_accept[M+1] (entry 0 unused), u_resid[M+1].  temperature == 0 selects the
 * greedy tree rule.  out_margin as in orc_verify_one.  Returns status bits. */
uint32_t orc_verify_tree_sampled_one(const void *ar, int64_t ar_row_stride,
                                     int dtype, const int32_t *node_tokens,
                                     const int32_t *parents, int32_t M,
                                     int32_t V, double temperature,
                                     int32_t top_k, double top_p,
                                     const double *u_accept,
                                     const double *u_resid,
                                     int32_t *out_path_nodes,
                                     int32_t *out_path_len, int32_t *out_tokens,
                                     double *out_margin);

/* Batch sampled tree verify with the counter RNG: node k's acceptance
 * uniform is U(seed, seq, step, k+1, ACCEPT), the draw at row j uses
 * U(seed, seq, step, j, RESID); seq = seq_ids ? seq_ids[n] : n.
 * out_margin [N] may be NULL.  Returns OR of status bits. */
uint32_t orc_verify_tree_sampled(const void *ar, int64_t ar_row_stride,
                                 int dtype, const int32_t *node_tokens,
                                 const int32_t *parents, int32_t N, int32_t M,
                                 int32_t V, double temperature, int32_t top_k,
                                 double top_p, uint64_t seed,
                                 const uint64_t *seq_ids,
                                 uint64_t step, int32_t *out_path_nodes,
                                 int32_t *out_path_len, int32_t *out_tokens,
                                 double *out_margin);

/* Index of the largest logit in a row (lowest index among equals). */
int32_t orc_row_argmax(const void *row, int dtype, int32_t V,
                       uint32_t *status);

#ifdef __cplusplus
}
#endif
#endif
