/*
 * psi_oracle.c - plain, slow, double-precision CPU oracle of the Psi-Spec
 * verify step.
 *
 * TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check and the CPU
 * baseline of the benchmark, never by the product library.  It shares no
 * code with the CUDA kernels.  Every step is written the direct way: one
 * row at a time, a full sort for top-p, a linear scan for the inverse CDF.
 *
 * Page citations are given as (page, section); the page titles are spelled
 * out in psi_oracle.h as [P1] and [P3].
 *
 * Readings of points the pages leave open (each listed in the design notes):
 *  - B counts the DRAFTED tokens; AR rows are B+1, the last one is the
 *    bonus row; 1..B+1 tokens are emitted ([P3] walkthrough: the first
 *    block token is the verifier's own sample, i.e. the previous step's
 *    correction or bonus).
 *  - Acceptance is the strict test u < p(x)/q(x), evaluated as u*q < p:
 *    q(x) = 0 < p(x) accepts, p(x) = q(x) = 0 rejects.
 *  - The correction is drawn from max(0, p_L - q_L) by inverse CDF in
 *    vocabulary order: the smallest v whose running sum exceeds u' * R.
 *    If rounding leaves no crossing, the last v with positive weight.  If
 *    R == 0 (reachable only when the drafted token had q(x) = 0), the
 *    correction is drawn from p_L itself.
 *  - Top-p keeps, after temperature, the smallest descending-probability
 *    set whose mass reaches top_p, together with every token tied with the
 *    last one admitted, then renormalises; applied to p and q alike.
 *  - Top-k (run card: "top-k／top-p") is taken after temperature and before
 *    top-p: every token whose probability is at least the k-th largest stays
 *    (ties with the k-th included), renormalised; top-p then cuts that
 *    distribution.  k = 0 or k >= V means off; applied to p and q alike.
 *  - Greedy ties resolve to the lowest vocabulary index.
 *  - Sampled tree (the pages give no rule): recursive rejection over each
 *    reached node's children in index order, each child its own point-mass
 *    proposal; node k's acceptance uses the uniform of row k+1, the final
 *    draw the uniform of the row it is drawn from.
 */
#include "psi_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

static double load_logit(const void *row, int dtype, int32_t v) {
  if (dtype == ORC_F32) return (double)((const float *)row)[v];
  uint32_t w = (uint32_t)((const uint16_t *)row)[v] << 16;
  float f;
  memcpy(&f, &w, sizeof f);
  return (double)f;
}

static size_t elem_bytes(int dtype) { return dtype == ORC_F32 ? 4u : 2u; }

static const void *row_ptr(const void *base, int dtype, int64_t stride,
                           int64_t row) {
  return (const char *)base + (size_t)(row * stride) * elem_bytes(dtype);
}

static int bad_value(double x) { return isnan(x) || (isinf(x) && x > 0); }

static double dmin(double a, double b) { return a < b ? a : b; }

/* ---- counter RNG ------------------------------------------------------ */

/* SplitMix64 output function (Steele, Lea & Flood, OOPSLA 2014): add the
 * golden-ratio increment, then two xor-shift-multiply rounds and a final
 * xor-shift. */
uint64_t orc_splitmix64_mix(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

uint64_t orc_counter_hash(uint64_t seed, uint64_t seq, uint64_t step,
                          uint64_t row, uint64_t purpose) {
  uint64_t h = orc_splitmix64_mix(seed);
  h = orc_splitmix64_mix(h ^ seq);
  h = orc_splitmix64_mix(h ^ step);
  h = orc_splitmix64_mix(h ^ row);
  h = orc_splitmix64_mix(h ^ purpose);
  return h;
}

double orc_uniform(uint64_t seed, uint64_t seq, uint64_t step, uint64_t row,
                   uint64_t purpose) {
  uint64_t h = orc_counter_hash(seed, seq, step, row, purpose);
  return (double)(h >> 40) / 16777216.0; /* top 24 bits / 2^24 */
}

/* ---- one row: temperature softmax and top-p --------------------------- */

typedef struct {
  double prob;
  int32_t id;
} prob_id;

/* Descending probability; equal probabilities by ascending id. */
static int by_prob_desc(const void *a, const void *b) {
  const prob_id *x = (const prob_id *)a;
  const prob_id *y = (const prob_id *)b;
  if (x->prob > y->prob) return -1;
  if (x->prob < y->prob) return 1;
  return (x->id > y->id) - (x->id < y->id);
}

uint32_t orc_row_probs(const void *row, int dtype, int32_t V,
                       double temperature, int32_t top_k, double top_p,
                       double *out_prob, double *out_topp_margin) {
  uint32_t status = 0;
  if (out_topp_margin) *out_topp_margin = INFINITY;

  /* softmax(x / T): [P3] run card (temperature); [P1]/[P3] the target
   * distribution is the AR model's. */
  double m = -INFINITY;
  for (int32_t v = 0; v < V; ++v) {
    double x = load_logit(row, dtype, v);
    if (bad_value(x)) status |= ORC_NONFINITE;
    double z = x / temperature;
    if (z > m) m = z;
  }
  if (m == -INFINITY) {
    /* no finite logit: no distribution; all probabilities zero */
    for (int32_t v = 0; v < V; ++v) out_prob[v] = 0.0;
    return status | ORC_NONFINITE;
  }
  double total = 0.0;
  for (int32_t v = 0; v < V; ++v) {
    double z = load_logit(row, dtype, v) / temperature;
    double e = (z == -INFINITY) ? 0.0 : exp(z - m);
    out_prob[v] = e;
    total += e;
  }
  for (int32_t v = 0; v < V; ++v) out_prob[v] /= total;

  if (top_k > 0 && top_k < V) {
    /* Top-k: the k-th largest probability is the threshold; ties with it
     * stay.  Then renormalise. */
    prob_id *sorted = (prob_id *)malloc((size_t)V * sizeof(prob_id));
    for (int32_t v = 0; v < V; ++v) {
      sorted[v].prob = out_prob[v];
      sorted[v].id = v;
    }
    qsort(sorted, (size_t)V, sizeof(prob_id), by_prob_desc);
    const double kth = sorted[top_k - 1].prob;
    free(sorted);
    double kept = 0.0;
    for (int32_t v = 0; v < V; ++v)
      if (out_prob[v] >= kth) kept += out_prob[v];
    for (int32_t v = 0; v < V; ++v)
      out_prob[v] = (out_prob[v] >= kth) ? out_prob[v] / kept : 0.0;
  }

  if (top_p < 1.0) {
    /* Nucleus: sort, find the first prefix whose mass reaches top_p. */
    prob_id *sorted = (prob_id *)malloc((size_t)V * sizeof(prob_id));
    for (int32_t v = 0; v < V; ++v) {
      sorted[v].prob = out_prob[v];
      sorted[v].id = v;
    }
    qsort(sorted, (size_t)V, sizeof(prob_id), by_prob_desc);
    double running = 0.0;
    double tau = sorted[V - 1].prob;
    for (int32_t k = 0; k < V; ++k) {
      running += sorted[k].prob;
      if (running >= top_p) {
        tau = sorted[k].prob;
        break;
      }
    }
    free(sorted);
    /* Keep every token at or above tau (ties at tau included). */
    double above = 0.0, kept = 0.0;
    for (int32_t v = 0; v < V; ++v) {
      if (out_prob[v] > tau) above += out_prob[v];
      if (out_prob[v] >= tau) kept += out_prob[v];
    }
    if (out_topp_margin)
      *out_topp_margin = dmin(fabs(above - top_p), fabs(kept - top_p));
    for (int32_t v = 0; v < V; ++v)
      out_prob[v] = (out_prob[v] >= tau) ? out_prob[v] / kept : 0.0;
  }
  return status;
}

int32_t orc_row_argmax(const void *row, int dtype, int32_t V,
                       uint32_t *status) {
  int32_t best = 0;
  double best_x = load_logit(row, dtype, 0);
  for (int32_t v = 0; v < V; ++v) {
    double x = load_logit(row, dtype, v);
    if (bad_value(x) && status) *status |= ORC_NONFINITE;
    if (x > best_x) {
      best_x = x;
      best = v;
    }
  }
  return best;
}

/* Inverse CDF over nonnegative weights in vocabulary order.  Returns the
 * smallest v whose running sum exceeds u * W; without a crossing, the last
 * v with positive weight; without any positive weight, 0.  *margin gets the
 * distance of u from the two crossing boundaries (as fractions of W). */
static int32_t inverse_cdf(const double *w, int32_t V, double u,
                           double *margin) {
  double total = 0.0;
  int32_t last_pos = -1;
  for (int32_t v = 0; v < V; ++v) {
    total += w[v];
    if (w[v] > 0.0) last_pos = v;
  }
  *margin = INFINITY;
  if (last_pos < 0) return 0;
  double target = u * total;
  double running = 0.0;
  for (int32_t v = 0; v < V; ++v) {
    double before = running;
    running += w[v];
    if (running > target) {
      *margin = dmin(fabs(u - before / total), fabs(u - running / total));
      return v;
    }
  }
  return last_pos;
}

/* ---- one sequence ------------------------------------------------------ */

static uint32_t verify_greedy_one(const void *ar, int64_t ar_row_stride,
                                  int dtype, const int32_t *ids, int32_t B,
                                  int32_t V, int32_t *out_tokens,
                                  int32_t *out_n) {
  uint32_t status = 0;
  int32_t *am = (int32_t *)malloc((size_t)(B + 1) * sizeof(int32_t));
  for (int32_t i = 0; i <= B; ++i)
    am[i] = orc_row_argmax(row_ptr(ar, dtype, ar_row_stride, i), dtype, V,
                           &status);
  int32_t L = B;
  for (int32_t i = 0; i < B; ++i) {
    int32_t x = ids[i];
    if (x < 0 || x >= V) status |= ORC_BAD_TOKEN_ID;
    if (L == B && x != am[i]) L = i; /* first mismatch */
  }
  for (int32_t i = 0; i <= B; ++i) out_tokens[i] = -1;
  for (int32_t i = 0; i < L; ++i) out_tokens[i] = ids[i];
  out_tokens[L] = am[L];
  *out_n = L + 1;
  free(am);
  return status;
}

uint32_t orc_verify_one(const void *ar, int64_t ar_row_stride,
                        const void *draft, int64_t draft_row_stride,
                        int dtype, const int32_t *ids, int32_t B, int32_t V,
                        double temperature, int32_t top_k, double top_p,
                        const double *u_accept, const double *u_resid,
                        int32_t *out_tokens, int32_t *out_n, double *out_p,
                        double *out_q, double *out_margin) {
  if (out_margin) *out_margin = INFINITY;
  if (temperature == 0.0)
    return verify_greedy_one(ar, ar_row_stride, dtype, ids, B, V, out_tokens,
                             out_n);

  uint32_t status = 0;
  double *p = (double *)malloc((size_t)V * sizeof(double));
  double *q = (double *)malloc((size_t)V * sizeof(double));
  double *w = (double *)malloc((size_t)V * sizeof(double));
  double *px = (double *)malloc((size_t)B * sizeof(double));
  double *qx = (double *)malloc((size_t)B * sizeof(double));
  double *mp = (double *)malloc((size_t)(B + 1) * sizeof(double));
  double *mq = (double *)malloc((size_t)(B + 1) * sizeof(double));

  /* p_i(x_i) and q_i(x_i) for every drafted position ([P3] walkthrough,
   * step 3: the frozen AR scores the whole block in one pass). */
  for (int32_t i = 0; i < B; ++i) {
    status |= orc_row_probs(row_ptr(ar, dtype, ar_row_stride, i), dtype, V,
                            temperature, top_k, top_p, p, &mp[i]);
    status |= orc_row_probs(row_ptr(draft, dtype, draft_row_stride, i), dtype,
                            V, temperature, top_k, top_p, q, &mq[i]);
    int32_t x = ids[i];
    if (x >= 0 && x < V) {
      px[i] = p[x];
      qx[i] = q[x];
    } else {
      status |= ORC_BAD_TOKEN_ID;
      px[i] = 0.0; /* an invalid id is rejected */
      qx[i] = 0.0;
    }
    if (out_p) out_p[i] = px[i];
    if (out_q) out_q[i] = qx[i];
  }
  /* The bonus row is read too; its top-p margin matters only if used. */
  status |= orc_row_probs(row_ptr(ar, dtype, ar_row_stride, B), dtype, V,
                          temperature, top_k, top_p, p, &mp[B]);

  /* Longest accepted prefix: accept x_i while u_i < p_i(x_i)/q_i(x_i)
   * ([P1] "Psi-Spec이 한 스텝에서 하는 일"; [P3] walkthrough step 3). */
  double margin = INFINITY;
  int32_t L = B;
  for (int32_t i = 0; i < B; ++i) {
    margin = dmin(margin, dmin(mp[i], mq[i]));
    if (qx[i] > 0.0) margin = dmin(margin, fabs(u_accept[i] - px[i] / qx[i]));
    int accept = u_accept[i] * qx[i] < px[i];
    if (!accept) {
      L = i;
      break;
    }
  }

  /* Correction at the first rejection from the residual max(0, p - q)
   * ([P3] walkthrough step 4), or the bonus token from the block-end row
   * when every draft passed ([P3], paragraph after the walkthrough). */
  double sample_margin;
  int32_t token;
  if (L < B) {
    orc_row_probs(row_ptr(ar, dtype, ar_row_stride, L), dtype, V, temperature,
                  top_k, top_p, p, NULL);
    orc_row_probs(row_ptr(draft, dtype, draft_row_stride, L), dtype, V,
                  temperature, top_k, top_p, q, NULL);
    double residual_mass = 0.0;
    for (int32_t v = 0; v < V; ++v) {
      double r = p[v] - q[v];
      w[v] = r > 0.0 ? r : 0.0;
      residual_mass += w[v];
    }
    if (residual_mass <= 0.0) memcpy(w, p, (size_t)V * sizeof(double));
  } else {
    margin = dmin(margin, mp[B]);
    orc_row_probs(row_ptr(ar, dtype, ar_row_stride, B), dtype, V, temperature,
                  top_k, top_p, w, NULL);
  }
  token = inverse_cdf(w, V, u_resid[L], &sample_margin);
  margin = dmin(margin, sample_margin);

  for (int32_t i = 0; i <= B; ++i) out_tokens[i] = -1;
  for (int32_t i = 0; i < L; ++i) out_tokens[i] = ids[i];
  out_tokens[L] = token;
  *out_n = L + 1;
  if (out_margin) *out_margin = margin;

  free(p);
  free(q);
  free(w);
  free(px);
  free(qx);
  free(mp);
  free(mq);
  return status;
}

uint32_t orc_verify_linear(const void *ar, int64_t ar_row_stride,
                           const void *draft, int64_t draft_row_stride,
                           int dtype, const int32_t *ids, int32_t N, int32_t B,
                           int32_t V, double temperature, int32_t top_k,
                           double top_p, uint64_t seed, const uint64_t *seq_ids,
                           uint64_t step, int32_t *out_tokens,
                           int32_t *out_n_emitted, double *out_p_draft,
                           double *out_q_draft, double *out_margin) {
  uint32_t status = 0;
  double *u_accept = (double *)malloc((size_t)B * sizeof(double));
  double *u_resid = (double *)malloc((size_t)(B + 1) * sizeof(double));
  for (int32_t n = 0; n < N; ++n) {
    uint64_t seq = seq_ids ? seq_ids[n] : (uint64_t)n;
    for (int32_t i = 0; i < B; ++i)
      u_accept[i] = orc_uniform(seed, seq, step, (uint64_t)i,
                                ORC_PURPOSE_ACCEPT);
    for (int32_t i = 0; i <= B; ++i)
      u_resid[i] = orc_uniform(seed, seq, step, (uint64_t)i, ORC_PURPOSE_RESID);
    const void *ar_n = row_ptr(ar, dtype, ar_row_stride, (int64_t)n * (B + 1));
    const void *dr_n = draft ? row_ptr(draft, dtype, draft_row_stride,
                                       (int64_t)n * B)
                             : NULL;
    status |= orc_verify_one(
        ar_n, ar_row_stride, dr_n, draft_row_stride, dtype, ids + (size_t)n * B,
        B, V, temperature, top_k, top_p, u_accept, u_resid,
        out_tokens + (size_t)n * (B + 1), out_n_emitted + n,
        out_p_draft ? out_p_draft + (size_t)n * B : NULL,
        out_q_draft ? out_q_draft + (size_t)n * B : NULL,
        out_margin ? out_margin + n : NULL);
  }
  free(u_accept);
  free(u_resid);
  return status;
}

/* ---- greedy tree ------------------------------------------------------- */

/* [P3] "Linear 與 Tree sampler": several candidates per position, pruned to
 * a finite prefix tree and verified in one pass.  Greedy rule: a node is
 * matched when its token equals the AR argmax of its parent's row and its
 * parent is matched; the deepest matched node (lowest index on ties) ends
 * the accepted path, followed by the argmax of that node's own row. */
uint32_t orc_verify_tree_greedy(const void *ar, int64_t ar_row_stride,
                                int dtype, const int32_t *node_tokens,
                                const int32_t *parents, int32_t N, int32_t M,
                                int32_t V, int32_t *out_path_nodes,
                                int32_t *out_path_len, int32_t *out_tokens) {
  uint32_t status = 0;
  int32_t *am = (int32_t *)malloc((size_t)(M + 1) * sizeof(int32_t));
  int32_t *matched = (int32_t *)malloc((size_t)(M > 0 ? M : 1) * sizeof(int32_t));
  int32_t *depth = (int32_t *)malloc((size_t)(M > 0 ? M : 1) * sizeof(int32_t));
  for (int32_t n = 0; n < N; ++n) {
    const void *ar_n = row_ptr(ar, dtype, ar_row_stride, (int64_t)n * (M + 1));
    const int32_t *tok = node_tokens + (size_t)n * M;
    const int32_t *par = parents + (size_t)n * M;
    for (int32_t j = 0; j <= M; ++j)
      am[j] = orc_row_argmax(row_ptr(ar_n, dtype, ar_row_stride, j), dtype, V,
                             &status);
    int32_t best = -1, best_depth = 0;
    for (int32_t k = 0; k < M; ++k) {
      matched[k] = 0;
      depth[k] = 0;
      int32_t pk = par[k];
      if (pk < -1 || pk >= k) {
        status |= ORC_BAD_PARENT;
        continue;
      }
      if (tok[k] < 0 || tok[k] >= V) {
        status |= ORC_BAD_TOKEN_ID;
        continue;
      }
      int parent_ok = (pk == -1) || matched[pk];
      int32_t parent_row = pk + 1; /* root row is row 0 */
      if (parent_ok && tok[k] == am[parent_row]) {
        matched[k] = 1;
        depth[k] = (pk == -1) ? 1 : depth[pk] + 1;
        if (depth[k] > best_depth) {
          best_depth = depth[k];
          best = k;
        }
      }
    }
    int32_t *path = out_path_nodes + (size_t)n * M;
    int32_t *toks = out_tokens + (size_t)n * (M + 1);
    for (int32_t k = 0; k < M; ++k) path[k] = -1;
    for (int32_t k = 0; k <= M; ++k) toks[k] = -1;
    /* walk back from the deepest matched node to the root */
    int32_t d = best_depth;
    for (int32_t k = best; k >= 0; k = par[k]) {
      --d;
      path[d] = k;
      toks[d] = tok[k];
    }
    out_path_len[n] = best_depth;
    toks[best_depth] = am[best + 1];
  }
  free(am);
  free(matched);
  free(depth);
  return status;
}

/* ---- sampled tree ------------------------------------------------------ */

/* [P3] "Linear 與 Tree sampler" keeps several candidates per position in a
 * finite prefix tree and verifies the tree in one pass, but gives no rule
 * for sampled decoding.  The rule taken here is recursive rejection over
 * each node's candidate list, the multi-candidate scheme of Miao et al.
 * ("SpecInfer", ASPLOS 2024, multi-step speculative sampling), with every
 * candidate taken as its own point-mass proposal so the result stays
 * lossless for candidates that were chosen (top-k) rather than sampled:
 * at a node with target P, candidate x is accepted with probability
 * P'(x) = P(x) / R (R = mass not yet removed); on rejection x's mass is
 * removed, which is max(0, P' - delta_x) renormalised.  Each round is one
 * speculative-sampling step, so the emitted token at every node has law P.
 *
 * Node validity follows the greedy tree: a bad parent or token makes the
 * node unusable (flagged, never accepted, its subtree unreachable). */
static uint32_t tree_validate(const int32_t *tok, const int32_t *par,
                              int32_t M, int32_t V, unsigned char *valid) {
  uint32_t status = 0;
  for (int32_t k = 0; k < M; ++k) {
    valid[k] = 1;
    if (par[k] < -1 || par[k] >= k) {
      status |= ORC_BAD_PARENT;
      valid[k] = 0;
    } else if (tok[k] < 0 || tok[k] >= V) {
      status |= ORC_BAD_TOKEN_ID;
      valid[k] = 0;
    }
  }
  return status;
}

uint32_t orc_verify_tree_sampled_one(const void *ar, int64_t ar_row_stride,
                                     int dtype, const int32_t *node_tokens,
                                     const int32_t *parents, int32_t M,
                                     int32_t V, double temperature,
                                     int32_t top_k, double top_p,
                                     const double *u_accept,
                                     const double *u_resid,
                                     int32_t *out_path_nodes,
                                     int32_t *out_path_len, int32_t *out_tokens,
                                     double *out_margin) {
  if (out_margin) *out_margin = INFINITY;
  if (temperature == 0.0)
    return orc_verify_tree_greedy(ar, ar_row_stride, dtype, node_tokens,
                                  parents, 1, M, V, out_path_nodes,
                                  out_path_len, out_tokens);

  unsigned char *valid = (unsigned char *)malloc((size_t)(M > 0 ? M : 1));
  double *P = (double *)malloc((size_t)V * sizeof(double));
  double *w = (double *)malloc((size_t)V * sizeof(double));
  uint32_t status = tree_validate(node_tokens, parents, M, V, valid);

  for (int32_t k = 0; k < M; ++k) out_path_nodes[k] = -1;
  for (int32_t k = 0; k <= M; ++k) out_tokens[k] = -1;

  double margin = INFINITY;
  int32_t node = -1; /* -1 = root */
  int32_t depth = 0;
  int32_t token;
  for (;;) {
    const int32_t row = node + 1;
    double mtop;
    status |= orc_row_probs(row_ptr(ar, dtype, ar_row_stride, row), dtype, V,
                            temperature, top_k, top_p, P, &mtop);
    margin = dmin(margin, mtop);
    memcpy(w, P, (size_t)V * sizeof(double)); /* what remains of P */
    int32_t next = -1;
    for (int32_t k = node + 1; k < M; ++k) {
      if (parents[k] != node || !valid[k]) continue;
      const int32_t x = node_tokens[k];
      double R = 0.0;
      for (int32_t v = 0; v < V; ++v) R += w[v];
      const double px = w[x]; /* 0 once x was rejected at this node */
      const double u = u_accept[k + 1];
      if (R > 0.0) margin = dmin(margin, fabs(u - px / R));
      if (u * R < px) {
        next = k;
        break;
      }
      w[x] = 0.0; /* remove the rejected candidate's mass */
    }
    if (next < 0) {
      double total = 0.0;
      for (int32_t v = 0; v < V; ++v) total += w[v];
      if (total <= 0.0) memcpy(w, P, (size_t)V * sizeof(double));
      double m2;
      token = inverse_cdf(w, V, u_resid[row], &m2);
      margin = dmin(margin, m2);
      break;
    }
    out_path_nodes[depth] = next;
    out_tokens[depth] = node_tokens[next];
    ++depth;
    node = next;
  }
  out_tokens[depth] = token;
  *out_path_len = depth;
  if (out_margin) *out_margin = margin;
  free(valid);
  free(P);
  free(w);
  return status;
}

uint32_t orc_verify_tree_sampled(const void *ar, int64_t ar_row_stride,
                                 int dtype, const int32_t *node_tokens,
                                 const int32_t *parents, int32_t N, int32_t M,
                                 int32_t V, double temperature, int32_t top_k,
                                 double top_p, uint64_t seed,
                                 const uint64_t *seq_ids,
                                 uint64_t step, int32_t *out_path_nodes,
                                 int32_t *out_path_len, int32_t *out_tokens,
                                 double *out_margin) {
  uint32_t status = 0;
  double *u_accept = (double *)malloc((size_t)(M + 1) * sizeof(double));
  double *u_resid = (double *)malloc((size_t)(M + 1) * sizeof(double));
  for (int32_t n = 0; n < N; ++n) {
    uint64_t seq = seq_ids ? seq_ids[n] : (uint64_t)n;
    u_accept[0] = 0.0; /* the root row has no acceptance test */
    for (int32_t j = 1; j <= M; ++j)
      u_accept[j] = orc_uniform(seed, seq, step, (uint64_t)j,
                                ORC_PURPOSE_ACCEPT);
    for (int32_t j = 0; j <= M; ++j)
      u_resid[j] = orc_uniform(seed, seq, step, (uint64_t)j, ORC_PURPOSE_RESID);
    status |= orc_verify_tree_sampled_one(
        row_ptr(ar, dtype, ar_row_stride, (int64_t)n * (M + 1)), ar_row_stride,
        dtype, node_tokens + (size_t)n * M, parents + (size_t)n * M, M, V,
        temperature, top_k, top_p, u_accept, u_resid,
        out_path_nodes + (size_t)n * M, out_path_len + n,
        out_tokens + (size_t)n * (M + 1), out_margin ? out_margin + n : NULL);
  }
  free(u_accept);
  free(u_resid);
  return status;
}
