"""Mutation check of the oracle's pins (CPU only).

Each mutant is ``oracle/psi_oracle.c`` with ONE plausible mistake planted in a
copy: a dropped term, a flipped sign or comparison, a wrong row, index or
uniform, transposed operands, a filter applied to one side only.  Every copy
is compiled into a temporary library and the oracle's pin tests
(``tests/test_oracle_rng.py``, ``test_oracle_tree.py``,
``test_oracle_tree_sampled.py``, ``test_oracle_linear.py``) run against it in a
subprocess; each mutant must make
at least one pin fail.  The unmodified source, built the same way, must pass
them all, so a failure is the mutant's doing and not the harness's.

No mistake planted here lets a NaN reach the top-p sort, reads outside a
buffer, or loops: each mutant changes a result, never memory safety.
Mistakes that cannot change any result are not listed (subtracting a
different constant before ``exp``: it cancels in the normalisation).
"""
import concurrent.futures as cf
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "psi_oracle.c")
PINS = [os.path.join("tests", f) for f in
        ("test_oracle_rng.py", "test_oracle_tree.py", "test_oracle_tree_sampled.py",
         "test_oracle_linear.py")]  # the slow statistics last: most mutants fail sooner

# (name, text in psi_oracle.c, the same text with the mistake planted)
MUTANTS = [
    # ---- counter RNG (SplitMix64 chain over seed, seq, step, row, purpose)
    ("splitmix_increment", "0x9E3779B97F4A7C15ull", "0x9E3779B97F4A7C16ull"),
    ("splitmix_final_shift", "  return z ^ (z >> 31);", "  return z ^ (z >> 33);"),
    ("hash_drops_row", "  h = orc_splitmix64_mix(h ^ row);", "  h = orc_splitmix64_mix(h);"),
    ("hash_drops_step", "  h = orc_splitmix64_mix(h ^ step);", "  h = orc_splitmix64_mix(h);"),
    ("uniform_low_bits", "(double)(h >> 40) / 16777216.0",
     "(double)(h & 0xFFFFFFull) / 16777216.0"),
    ("verify_ignores_seq_ids",
     "    uint64_t seq = seq_ids ? seq_ids[n] : (uint64_t)n;\n    for (int32_t i = 0; i < B; ++i)",
     "    uint64_t seq = (uint64_t)n;\n    for (int32_t i = 0; i < B; ++i)"),
    ("verify_ignores_step",
     "      u_accept[i] = orc_uniform(seed, seq, step, (uint64_t)i,",
     "      u_accept[i] = orc_uniform(seed, seq, 0, (uint64_t)i,"),
    ("residual_uniform_uses_accept_purpose",
     "u_resid[i] = orc_uniform(seed, seq, step, (uint64_t)i, ORC_PURPOSE_RESID);",
     "u_resid[i] = orc_uniform(seed, seq, step, (uint64_t)i, ORC_PURPOSE_ACCEPT);"),
    # ---- logit decoding and addressing
    ("bf16_wrong_shift", "(uint32_t)((const uint16_t *)row)[v] << 16;",
     "(uint32_t)((const uint16_t *)row)[v] << 8;"),
    ("row_offset_in_elements_as_bytes",
     "(size_t)(row * stride) * elem_bytes(dtype);", "(size_t)(row * stride);"),
    # ---- temperature softmax
    ("softmax_ignores_temperature", "    double z = load_logit(row, dtype, v) / temperature;",
     "    double z = load_logit(row, dtype, v);"),
    ("softmax_not_normalised", "out_prob[v] /= total;", "out_prob[v] /= 1.0;"),
    # ---- top-p
    ("topp_sorted_ascending",
     "  if (x->prob > y->prob) return -1;\n  if (x->prob < y->prob) return 1;",
     "  if (x->prob > y->prob) return 1;\n  if (x->prob < y->prob) return -1;"),
    ("topp_cut_one_early", "        tau = sorted[k].prob;",
     "        tau = sorted[k > 0 ? k - 1 : 0].prob;"),
    ("topp_reach_is_strict", "      if (running >= top_p) {", "      if (running > top_p) {"),
    ("topp_drops_threshold_ties", "(out_prob[v] >= tau) ? out_prob[v] / kept : 0.0;",
     "(out_prob[v] > tau) ? out_prob[v] / kept : 0.0;"),
    ("topp_not_renormalised", "(out_prob[v] >= tau) ? out_prob[v] / kept : 0.0;",
     "(out_prob[v] >= tau) ? out_prob[v] : 0.0;"),
    ("topp_not_applied_to_draft_at_acceptance",
     "                            V, temperature, top_k, top_p, q, &mq[i]);",
     "                            V, temperature, top_k, 1.0, q, &mq[i]);"),
    ("topp_not_applied_to_draft_in_residual",
     "    orc_row_probs(row_ptr(draft, dtype, draft_row_stride, L), dtype, V,\n"
     "                  temperature, top_k, top_p, q, NULL);",
     "    orc_row_probs(row_ptr(draft, dtype, draft_row_stride, L), dtype, V,\n"
     "                  temperature, top_k, 1.0, q, NULL);"),
    ("topp_not_applied_to_bonus",
     "    orc_row_probs(row_ptr(ar, dtype, ar_row_stride, B), dtype, V, temperature,\n"
     "                  top_k, top_p, w, NULL);",
     "    orc_row_probs(row_ptr(ar, dtype, ar_row_stride, B), dtype, V, temperature,\n"
     "                  top_k, 1.0, w, NULL);"),
    # ---- top-k (before top-p)
    ("topk_drops_kth_ties", "(out_prob[v] >= kth) ? out_prob[v] / kept : 0.0;",
     "(out_prob[v] > kth) ? out_prob[v] / kept : 0.0;"),
    ("topk_threshold_one_late", "    const double kth = sorted[top_k - 1].prob;",
     "    const double kth = sorted[top_k].prob;"),
    ("topk_not_renormalised", "(out_prob[v] >= kth) ? out_prob[v] / kept : 0.0;",
     "(out_prob[v] >= kth) ? out_prob[v] : 0.0;"),
    ("topk_one_treated_as_off", "  if (top_k > 0 && top_k < V) {", "  if (top_k > 1 && top_k < V) {"),
    ("topk_not_applied_to_draft_at_acceptance",
     "                            V, temperature, top_k, top_p, q, &mq[i]);",
     "                            V, temperature, 0, top_p, q, &mq[i]);"),
    ("topk_not_applied_to_bonus",
     "    orc_row_probs(row_ptr(ar, dtype, ar_row_stride, B), dtype, V, temperature,\n"
     "                  top_k, top_p, w, NULL);",
     "    orc_row_probs(row_ptr(ar, dtype, ar_row_stride, B), dtype, V, temperature,\n"
     "                  0, top_p, w, NULL);"),
    # ---- acceptance test u < p(x) / q(x)
    ("accept_non_strict", "int accept = u_accept[i] * qx[i] < px[i];",
     "int accept = u_accept[i] * qx[i] <= px[i];"),
    ("accept_ratio_inverted", "int accept = u_accept[i] * qx[i] < px[i];",
     "int accept = u_accept[i] * px[i] < qx[i];"),
    ("accept_uses_residual_uniform", "int accept = u_accept[i] * qx[i] < px[i];",
     "int accept = u_resid[i] * qx[i] < px[i];"),
    ("accept_keeps_going_after_rejection", "      L = i;\n      break;", "      L = i;"),
    ("invalid_id_gets_mass", "      px[i] = 0.0; /* an invalid id is rejected */",
     "      px[i] = 1.0; /* an invalid id is rejected */"),
    # ---- correction from max(0, p - q), bonus from the block-end row
    ("residual_sign_flipped", "      double r = p[v] - q[v];", "      double r = q[v] - p[v];"),
    ("residual_is_abs_difference", "      w[v] = r > 0.0 ? r : 0.0;",
     "      w[v] = r > 0.0 ? r : -r;"),
    ("correction_drawn_from_p", "      double r = p[v] - q[v];", "      double r = p[v];"),
    ("residual_reads_next_ar_row",
     "    orc_row_probs(row_ptr(ar, dtype, ar_row_stride, L), dtype, V, temperature,",
     "    orc_row_probs(row_ptr(ar, dtype, ar_row_stride, L + 1), dtype, V, temperature,"),
    ("bonus_reads_last_draft_position",
     "    orc_row_probs(row_ptr(ar, dtype, ar_row_stride, B), dtype, V, temperature,\n"
     "                  top_k, top_p, w, NULL);",
     "    orc_row_probs(row_ptr(ar, dtype, ar_row_stride, B - 1), dtype, V, temperature,\n"
     "                  top_k, top_p, w, NULL);"),
    ("correction_uses_first_row_uniform",
     "token = inverse_cdf(w, V, u_resid[L], &sample_margin);",
     "token = inverse_cdf(w, V, u_resid[0], &sample_margin);"),
    # ---- inverse CDF
    ("icdf_target_not_scaled", "  double target = u * total;", "  double target = u;"),
    ("icdf_non_strict_crossing", "    if (running > target) {", "    if (running >= target) {"),
    # ---- greedy
    ("argmax_last_of_ties", "    if (x > best_x) {", "    if (x >= best_x) {"),
    ("greedy_last_mismatch", "    if (L == B && x != am[i]) L = i;", "    if (x != am[i]) L = i;"),
    ("greedy_emits_bonus_row", "  out_tokens[L] = am[L];", "  out_tokens[L] = am[B];"),
    # ---- greedy tree
    ("tree_compares_own_row", "      int32_t parent_row = pk + 1;", "      int32_t parent_row = k + 1;"),
    # (matching under an unmatched parent is not planted: the walk back from
    # such a node would write outside the path buffer)
    ("tree_only_root_children_match", "      int parent_ok = (pk == -1) || matched[pk];",
     "      int parent_ok = (pk == -1);"),
    ("tree_depth_ties_to_last", "        if (depth[k] > best_depth) {",
     "        if (depth[k] >= best_depth) {"),
    ("tree_next_token_from_root", "    toks[best_depth] = am[best + 1];",
     "    toks[best_depth] = am[0];"),
    ("tree_self_parent_not_flagged", "      if (pk < -1 || pk >= k) {",
     "      if (pk < -1 || pk > k) {"),
    # ---- sampled tree: recursive rejection over each node's children
    ("stree_accept_not_renormalised", "      if (u * R < px) {", "      if (u < px) {"),
    ("stree_rejected_mass_kept", "      w[x] = 0.0; /* remove the rejected candidate's mass */",
     "      /* the rejected candidate's mass is kept */"),
    ("stree_accept_uses_parent_row_uniform", "      const double u = u_accept[k + 1];",
     "      const double u = u_accept[node + 1];"),
    ("stree_draw_ignores_removed_mass", "      token = inverse_cdf(w, V, u_resid[row], &m2);",
     "      token = inverse_cdf(P, V, u_resid[row], &m2);"),
    ("stree_draw_uses_root_uniform", "      token = inverse_cdf(w, V, u_resid[row], &m2);",
     "      token = inverse_cdf(w, V, u_resid[0], &m2);"),
    ("stree_children_in_reverse", "    for (int32_t k = node + 1; k < M; ++k) {\n      if (parents[k] != node",
     "    for (int32_t k = M - 1; k > node; --k) {\n      if (parents[k] != node"),
    ("stree_batch_accept_row_offset",
     "      u_accept[j] = orc_uniform(seed, seq, step, (uint64_t)j,",
     "      u_accept[j] = orc_uniform(seed, seq, step, (uint64_t)(j - 1),"),
    ("stree_batch_ignores_seq_ids",
     "    uint64_t seq = seq_ids ? seq_ids[n] : (uint64_t)n;\n    u_accept[0] = 0.0;",
     "    uint64_t seq = (uint64_t)n;\n    u_accept[0] = 0.0;"),
    ("stree_emits_node_index", "    out_tokens[depth] = node_tokens[next];",
     "    out_tokens[depth] = next;"),
    ("stree_bad_parent_not_flagged", "      status |= ORC_BAD_PARENT;\n      valid[k] = 0;",
     "      valid[k] = 0;"),
    # ---- near-tie margins (the GPU parity tests excuse token differences only
    # within them, so a margin that is too wide would hide a real mismatch)
    ("margin_skips_acceptance_ratio",
     "    if (qx[i] > 0.0) margin = dmin(margin, fabs(u_accept[i] - px[i] / qx[i]));",
     "    (void)0;"),
    ("margin_skips_the_draw", "  margin = dmin(margin, sample_margin);", "  (void)sample_margin;"),
    ("margin_skips_draft_top_p", "    margin = dmin(margin, dmin(mp[i], mq[i]));",
     "    margin = dmin(margin, mp[i]);"),
    ("margin_skips_bonus_top_p", "    margin = dmin(margin, mp[B]);", "    (void)mp;"),
    ("icdf_margin_one_side",
     "      *margin = dmin(fabs(u - before / total), fabs(u - running / total));",
     "      *margin = fabs(u - running / total);"),
    ("topp_margin_one_side",
     "      *out_topp_margin = dmin(fabs(above - top_p), fabs(kept - top_p));",
     "      *out_topp_margin = fabs(kept - top_p);"),
    ("stree_margin_skips_tests", "      if (R > 0.0) margin = dmin(margin, fabs(u - px / R));",
     "      (void)0;"),
    ("stree_margin_skips_top_p", "    margin = dmin(margin, mtop);", "    (void)mtop;"),
    # ---- malformed input flags
    ("posinf_not_flagged", "return isnan(x) || (isinf(x) && x > 0);", "return isnan(x);"),
    ("neginf_flagged", "return isnan(x) || (isinf(x) && x > 0);",
     "return isnan(x) || isinf(x);"),
]

WORKERS = max(1, min(8, os.cpu_count() or 1))


def _build(text, out_dir, name):
    c_path = os.path.join(out_dir, f"{name}.c")
    so_path = os.path.join(out_dir, f"lib{name}.so")
    with open(c_path, "w") as f:
        f.write(text)
    subprocess.check_call(
        ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
         "-I", os.path.join(ROOT, "oracle"), c_path, "-o", so_path, "-lm"])
    return so_path


def _run_pins(text, out_dir, name):
    """(pytest exit code, last lines of its output) for the pins on one copy."""
    lib = _build(text, out_dir, name)
    env = dict(os.environ, PSI_ORACLE_LIB=lib, OMP_NUM_THREADS="1",
               OPENBLAS_NUM_THREADS="1", MKL_NUM_THREADS="1")
    env.pop("PYTEST_ADDOPTS", None)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "not gpu", *PINS],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    tail = "\n".join((r.stdout + r.stderr).strip().splitlines()[-6:])
    return r.returncode, tail


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    out_dir = str(tmp_path_factory.mktemp("oracle_mutants"))
    with open(SRC) as f:
        text = f.read()
    jobs = {"control": text}
    for name, old, new in MUTANTS:
        assert text.count(old) == 1, f"{name}: the text to mutate is not unique in psi_oracle.c"
        jobs[name] = text.replace(old, new)
    with cf.ThreadPoolExecutor(max_workers=WORKERS) as ex:
        futs = {name: ex.submit(_run_pins, src, out_dir, name) for name, src in jobs.items()}
        return {name: f.result() for name, f in futs.items()}


def test_mutant_names_unique():
    names = [m[0] for m in MUTANTS]
    assert len(names) == len(set(names)) and "control" not in names


def test_control_passes_every_pin(outcomes):
    rc, tail = outcomes["control"]
    assert rc == 0, tail


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_pins_catch_mutant(outcomes, name):
    rc, tail = outcomes[name]
    # pytest exits 1 when a test failed; 0 means the mistake went unnoticed,
    # anything else (a crash, a collection error) is not a clean catch
    assert rc == 1, f"{name} not caught (pytest exit {rc}):\n{tail}"
