"""Pins for the oracle's linear verify (CPU only).

What fixes the oracle here, other than itself:
  * hand-worked fixtures of the pages' four-token walkthrough
    (tests/golden/walkthrough_b4.json);
  * the lossless invariant, integrated EXACTLY: the oracle's decisions are
    monotone step functions of each uniform, so bisection on the oracle's own
    outputs gives the measure of every outcome; the emitted-token law must
    equal the target softmax (scipy) to 1e-12;
  * the pages' 70/30 example;
  * chi-square over 10^6 RNG-driven draws, the closed-form acceptance rate
    sum_v min(p, q) and the mean accepted length;
  * the emitted-count bounds 1..B+1;
  * top-p cases worked by hand, and its two limits (top_p = 1 is the plain
    softmax, a tiny top_p keeps only the argmax tie group);
  * the greedy rule on hand cases and as the T -> 0 limit of the sampled rule.
"""
import json
import math
import os

import numpy as np
import pytest
from scipy import stats
from scipy.special import softmax

import oracle
import psi_inputs

HERE = os.path.dirname(__file__)
NEXT1 = float(np.nextafter(1.0, 0.0))


def _row(vals):
    return np.array([-np.inf if v == "-inf" else float(v) for v in vals], dtype=np.float32)


# ---- the pages' walkthrough -------------------------------------------------

def test_walkthrough_fixtures():
    with open(os.path.join(HERE, "golden", "walkthrough_b4.json")) as f:
        fx = json.load(f)
    for case in fx["cases"]:
        T = case.get("temperature", fx["temperature"])
        ar = np.stack([_row(r) for r in case["ar"]])
        draft = None if case["draft"] is None else np.stack([_row(r) for r in case["draft"]])
        r = oracle.verify_one(ar, draft, case["ids"], T, 1.0, case["u_accept"], case["u_resid"])
        exp = case["expected"]
        assert r["tokens"].tolist() == exp["tokens"], case["name"]
        assert r["n_emitted"] == exp["n_emitted"], case["name"]
        if "p_draft" in exp:
            np.testing.assert_allclose(r["p_draft"], exp["p_draft"], atol=1e-15)
            np.testing.assert_allclose(r["q_draft"], exp["q_draft"], atol=1e-15)
        assert r["status"] == 0


# ---- exact integration of the oracle's decisions ------------------------------

def _sup_true(pred, iters=60):
    """sup{u in [0,1): pred(u)} for a predicate true on [0, t), false on [t, 1)."""
    if not pred(0.0):
        return 0.0
    if pred(NEXT1):
        return 1.0
    lo, hi = 0.0, 1.0
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if pred(mid):
            lo = mid
        else:
            hi = mid
    return hi


def _correction_law(ar, draft, ids, pos, T, top_p, u_accept, top_k=0):
    """Law of the token emitted at `pos` when the step stops there, as a
    function of the residual uniform, measured interval by interval."""
    B, V = ar.shape[0] - 1, ar.shape[1]

    def token(u2):
        ur = np.full(B + 1, 0.5)
        ur[pos] = u2
        r = oracle.verify_one(ar, draft, ids, T, top_p, u_accept, ur, top_k=top_k)
        assert r["n_emitted"] == pos + 1
        return int(r["tokens"][pos])

    law = np.zeros(V)
    prev = 0.0
    for v in range(V):
        b = _sup_true(lambda u: token(u) <= v)
        law[v] = b - prev
        prev = b
    return law


def emission_law(ar, draft, ids, pos, T, top_p, q_pos, top_k=0):
    """P(token at pos = v | the step reached pos), drafts at pos ~ q_pos."""
    B, V = ar.shape[0] - 1, ar.shape[1]
    if pos == B:
        return _correction_law(ar, draft, ids, pos, T, top_p, np.zeros(B), top_k)
    law = np.zeros(V)
    for x in range(V):
        if q_pos[x] == 0.0:
            continue
        ids_x = np.array(ids, dtype=np.int32)
        ids_x[pos] = x

        def accepted(u):
            ua = np.zeros(B)
            ua[pos] = u
            r = oracle.verify_one(ar, draft, ids_x, T, top_p, ua, np.full(B + 1, 0.5),
                                  top_k=top_k)
            return r["n_emitted"] > pos + 1

        a = _sup_true(accepted)
        law[x] += q_pos[x] * a
        if a < 1.0:
            ua = np.zeros(B)
            ua[pos] = NEXT1
            law += q_pos[x] * (1.0 - a) * _correction_law(ar, draft, ids_x, pos, T, top_p, ua,
                                                          top_k)
    return law


def _target(row, T, top_p, top_k=0):
    if top_p >= 1.0 and top_k == 0:
        return softmax(row.astype(np.float64) / T)
    return oracle.row_probs(row, T, top_p, top_k)[0]  # pinned by the hand cases below


@pytest.mark.parametrize("case", range(12))
def test_lossless_exact(case):
    rng = np.random.default_rng(1000 + case)
    V = [2, 3, 5, 8][case % 4]
    B = [1, 2, 3][case % 3]
    T = [1.0, 0.7][case % 2]
    top_p = 1.0 if case < 8 else 0.8
    ar = rng.normal(0, 1.5, (B + 1, V)).astype(np.float32)
    draft = (ar[:B] + rng.normal(0, 1.0, (B, V))).astype(np.float32)
    if case % 5 == 4:  # a token the AR path can never emit
        ar[0, 0] = -np.inf
    # earlier positions must pass at u = 0: give them the AR argmax
    ids = np.array([int(np.argmax(ar[i])) for i in range(B)], dtype=np.int32)
    for pos in sorted({0, min(1, B - 1), B}):
        q_pos = _target(draft[pos], T, top_p) if pos < B else None
        law = emission_law(ar, draft, ids, pos, T, top_p, q_pos)
        np.testing.assert_allclose(law, _target(ar[pos], T, top_p), rtol=0, atol=1e-12,
                                   err_msg=f"pos {pos}")


@pytest.mark.parametrize("T", [1.0, 0.8])
def test_lossless_exact_spread_residual_under_top_p(T):
    """Top-p on both sides with a correction spread over several tokens, part
    of them in the draft's tail that its nucleus drops: the target keeps
    tokens 0-3, the draft mostly 5 and 6, so the residual max(0, p' - q') is
    p' itself on 0-3 and any use of the unfiltered q shifts its ratios."""
    ar_p = np.array([[0.25, 0.2, 0.2, 0.15, 0.1, 0.04, 0.03, 0.03],
                     [0.1, 0.3, 0.2, 0.1, 0.1, 0.1, 0.05, 0.05]])
    dr_p = np.array([[0.05, 0.05, 0.02, 0.02, 0.01, 0.5, 0.3, 0.05]])
    ar = np.log(ar_p).astype(np.float32)
    draft = np.log(dr_p).astype(np.float32)
    top_p = 0.7
    q_pos = _target(draft[0], T, top_p)
    law = emission_law(ar, draft, [5], 0, T, top_p, q_pos)
    np.testing.assert_allclose(law, _target(ar[0], T, top_p), rtol=0, atol=1e-12)
    assert np.count_nonzero(law > 0) >= 3


@pytest.mark.parametrize("q", [(0.5, 0.5), (0.9, 0.1), (0.2, 0.8), (1.0, 0.0)])
def test_seventy_thirty_exact(q):
    """The pages' example: a 70/30 target must come out 70/30."""
    ar = np.log(np.array([[0.7, 0.3], [0.5, 0.5]])).astype(np.float32)
    with np.errstate(divide="ignore"):
        draft = np.log(np.array([q])).astype(np.float32)
    q_pos = softmax(draft[0].astype(np.float64))
    law = emission_law(ar, draft, [0], 0, 1.0, 1.0, q_pos)
    np.testing.assert_allclose(law, softmax(ar[0].astype(np.float64)), atol=1e-12)
    np.testing.assert_allclose(law, [0.7, 0.3], atol=1e-7)


def test_seventy_thirty_sampled():
    n = 100_000
    ar = np.log(np.array([[0.7, 0.3], [0.5, 0.5]], dtype=np.float32))
    draft = np.log(np.array([[0.2, 0.8]], dtype=np.float32))
    rng = np.random.default_rng(7)
    ids = (rng.random(n) < 0.8).astype(np.int32).reshape(n, 1)
    r = oracle.verify_linear(np.broadcast_to(ar, (n, 2, 2)), np.broadcast_to(draft, (n, 1, 2)),
                             ids, 1.0, 1.0, seed=3, step=0)
    freq_a = np.mean(r["tokens"][:, 0] == 0)
    assert abs(freq_a - 0.7) < 4 * np.sqrt(0.21 / n)


def test_verify_draws_uniforms_from_the_counter():
    """The batch verify gives sequence s at step t the counter uniforms
    u(seed, s, t, row, purpose) (the generator is pinned by the published
    SplitMix64 vector and the chain test): purpose 0 for the acceptance test
    of each drafted row, purpose 1 for the draw at each row.  With those
    uniforms passed in, the single-sequence verify must agree exactly."""
    rng = np.random.default_rng(21)
    N, B, V = 12, 4, 6
    ar = rng.normal(0, 1, (N, B + 1, V)).astype(np.float32)
    draft = (ar[:, :B] + rng.normal(0, 0.7, (N, B, V))).astype(np.float32)
    ids = rng.integers(0, V, (N, B)).astype(np.int32)
    seq_ids = np.arange(N, dtype=np.uint64) * 7919 + 3
    seed = 17
    by_step = []
    for step in (0, 5):
        r = oracle.verify_linear(ar, draft, ids, 1.0, 1.0, seed=seed, step=step,
                                 seq_ids=seq_ids)
        for n in range(N):
            s = int(seq_ids[n])
            ua = [oracle.uniform(seed, s, step, i, oracle.PURPOSE_ACCEPT) for i in range(B)]
            ur = [oracle.uniform(seed, s, step, i, oracle.PURPOSE_RESID) for i in range(B + 1)]
            one = oracle.verify_one(ar[n], draft[n], ids[n], 1.0, 1.0, ua, ur)
            assert r["tokens"][n].tolist() == one["tokens"].tolist(), (step, n)
            assert r["n_emitted"][n] == one["n_emitted"], (step, n)
        by_step.append(r["tokens"])
    assert not np.array_equal(by_step[0], by_step[1])


# ---- statistics over RNG-driven draws ----------------------------------------

def _tiny_case():
    b = psi_inputs.linear_batch(psi_inputs.CONFIGS["tiny"])
    return psi_inputs.to_host_logits(b.ar)[0], psi_inputs.to_host_logits(b.draft)[0]


def _sample_ids(q, n, rng):
    cdf = np.cumsum(q, axis=-1)
    cdf[:, -1] = 1.0
    u = rng.random((n, q.shape[0]))
    return np.stack([np.searchsorted(cdf[i], u[:, i], side="right") for i in range(q.shape[0])],
                    axis=1).astype(np.int32)


def _draws(ar, draft, T, n_total, seed, chunk=50_000):
    B = draft.shape[0]
    q = softmax(draft.astype(np.float64) / T, axis=-1)
    rng = np.random.default_rng(seed)
    toks, ns = [], []
    for c0 in range(0, n_total, chunk):
        n = min(chunk, n_total - c0)
        ids = _sample_ids(q, n, rng)
        r = oracle.verify_linear(np.broadcast_to(ar, (n,) + ar.shape),
                                 np.broadcast_to(draft, (n,) + draft.shape), ids, T, 1.0,
                                 seed=seed, step=0, seq_ids=np.arange(c0, c0 + n, dtype=np.uint64))
        toks.append(r["tokens"])
        ns.append(r["n_emitted"])
    return np.concatenate(toks), np.concatenate(ns)


@pytest.fixture(scope="module")
def tiny_draws():
    ar, draft = _tiny_case()
    toks, ns = _draws(ar, draft, 1.0, 1_000_000, seed=0)
    return ar, draft, toks, ns


def test_chi_square_per_position(tiny_draws):
    ar, draft, toks, ns = tiny_draws
    B, V = draft.shape
    for i in range(B + 1):
        reached = ns > i
        counts = np.bincount(toks[reached, i], minlength=V)
        p = softmax(ar[i].astype(np.float64))
        if reached.sum() < 2000:
            continue
        res = stats.chisquare(counts, reached.sum() * p)
        assert res.pvalue > 1e-3, (i, res)


def test_acceptance_closed_form(tiny_draws):
    ar, draft, toks, ns = tiny_draws
    B = draft.shape[0]
    p = softmax(ar[:B].astype(np.float64), axis=-1)
    q = softmax(draft.astype(np.float64), axis=-1)
    alpha = np.minimum(p, q).sum(axis=-1)
    for i in range(B):
        reached = ns > i
        n = reached.sum()
        acc = np.mean(ns[reached] > i + 1)
        assert abs(acc - alpha[i]) < 4 * np.sqrt(alpha[i] * (1 - alpha[i]) / n) + 1e-12, i
    accepted = ns - 1
    expect = sum(np.prod(alpha[:k]) for k in range(1, B + 1))
    assert abs(accepted.mean() - expect) < 4 * accepted.std() / np.sqrt(len(ns))


def test_emitted_count_bounds(tiny_draws):
    _, draft, toks, ns = tiny_draws
    B, V = draft.shape
    assert ns.min() >= 1 and ns.max() <= B + 1
    col = np.arange(B + 1)[None, :]
    assert np.all((toks >= 0) == (col < ns[:, None]))
    assert toks.max() < V


# ---- top-p -------------------------------------------------------------------

def _probs(vals, T=1.0, top_p=1.0):
    p, st, _ = oracle.row_probs(np.asarray(vals, dtype=np.float32), T, top_p)
    assert st == 0
    return p


def test_top_p_hand_cases():
    ln = np.log(np.array([0.5, 0.3, 0.15, 0.05]))
    np.testing.assert_allclose(_probs(ln, 1.0, 0.7), [0.625, 0.375, 0, 0], atol=1e-7)
    np.testing.assert_allclose(_probs(ln, 1.0, 0.85),
                               [0.5 / 0.95, 0.3 / 0.95, 0.15 / 0.95, 0], atol=1e-7)
    np.testing.assert_allclose(_probs(ln, 1.0, 0.96), [0.5, 0.3, 0.15, 0.05], atol=1e-7)
    np.testing.assert_allclose(_probs(ln, 1.0, 0.45), [1, 0, 0, 0], atol=1e-7)
    # the same row in another vocabulary order
    perm = [2, 0, 3, 1]
    np.testing.assert_allclose(_probs(ln[perm], 1.0, 0.7), [0, 0.625, 0, 0.375], atol=1e-7)
    # temperature 0.5 squares the probabilities before the cut:
    # (.25, .09, .0225, .0025) / .365; top 0.9 keeps the first two
    np.testing.assert_allclose(_probs(ln, 0.5, 1.0),
                               np.array([0.25, 0.09, 0.0225, 0.0025]) / 0.365, atol=1e-7)
    np.testing.assert_allclose(_probs(ln, 0.5, 0.9), [0.25 / 0.34, 0.09 / 0.34, 0, 0], atol=1e-7)


def test_top_p_keeps_ties_at_threshold():
    a = np.e / (2 * np.e + 2)
    # first token alone reaches 0.3, its tie partner must be kept too
    np.testing.assert_allclose(_probs([1, 1, 0, 0], 1.0, 0.3), [0.5, 0.5, 0, 0], atol=1e-7)
    # crossing inside the lower tie group keeps the whole group
    assert 2 * a < 0.8
    np.testing.assert_allclose(_probs([1, 1, 0, 0], 1.0, 0.8), softmax([1.0, 1, 0, 0]), atol=1e-7)


def test_top_p_mass_reaching_exactly_stops_there():
    """The nucleus is the smallest set whose mass reaches top_p (>=): with
    top_p equal to the top token's mass that token alone is kept, one ulp more
    brings in the next.  top_p is set to that mass as double arithmetic gives
    it (e_0 = exp(0) = 1, e_v = exp(x_v - x_0), the total summed in vocabulary
    order); math.exp is the C library's exp."""
    x = np.array([0.0, -1.0, -3.0], dtype=np.float32)
    mass0 = 1.0 / ((1.0 + math.exp(-1.0)) + math.exp(-3.0))
    p, st, margin = oracle.row_probs(x, 1.0, mass0)
    assert st == 0 and p.tolist() == [1.0, 0.0, 0.0]
    assert margin == 0.0  # the cut sits exactly on the boundary
    p2 = _probs(x, 1.0, float(np.nextafter(mass0, 1.0)))
    assert p2[0] > 0 and p2[1] > 0 and p2[2] == 0


def test_top_p_limits():
    rng = np.random.default_rng(3)
    for _ in range(20):
        row = rng.normal(0, 2, 257).astype(np.float32)
        for T in (1.0, 0.7, 2.5):
            np.testing.assert_allclose(_probs(row, T, 1.0), softmax(row.astype(np.float64) / T),
                                       rtol=1e-12, atol=1e-15)
        row[[5, 77]] = row.max() + 1.0  # a two-way tie at the top
        p = _probs(row, 0.9, 1e-6)
        want = np.zeros(257)
        want[[5, 77]] = 0.5
        np.testing.assert_allclose(p, want, atol=1e-15)


# ---- top-k (run card: "top-k／top-p") ---------------------------------------------

def test_top_k_hand_cases():
    ln = np.log(np.array([0.5, 0.3, 0.15, 0.05]))
    np.testing.assert_allclose(_probs_k(ln, 1.0, 2), [0.625, 0.375, 0, 0], atol=1e-7)
    np.testing.assert_allclose(_probs_k(ln, 1.0, 3), [0.5 / 0.95, 0.3 / 0.95, 0.15 / 0.95, 0],
                               atol=1e-7)
    np.testing.assert_allclose(_probs_k(ln, 1.0, 1), [1, 0, 0, 0], atol=1e-7)
    for k in (0, 4, 9):  # off
        np.testing.assert_allclose(_probs_k(ln, 1.0, k), [0.5, 0.3, 0.15, 0.05], atol=1e-7)
    # another vocabulary order, and temperature first: T = 0.5 squares
    perm = [2, 0, 3, 1]
    np.testing.assert_allclose(_probs_k(ln[perm], 1.0, 2), [0, 0.625, 0, 0.375], atol=1e-7)
    np.testing.assert_allclose(_probs_k(ln, 0.5, 2), [0.25 / 0.34, 0.09 / 0.34, 0, 0], atol=1e-7)


def test_top_k_keeps_ties_with_the_kth():
    np.testing.assert_allclose(_probs_k([1, 1, 1, 0], 1.0, 2), [1 / 3, 1 / 3, 1 / 3, 0],
                               atol=1e-7)
    np.testing.assert_allclose(_probs_k([2, 1, 1, 0], 1.0, 2),
                               softmax([2.0, 1, 1]).tolist() + [0], atol=1e-7)


def test_top_k_comes_before_top_p():
    # top-k 3 renormalises to (.526, .316, .158); top-p 0.82 then stops at
    # .842 (two tokens).  top-p first would keep three (.5, .8, .95).
    ln = np.log(np.array([0.5, 0.3, 0.15, 0.05]))
    np.testing.assert_allclose(_probs_k(ln, 1.0, 3, 0.82), [0.625, 0.375, 0, 0], atol=1e-7)
    np.testing.assert_allclose(_probs(ln, 1.0, 0.82), [0.5 / 0.95, 0.3 / 0.95, 0.15 / 0.95, 0],
                               atol=1e-7)


def _probs_k(vals, T, top_k, top_p=1.0):
    p, st, _ = oracle.row_probs(np.asarray(vals, dtype=np.float32), T, top_p, top_k)
    assert st == 0
    return p


def test_top_k_one_is_greedy_decoding():
    """k = 1 leaves each distribution a point mass on its argmax: with the
    draft's argmax drafted, the sampled rule is the greedy rule."""
    rng = np.random.default_rng(15)
    N, B, V = 50, 5, 20
    ar = rng.normal(0, 1, (N, B + 1, V)).astype(np.float32)
    draft = (ar[:, :B] + rng.normal(0, 0.5, (N, B, V))).astype(np.float32)
    ids = np.argmax(draft, axis=-1).astype(np.int32)
    s = oracle.verify_linear(ar, draft, ids, 0.9, 1.0, seed=4, step=0, top_k=1)
    g = oracle.verify_linear(ar, None, ids, 0.0, 1.0, seed=4, step=0)
    assert np.array_equal(s["tokens"], g["tokens"])
    assert 1 < g["n_emitted"].mean() < B + 1


@pytest.mark.parametrize("case", range(4))
def test_lossless_exact_top_k(case):
    rng = np.random.default_rng(2000 + case)
    V, B = 6, 2
    T = [1.0, 0.7][case % 2]
    top_k = [2, 4][case // 2]
    top_p = [1.0, 0.9][case % 2]
    ar = rng.normal(0, 1.5, (B + 1, V)).astype(np.float32)
    draft = rng.normal(0, 1.5, (B, V)).astype(np.float32)
    ids = np.array([int(np.argmax(ar[i])) for i in range(B)], dtype=np.int32)
    for pos in (0, 1, B):
        q_pos = _target(draft[pos], T, top_p, top_k) if pos < B else None
        law = emission_law(ar, draft, ids, pos, T, top_p, q_pos, top_k)
        np.testing.assert_allclose(law, _target(ar[pos], T, top_p, top_k), rtol=0, atol=1e-12,
                                   err_msg=f"pos {pos}")


# ---- near-tie margins (O14) ----------------------------------------------------------
# The smallest distance of any decision from its threshold: each acceptance
# ratio, the top-p crossing (both sides) of every row used, and the draw's
# crossing (both sides).  The GPU parity tests excuse token differences only
# below 1e-5 of it, so each term is pinned by a case where it is the smallest.

def _margin(ar_p, dr_p, x, ua, ur, top_p=1.0):
    r = oracle.verify_one(_logp(ar_p), _logp(dr_p), [x], 1.0, top_p, ua, ur)
    return r["margin"], r


def _logp(rows):
    with np.errstate(divide="ignore"):
        return np.log(np.asarray(rows, dtype=np.float64)).astype(np.float32)


def test_margin_acceptance_ratio_and_draw():
    ar_p = [[0.5, 0.3, 0.2], [0.6, 0.2, 0.2]]
    dr_p = [[0.2, 0.6, 0.2]]
    # x = 1: p/q = 0.5; u = 0.7 rejects (distance 0.2); the residual (.3, 0, 0)
    # gives token 0, the draw at 0.5 is 0.5 from both crossings
    m, r = _margin(ar_p, dr_p, 1, [0.7], [0.5, 0.5])
    assert r["tokens"].tolist() == [0, -1] and abs(m - 0.2) < 1e-6
    # u = 0.99 (distance 0.49); the draw at 0.05 is 0.05 above the lower
    # crossing and 0.95 below the upper one
    m, r = _margin(ar_p, dr_p, 1, [0.99], [0.05, 0.5])
    assert r["tokens"].tolist() == [0, -1] and abs(m - 0.05) < 1e-6


def test_margin_top_p_crossings_of_draft_and_bonus_rows():
    # top_p = 0.52 everywhere.  AR row 0 (.4, .35, .15, .1): crossing masses
    # .4 / .75, margin .12.  Draft (.3, .51, .1, .09): .51 / .81, margin .01.
    # x = 1 accepted at u = .2 (ratio .741); bonus row (.7, .1, .1, .1): 0 / .7,
    # margin .18; the bonus draw (.7 alone) is .5 from both crossings.
    m, r = _margin([[0.4, 0.35, 0.15, 0.1], [0.7, 0.1, 0.1, 0.1]],
                   [[0.3, 0.51, 0.1, 0.09]], 1, [0.2], [0.5, 0.5], top_p=0.52)
    assert r["n_emitted"] == 2 and abs(m - 0.01) < 1e-6
    # the bonus row's crossing the smallest: bonus (.515, .3, .1, .085) gives
    # .515 / .815 (margin .005); draft (.3, .6, .05, .05): 0 / .6 (.08)
    m, r = _margin([[0.4, 0.35, 0.15, 0.1], [0.515, 0.3, 0.1, 0.085]],
                   [[0.3, 0.6, 0.05, 0.05]], 1, [0.1], [0.5, 0.3], top_p=0.52)
    assert r["n_emitted"] == 2 and r["tokens"].tolist() == [1, 0] and abs(m - 0.005) < 1e-6


def test_top_p_margin_is_two_sided():
    ln = np.log(np.array([0.5, 0.3, 0.15, 0.05]))
    # crossing between .5 and .8: distances .02 (below) and .28 (above)
    _, _, m = oracle.row_probs(ln.astype(np.float32), 1.0, 0.52)
    assert abs(m - 0.02) < 1e-6
    _, _, m = oracle.row_probs(ln.astype(np.float32), 1.0, 0.78)
    assert abs(m - 0.02) < 1e-6
    assert oracle.row_probs(ln.astype(np.float32), 1.0, 1.0)[2] == np.inf


def test_bf16_rows_decode_exactly():
    # hand-written bfloat16 bit patterns of 1, 0.5, -1, 2, 0, 3, -inf, -2
    bits = np.array([0x3F80, 0x3F00, 0xBF80, 0x4000, 0x0000, 0x4040, 0xFF80, 0xC000],
                    dtype=np.uint16)
    vals = np.array([1, 0.5, -1, 2, 0, 3, -np.inf, -2], dtype=np.float32)
    for T, tp in [(1.0, 1.0), (0.7, 0.9)]:
        pb, _, _ = oracle.row_probs(bits, T, tp)
        pf, _, _ = oracle.row_probs(vals, T, tp)
        assert np.array_equal(pb, pf)
    assert oracle.row_argmax(bits) == 5


def test_p_q_outputs_are_softmax_at_ids():
    rng = np.random.default_rng(11)
    N, B, V = 6, 5, 40
    ar = rng.normal(0, 2, (N, B + 1, V)).astype(np.float32)
    draft = rng.normal(0, 2, (N, B, V)).astype(np.float32)
    ids = rng.integers(0, V, (N, B)).astype(np.int32)
    r = oracle.verify_linear(ar, draft, ids, 0.8, 1.0, seed=1, step=2)
    p = softmax(ar[:, :B].astype(np.float64) / 0.8, axis=-1)
    q = softmax(draft.astype(np.float64) / 0.8, axis=-1)
    np.testing.assert_allclose(r["p_draft"], np.take_along_axis(p, ids[..., None], -1)[..., 0],
                               rtol=1e-12)
    np.testing.assert_allclose(r["q_draft"], np.take_along_axis(q, ids[..., None], -1)[..., 0],
                               rtol=1e-12)


# ---- greedy --------------------------------------------------------------------

def test_greedy_is_low_temperature_limit():
    rng = np.random.default_rng(5)
    N, B, V = 64, 6, 50
    ar = rng.normal(0, 1, (N, B + 1, V)).astype(np.float32)
    draft = (ar[:, :B] + rng.normal(0, 0.4, (N, B, V))).astype(np.float32)
    for x in (ar, draft):  # a clear winner in every row
        top = np.argmax(x, axis=-1)
        np.put_along_axis(x, top[..., None], x.max(axis=-1, keepdims=True) + 0.5, axis=-1)
    ids = np.argmax(draft, axis=-1).astype(np.int32)
    g = oracle.verify_linear(ar, None, ids, 0.0, 1.0, seed=9, step=0)
    s = oracle.verify_linear(ar, draft, ids, 1e-3, 1.0, seed=9, step=0)
    assert np.array_equal(g["tokens"], s["tokens"])
    assert np.array_equal(g["n_emitted"], s["n_emitted"])
    assert 1 < g["n_emitted"].mean() < B + 1


def test_greedy_ignores_draft_and_top_p():
    rng = np.random.default_rng(6)
    ar = rng.normal(0, 1, (4, 5, 30)).astype(np.float32)
    ids = np.argmax(ar[:, :4], axis=-1).astype(np.int32)
    ids[1, 2] = (ids[1, 2] + 1) % 30
    a = oracle.verify_linear(ar, None, ids, 0.0, 1.0, seed=0, step=0)
    b = oracle.verify_linear(ar, ar[:, :4].copy(), ids, 0.0, 0.3, seed=5, step=9)
    assert np.array_equal(a["tokens"], b["tokens"])
    assert a["n_emitted"].tolist() == [5, 3, 5, 5]


# ---- malformed inputs ------------------------------------------------------------

def test_bad_ids_are_rejected_and_flagged():
    ar = np.zeros((1, 3, 8), np.float32)
    draft = np.zeros((1, 2, 8), np.float32)
    for bad in (-1, 8, 1 << 30):
        ids = np.array([[bad, 0]], np.int32)
        r = oracle.verify_linear(ar, draft, ids, 1.0, 1.0, seed=0, step=0)
        assert r["status"] & oracle.BAD_TOKEN_ID
        assert r["n_emitted"][0] == 1 and r["p_draft"][0, 0] == 0 and r["q_draft"][0, 0] == 0
        g = oracle.verify_linear(ar, None, ids, 0.0, 1.0, seed=0, step=0)
        assert g["status"] & oracle.BAD_TOKEN_ID and g["n_emitted"][0] == 1


def test_nonfinite_flagged_but_neg_inf_allowed():
    ar = np.zeros((1, 3, 8), np.float32)
    draft = np.zeros((1, 2, 8), np.float32)
    ids = np.zeros((1, 2), np.int32)
    ar[0, 1, 3] = -np.inf
    assert oracle.verify_linear(ar, draft, ids, 1.0, 1.0, 0, 0)["status"] == 0
    for val in (np.nan, np.inf):
        a2 = ar.copy()
        a2[0, 2, 5] = val
        assert oracle.verify_linear(a2, draft, ids, 1.0, 1.0, 0, 0)["status"] & oracle.NONFINITE
        assert oracle.verify_linear(a2, None, ids, 0.0, 1.0, 0, 0)["status"] & oracle.NONFINITE
