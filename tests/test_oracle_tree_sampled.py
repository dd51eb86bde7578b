"""Pins for the oracle's sampled tree verify (CPU only).

The pages' tree sampler ([P3] "Linear 與 Tree sampler") keeps several
candidates per position in a prefix tree but gives no sampled rule; the
oracle takes recursive rejection over each node's children, every child its
own point-mass proposal.  What fixes it here, other than itself:
  * hand-worked cases (arithmetic in the comments);
  * losslessness integrated EXACTLY: every decision is a step function of one
    uniform, so nested bisection on the oracle's outputs gives the probability
    of every emitted sequence; it must equal the autoregressive law of the
    tree's targets (a token equal to a child's token continues at that child,
    any other token ends the step) to 1e-12;
  * the batch form draws node k's acceptance uniform at row k+1 and the final
    draw's at its row, from the counter generator;
  * as T -> 0 on trees with distinct sibling tokens it is the greedy tree;
  * chi-square of the RNG-driven first and second tokens;
  * invalid nodes are flagged and never taken.
"""
import numpy as np
import pytest
from scipy import stats
from scipy.special import softmax

import oracle

NEXT1 = float(np.nextafter(1.0, 0.0))


def _logp(rows):
    with np.errstate(divide="ignore"):
        return np.log(np.asarray(rows, dtype=np.float64)).astype(np.float32)


def _one(ar, tok, par, ua, ur, T=1.0, top_p=1.0, top_k=0):
    return oracle.verify_tree_sampled_one(ar, tok, par, T, top_p, ua, ur, top_k=top_k)


# ---- hand-worked cases ---------------------------------------------------------

# root P = (.5, .3, .2); row 1 P = (.1, .8, .1); row 2 P = (.6, .2, .2)
ROWS = _logp([[0.5, 0.3, 0.2], [0.1, 0.8, 0.1], [0.6, 0.2, 0.2]])


def test_reject_first_child_accept_second_then_bonus():
    # child 0 (token 1): 0.35 < 0.3? no -> removed, R = 0.7
    # child 1 (token 2): 0.25 * 0.7 = 0.175 < 0.2 -> accepted
    # node 1 is a leaf: bonus from row 2 at u = 0.5 -> cumulative 0.6 > 0.5 -> 0
    r = _one(ROWS, [1, 2], [-1, -1], [0, 0.35, 0.25], [0.5, 0.5, 0.5])
    assert r["path_nodes"].tolist() == [1, -1] and r["path_len"] == 1
    assert r["tokens"].tolist() == [2, 0, -1]
    assert r["status"] == 0
    assert abs(r["margin"] - abs(0.25 - 0.2 / 0.7)) < 1e-6


def test_all_children_rejected_draws_from_what_remains():
    # 0.9 >= 0.3 rejects token 1; 0.9 * 0.7 >= 0.2 rejects token 2;
    # what remains is (.5, 0, 0): token 0 whatever the draw's uniform
    for u in (0.0, 0.5, NEXT1):
        r = _one(ROWS, [1, 2], [-1, -1], [0, 0.9, 0.9], [u, 0.5, 0.5])
        assert r["path_len"] == 0 and r["tokens"].tolist() == [0, -1, -1]


def test_two_levels_accepted():
    # chain root -> node 0 (token 1) -> node 1 (token 0)
    # 0.1 < 0.3 accepts node 0; at row 1, 0.05 < 0.1 accepts node 1;
    # node 1 is a leaf: row 2 at u = 0.7 -> 0.6, 0.8 > 0.7 -> token 1
    r = _one(ROWS, [1, 0], [-1, 0], [0, 0.1, 0.05], [0.5, 0.5, 0.7])
    assert r["path_nodes"].tolist() == [0, 1] and r["path_len"] == 2
    assert r["tokens"].tolist() == [1, 0, 1]


def test_duplicate_sibling_never_taken_after_its_token_was_rejected():
    # both children carry token 1; 0.5 >= 0.3 rejects the first and removes
    # token 1, so the second has mass 0 and is rejected even at u = 0;
    # the draw from (.5, 0, .2) / .7 at u = 0.75 crosses at token 2 (0.7 > 0.525)
    r = _one(ROWS, [1, 1], [-1, -1], [0, 0.5, 0.0], [0.75, 0.5, 0.5])
    assert r["path_len"] == 0 and r["tokens"].tolist() == [2, -1, -1]


def test_leaf_root_is_a_plain_draw():
    # the only node hangs off nothing usable (bad parent): the root is a leaf
    r = _one(ROWS[:2], [1], [5], [0, 0.0], [0.55, 0.5])
    assert r["status"] & oracle.BAD_PARENT
    assert r["path_len"] == 0 and r["tokens"].tolist() == [1, -1]  # 0.5, 0.8 > 0.55


def test_margin_includes_the_node_rows_top_p_crossing():
    # root (.515, .3, .1, .085) at top_p .52: crossing masses .515 / .815,
    # margin .005; the only child (token 3) is cut by top-p (P = 0, distance
    # .5 at u = .5); the draw from (.632, .368) at .3 is .3 from its crossings
    rows = _logp([[0.515, 0.3, 0.1, 0.085], [0.25, 0.25, 0.25, 0.25]])
    r = _one(rows, [3], [-1], [0, 0.5], [0.3, 0.5], top_p=0.52)
    assert r["path_len"] == 0 and r["tokens"].tolist() == [0, -1]
    assert abs(r["margin"] - 0.005) < 1e-6


def test_zero_temperature_is_the_greedy_tree():
    rng = np.random.default_rng(4)
    ar = rng.normal(0, 1, (7, 9)).astype(np.float32)
    par = [-1, -1, 0, 0, 1, 2]
    tok = [int(np.argmax(ar[0])), 3, int(np.argmax(ar[1])), 5, 1, int(np.argmax(ar[3]))]
    r = _one(ar, tok, par, np.full(7, 0.5), np.full(7, 0.5), T=0.0)
    g = oracle.verify_tree_greedy(ar[None], np.array([tok]), np.array([par]))
    assert r["tokens"].tolist() == g["tokens"][0].tolist()
    assert r["path_len"] == g["path_len"][0]


# ---- exact losslessness ----------------------------------------------------------

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


def _children(par, node):
    return [k for k in range(len(par)) if par[k] == node]


def oracle_sequence_law(ar, tok, par, T, top_p, top_k=0):
    """P(emitted token sequence), integrated over the verify's uniforms with
    the oracle as a black box."""
    M, V = len(tok), ar.shape[1]
    law = {}

    def run(ua, ur):
        return _one(ar, tok, par, ua, ur, T, top_p, top_k)

    def visit(node, depth, prefix, weight, ua, ur):
        ua = ua.copy()
        for k in _children(par, node):
            def accepted(u, k=k):
                trial = ua.copy()
                trial[k + 1] = u
                r = run(trial, ur)
                return r["path_len"] > depth and r["path_nodes"][depth] == k

            a = _sup_true(accepted)
            if a > 0.0:
                taken = ua.copy()
                taken[k + 1] = 0.0
                visit(k, depth + 1, prefix + (tok[k],), weight * a, taken, ur)
            weight *= 1.0 - a
            ua[k + 1] = NEXT1
            if weight == 0.0:
                return
        row, prev = node + 1, 0.0
        for v in range(V):
            def at_most(u, v=v):
                trial = ur.copy()
                trial[row] = u
                r = run(ua, trial)
                assert r["path_len"] == depth
                return r["tokens"][depth] <= v

            b = _sup_true(at_most)
            if b > prev:
                law[prefix + (v,)] = law.get(prefix + (v,), 0.0) + weight * (b - prev)
            prev = b

    visit(-1, 0, (), 1.0, np.full(M + 1, 0.5), np.full(M + 1, 0.5))
    return law


def _target(row, T, top_p, top_k=0):
    if top_p >= 1.0 and top_k == 0:
        return softmax(row.astype(np.float64) / T)
    return oracle.row_probs(row, T, top_p, top_k)[0]  # top-k / top-p are pinned on their own


def target_sequence_law(ar, tok, par, T, top_p, top_k=0):
    """The autoregressive law the step must reproduce: at a node, token v has
    the row's target probability; it continues at the first child carrying v,
    or ends the step."""
    law = {}

    def visit(node, prefix, weight):
        P = _target(ar[node + 1], T, top_p, top_k)
        first = {}
        for k in _children(par, node):
            first.setdefault(tok[k], k)
        for v in np.flatnonzero(P > 0):
            v = int(v)
            if v in first:
                visit(first[v], prefix + (v,), weight * P[v])
            else:
                law[prefix + (v,)] = weight * P[v]

    visit(-1, (), 1.0)
    return law


def _assert_same_law(got, want):
    keys = set(got) | set(want)
    for k in keys:
        assert abs(got.get(k, 0.0) - want.get(k, 0.0)) < 1e-12, (k, got.get(k), want.get(k))
    assert abs(sum(got.values()) - 1.0) < 1e-12


TREES = {
    "star": ([-1, -1, -1], [1, 3, 0]),
    "chain": ([-1, 0, 1], [2, 1, 1]),
    "mixed": ([-1, -1, 0, 0, 1, 2], [0, 2, 1, 3, 0, 4]),
    "duplicate_siblings": ([-1, -1, 0, 1], [1, 1, 2, 3]),
}


@pytest.mark.parametrize("name", sorted(TREES))
@pytest.mark.parametrize("T,top_p,top_k", [(1.0, 1.0, 0), (0.7, 1.0, 0), (1.0, 0.8, 0),
                                           (0.9, 1.0, 3)])
def test_lossless_exact_hand_trees(name, T, top_p, top_k):
    par, tok = TREES[name]
    rng = np.random.default_rng(sorted(TREES).index(name))
    ar = rng.normal(0, 1.5, (len(par) + 1, 5)).astype(np.float32)
    ar[0, 4] = -np.inf  # a token the root can never emit
    _assert_same_law(oracle_sequence_law(ar, tok, par, T, top_p, top_k),
                     target_sequence_law(ar, tok, par, T, top_p, top_k))


@pytest.mark.parametrize("case", range(6))
def test_lossless_exact_random_trees(case):
    rng = np.random.default_rng(500 + case)
    M, V = [3, 5, 7][case % 3], [3, 4, 6][case % 3]
    par = [int(rng.integers(-1, k)) for k in range(M)]
    tok = rng.integers(0, V, M).tolist()
    T, top_p = [(1.0, 1.0), (0.8, 0.9)][case % 2]
    ar = rng.normal(0, 1.5, (M + 1, V)).astype(np.float32)
    _assert_same_law(oracle_sequence_law(ar, tok, par, T, top_p),
                     target_sequence_law(ar, tok, par, T, top_p))


# ---- counter uniforms, limits, statistics -------------------------------------------

def test_batch_draws_uniforms_from_the_counter():
    rng = np.random.default_rng(8)
    N, M, V = 10, 6, 5
    par = np.array([[-1, -1, 0, 0, 1, 3]] * N, np.int32)
    ar = rng.normal(0, 1, (N, M + 1, V)).astype(np.float32)
    tok = rng.integers(0, V, (N, M)).astype(np.int32)
    seq_ids = np.arange(N, dtype=np.uint64) * 104729 + 11
    seed = 23
    by_step = []
    for step in (0, 4):
        r = oracle.verify_tree_sampled(ar, tok, par, 1.0, 1.0, seed, step, seq_ids=seq_ids)
        for n in range(N):
            s = int(seq_ids[n])
            ua = [0.0] + [oracle.uniform(seed, s, step, j, oracle.PURPOSE_ACCEPT)
                          for j in range(1, M + 1)]
            ur = [oracle.uniform(seed, s, step, j, oracle.PURPOSE_RESID) for j in range(M + 1)]
            one = _one(ar[n], tok[n], par[n], ua, ur)
            assert r["tokens"][n].tolist() == one["tokens"].tolist(), (step, n)
            assert r["path_len"][n] == one["path_len"]
        by_step.append(r["tokens"])
    assert not np.array_equal(by_step[0], by_step[1])


def test_low_temperature_is_greedy_on_distinct_siblings():
    rng = np.random.default_rng(12)
    N, M, V = 40, 8, 12
    ar = rng.normal(0, 1, (N, M + 1, V)).astype(np.float32)
    top = np.argmax(ar, axis=-1)
    np.put_along_axis(ar, top[..., None], ar.max(axis=-1, keepdims=True) + 0.5, axis=-1)
    par = np.array([[-1, -1, -1, 0, 0, 1, 3, 3]] * N, np.int32)
    tok = np.empty((N, M), np.int32)
    for n in range(N):  # distinct tokens among siblings, the argmax often among them
        for node in (-1, 0, 1, 3):
            kids = [k for k in range(M) if par[n, k] == node]
            choice = rng.permutation(V)[:len(kids)]
            if rng.random() < 0.7:
                am = top[n, node + 1]
                if am not in choice:
                    choice[rng.integers(len(kids))] = am
            tok[n, kids] = choice
    s = oracle.verify_tree_sampled(ar, tok, par, 1e-3, 1.0, seed=3, step=0)
    g = oracle.verify_tree_greedy(ar, tok, par)
    assert np.array_equal(s["tokens"], g["tokens"])
    assert np.array_equal(s["path_len"], g["path_len"])
    assert g["path_len"].max() >= 2


def test_chi_square_first_and_second_tokens():
    rng = np.random.default_rng(2)
    V = 6
    par, tok = [-1, -1, 0, 0], [1, 4, 0, 1]
    ar = rng.normal(0, 1, (5, V)).astype(np.float32)
    n = 200_000
    r = oracle.verify_tree_sampled(np.broadcast_to(ar, (n,) + ar.shape),
                                   np.broadcast_to(np.array(tok, np.int32), (n, 4)),
                                   np.broadcast_to(np.array(par, np.int32), (n, 4)),
                                   1.0, 1.0, seed=7, step=1)
    t0 = r["tokens"][:, 0]
    p0 = softmax(ar[0].astype(np.float64))
    assert stats.chisquare(np.bincount(t0, minlength=V), n * p0).pvalue > 1e-3
    # after the first token equals child 0's token (1), the second follows row 1
    sel = t0 == 1
    assert np.all(r["path_nodes"][sel, 0] == 0)
    p1 = softmax(ar[1].astype(np.float64))
    got = np.bincount(r["tokens"][sel, 1], minlength=V)
    assert stats.chisquare(got, sel.sum() * p1).pvalue > 1e-3


def test_paths_are_root_chains():
    rng = np.random.default_rng(31)
    N, M, V = 300, 9, 7
    ar = rng.normal(0, 1, (N, M + 1, V)).astype(np.float32)
    par = np.array([[int(rng.integers(-1, k)) for k in range(M)] for _ in range(N)], np.int32)
    tok = rng.integers(0, V, (N, M)).astype(np.int32)
    r = oracle.verify_tree_sampled(ar, tok, par, 0.9, 0.95, seed=1, step=2)
    assert r["status"] == 0
    for n in range(N):
        L = r["path_len"][n]
        path = r["path_nodes"][n]
        assert np.all(path[L:] == -1) and np.all(r["tokens"][n, L + 1:] == -1)
        prev = -1
        for d in range(L):
            assert par[n, path[d]] == prev and r["tokens"][n, d] == tok[n, path[d]]
            prev = path[d]
        assert 0 <= r["tokens"][n, L] < V


def test_invalid_nodes_flagged_and_never_taken():
    ar = np.zeros((4, 6), np.float32)
    ar[0, 2] = 5.0  # the root almost surely emits token 2
    # node 0: bad token; node 1: token 2 but parent index not below its own
    r = _one(ar, [9, 2, 2], [-1, 1, -1], np.zeros(4), np.full(4, 0.5))
    assert r["status"] & oracle.BAD_TOKEN_ID and r["status"] & oracle.BAD_PARENT
    assert r["path_nodes"].tolist()[:1] == [2] and r["tokens"][0] == 2
