"""Sampled tree verify on the GPU (through the C ABI) against the oracle's
orc_verify_tree_sampled on the same seeded inputs.

Paths, path lengths and tokens must be identical except on near-tie trees
(the oracle's margin < 1e-5: an acceptance ratio, a draw crossing or a top-p
crossing within 1e-5 of its uniform or threshold), and such disagreements
must stay below 0.1% of the trees.  The status word must match.
"""
import numpy as np
import pytest
import torch

import oracle
import psi_inputs
import rejection_sampling_verify_b200 as psi
from helpers import NEAR_TIE

pytestmark = pytest.mark.gpu
CFG = psi_inputs.CONFIGS


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    yield


def _gpu(ar, tok, par, T, top_p, seed, step, seq_ids=None):
    sid = None
    if seq_ids is not None:
        sid = torch.as_tensor(np.asarray(seq_ids, dtype=np.uint64).view(np.int64), device="cuda")
    r = psi.verify_tree_sampled(ar.cuda(), tok.cuda(), par.cuda(), T, top_p, seed=seed, step=step,
                                seq_ids=sid)
    torch.cuda.synchronize()
    return dict(path_nodes=r.path_nodes.cpu().numpy(), path_len=r.path_len.cpu().numpy(),
                tokens=r.tokens.cpu().numpy(), status=int(r.status.item()) & 0xFFFFFFFF)


def _oracle(ar, tok, par, T, top_p, seed, step, seq_ids=None):
    return oracle.verify_tree_sampled(psi_inputs.to_host_logits(ar), tok.cpu().numpy(),
                                      par.cpu().numpy(), T, top_p, seed, step, seq_ids=seq_ids)


def _compare(g, o):
    """(trees, near ties, trees that differ); differences only at near ties."""
    near = o["margin"] < NEAR_TIE
    differ = (g["path_len"] != o["path_len"]) | np.any(g["tokens"] != o["tokens"], axis=1) | \
        np.any(g["path_nodes"] != o["path_nodes"], axis=1)
    assert not np.any(differ & ~near), np.nonzero(differ & ~near)[0][:10]
    assert g["status"] == o["status"], (g["status"], o["status"])
    return len(near), int(near.sum()), int(differ.sum())


@pytest.mark.parametrize("iid", [False, True])
def test_tree_recipe_sampled_nucleus(iid):
    """The tree workload (N=16 trees of 64 nodes, V=151936 bf16) at T = 0.7,
    top-p 0.95, several steps of fresh inputs."""
    cfg = CFG["tree_greedy"]
    if iid:
        cfg = psi_inputs.TreeConfig(**{**cfg.__dict__, "iid": True})
    total = near = differ = 0
    depths = []
    for step in range(4 if not iid else 2):
        tb = psi_inputs.tree_batch(cfg, device="cuda", index=step)
        g = _gpu(tb.ar, tb.node_tokens, tb.parents, 0.7, 0.95, cfg.seed, step)
        o = _oracle(tb.ar, tb.node_tokens, tb.parents, 0.7, 0.95, cfg.seed, step)
        n, ne, d = _compare(g, o)
        total, near, differ = total + n, near + ne, differ + d
        depths.append(o["path_len"])
    print(f"\ntree recipe (iid={iid}): {total} trees, {differ} differ, {near} near ties")
    assert differ <= 0.001 * total
    if not iid:
        assert np.concatenate(depths).max() >= 2  # the walk goes past the root's children


@pytest.mark.parametrize("top_p", [1.0, 0.9])
@pytest.mark.parametrize("T", [0.5, 1.0, 2.0])
def test_tree_handmade_sampled(T, top_p):
    """Hand trees on a small vocabulary: chains, stars with duplicate sibling
    tokens, deep and shallow branches; many steps so that every kind of
    acceptance and rejection happens."""
    V = 7
    g = torch.Generator().manual_seed(int(T * 10) + int(top_p * 100))
    trees = [([-1, 0, 1, 2], [1, 3, 0, 5]),                 # chain
             ([-1, -1, -1, -1, -1], [2, 2, 4, 2, 6]),        # star with duplicates
             ([-1, -1, 0, 0, 1, 4], [1, 2, 1, 3, 2, 2]),     # branches
             ([-1, 0, 0, 1, 1, 3, 3], [0, 1, 2, 3, 4, 5, 6])]
    M = max(len(p) for p, _ in trees)
    total = differ = 0
    for t_i, (par_l, tok_l) in enumerate(trees):
        m = len(par_l)
        par = torch.full((64, M), -1, dtype=torch.int32)
        tok = torch.zeros((64, M), dtype=torch.int32)
        par[:, :m] = torch.tensor(par_l, dtype=torch.int32)
        tok[:, :m] = torch.tensor(tok_l, dtype=torch.int32)
        # padding nodes hang off the last real node as extra leaves
        for k in range(m, M):
            par[:, k] = m - 1
            tok[:, k] = k % V
        ar = (1.5 * torch.randn(64, M + 1, V, generator=g)).to(torch.bfloat16)
        for step in range(3):
            gg = _gpu(ar, tok, par, T, top_p, 17 + t_i, step)
            oo = _oracle(ar, tok, par, T, top_p, 17 + t_i, step)
            n, _, d = _compare(gg, oo)
            total, differ = total + n, differ + d
    assert differ <= 0.001 * total


def test_tree_sampled_flags_and_bad_nodes():
    """Bad parents and tokens are flagged and never taken, as in the oracle."""
    V = 6
    par = torch.tensor([[-1, 0, 5, 1], [-1, -1, 0, 2]], dtype=torch.int32)   # node 2 bad parent
    tok = torch.tensor([[1, 2, 3, 4], [0, 9, 1, 2]], dtype=torch.int32)      # token 9 bad
    ar = torch.randn(2, 5, V).to(torch.bfloat16)
    for step in range(8):
        g = _gpu(ar, tok, par, 1.0, 1.0, 5, step)
        o = _oracle(ar, tok, par, 1.0, 1.0, 5, step)
        assert o["status"] == oracle.BAD_PARENT | oracle.BAD_TOKEN_ID
        _compare(g, o)


@pytest.mark.parametrize("top_p", [0.9, 1.0])
def test_tree_sampled_flat_rows_exact_path(top_p):
    """Flat rows (i.i.d. N(0, 2^2) float32 logits, V = 40000): with top-p the
    nucleus does not fit the candidate lists and the walk settles the rows on
    its exact whole-row path; without top-p every draw is a whole-row draw."""
    g = torch.Generator().manual_seed(7)
    N, M, V = 4, 6, 40000
    par = torch.tensor([[-1, 0, 0, 1, 1, 2]] * N, dtype=torch.int32)
    ar = 2.0 * torch.randn(N, M + 1, V, generator=g)
    tok = torch.argmax(ar[:, 1:, :] + torch.randn(N, M, V, generator=g), dim=-1).to(torch.int32)
    for step in range(2):
        gg = _gpu(ar, tok, par, 1.0, top_p, 3, step)
        oo = _oracle(ar, tok, par, 1.0, top_p, 3, step)
        _compare(gg, oo)


def test_tree_sampled_seq_ids_and_batch_invariance():
    cfg = CFG["tree_greedy"]
    tb = psi_inputs.tree_batch(cfg, device="cuda", N=4, index=9)
    sids = np.array([100, 7, 2**63 + 1, 42], dtype=np.uint64)
    g = _gpu(tb.ar, tb.node_tokens, tb.parents, 0.8, 0.9, 1, 2, seq_ids=sids)
    o = _oracle(tb.ar, tb.node_tokens, tb.parents, 0.8, 0.9, 1, 2, seq_ids=sids)
    _compare(g, o)
    pick = [2, 0]
    g2 = _gpu(tb.ar[pick], tb.node_tokens[pick], tb.parents[pick], 0.8, 0.9, 1, 2,
              seq_ids=sids[pick])
    for k in ("path_nodes", "path_len", "tokens"):
        assert np.array_equal(g[k][pick], g2[k])


def test_tree_sampled_zero_temperature_is_greedy():
    cfg = CFG["tree_greedy"]
    tb = psi_inputs.tree_batch(cfg, device="cuda", N=3, index=2)
    g = _gpu(tb.ar, tb.node_tokens, tb.parents, 0.0, 0.9, 0, 0)
    r = psi.verify_tree_greedy(tb.ar, tb.node_tokens, tb.parents)
    torch.cuda.synchronize()
    assert np.array_equal(g["tokens"], r.tokens.cpu().numpy())
    assert np.array_equal(g["path_len"], r.path_len.cpu().numpy())
