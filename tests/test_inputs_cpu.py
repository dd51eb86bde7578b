"""The seeded input generators (CPU): they feed the same bytes to the oracle
and to the CUDA library, so their recipes are checked here against what they
state, not against either side of the verify step."""
import math

import numpy as np
import pytest
import torch
from scipy import stats
from scipy.special import softmax

import psi_inputs
from psi_inputs import CONFIGS, LinearConfig


def test_same_seed_and_index_give_the_same_bytes():
    cfg = CONFIGS["single_stream"]
    a = psi_inputs.linear_batch(cfg, N=2, V=3000, index=4)
    b = psi_inputs.linear_batch(cfg, N=2, V=3000, index=4)
    c = psi_inputs.linear_batch(cfg, N=2, V=3000, index=5)
    for x, y in ((a.ar, b.ar), (a.draft, b.draft), (a.ids, b.ids)):
        assert torch.equal(x, y)
    assert not torch.equal(a.ar, c.ar)


def test_shapes_and_dtypes():
    for name in ("tiny", "single_stream", "large_batch_nucleus", "max_batch_greedy"):
        cfg = CONFIGS[name]
        b = psi_inputs.linear_batch(cfg, N=2, V=min(cfg.V, 1000))
        V = min(cfg.V, 1000)
        assert tuple(b.ar.shape) == (2, cfg.B + 1, V) and tuple(b.draft.shape) == (2, cfg.B, V)
        assert b.ar.dtype == (torch.float32 if cfg.dtype == "f32" else torch.bfloat16)
        assert b.ids.dtype == torch.int32 and tuple(b.ids.shape) == (2, cfg.B)
        assert int(b.ids.min()) >= 0 and int(b.ids.max()) < V
        assert b.ar.is_contiguous() and b.draft.is_contiguous() and b.ids.is_contiguous()


def test_zipf_rows_follow_the_rank_law():
    """Each row is -1.1 ln(rank + 1) over a permutation plus N(0, 0.5^2): its
    mean and variance are those of the base law plus the noise's, and the
    permutation differs from row to row."""
    V, n = 4096, 64
    g = torch.Generator().manual_seed(1)
    rows = psi_inputs.zipf_rows(n, V, 0.5, g, "cpu").double()
    base = -1.1 * np.log(np.arange(V) + 1.0)
    means = rows.mean(dim=1).numpy()
    vars_ = rows.var(dim=1, unbiased=False).numpy()
    assert abs(means.mean() - base.mean()) < 4 * 0.5 / math.sqrt(V * n)
    assert abs(vars_.mean() - (base.var() + 0.25)) < 0.02 * (base.var() + 0.25)
    # the top of each row is the base's top: the largest value is near 0
    assert np.all(rows.max(dim=1).values.numpy() > -0.5 - 4 * 0.5)
    assert len(set(rows.argmax(dim=1).tolist())) > n // 2


def test_draft_is_ar_plus_gaussian_noise():
    cfg = LinearConfig("f32zipf", 4, 3, 5000, "f32", 1.0, 1.0, 9, 1, "zipf", 0.6)
    b = psi_inputs.linear_batch(cfg)
    d = (b.draft.double() - b.ar[:, :cfg.B].double()).flatten().numpy()
    assert abs(d.mean()) < 4 * 0.6 / math.sqrt(d.size)
    assert abs(d.std() - 0.6) < 0.01
    assert stats.kstest(d / 0.6, "norm").pvalue > 1e-3
    t = psi_inputs.linear_batch(CONFIGS["tiny"])
    e = (t.draft.double() - t.ar[:, :4].double()).flatten().numpy()
    assert abs(e.std() - 1.0) < 0.4  # 128 samples of N(0, 1)


@pytest.mark.parametrize("T", [1.0, 0.7])
def test_gumbel_max_samples_the_tempered_softmax(T):
    x = torch.tensor([1.0, 0.2, -0.5, 0.9, -2.0])
    n = 200_000
    g = torch.Generator().manual_seed(3)
    ids = psi_inputs.gumbel_max(x.expand(n, 5).contiguous(), T, g).numpy()
    p = softmax(x.double().numpy() / T)
    assert stats.chisquare(np.bincount(ids, minlength=5), n * p).pvalue > 1e-3


def test_zero_temperature_drafts_are_the_draft_argmax():
    x = torch.tensor([[0.5, 2.0, 2.0, -1.0], [3.0, 1.0, 3.0, 3.0]])
    assert psi_inputs.gumbel_max(x, 0.0, torch.Generator()).tolist() == [1, 0]
    cfg = CONFIGS["max_batch_greedy"]
    b = psi_inputs.linear_batch(cfg, N=3, V=2000)
    want = torch.argmax(b.draft.float(), dim=-1).to(torch.int32)
    assert torch.equal(b.ids, want)


def test_tree_batch_structure():
    cfg = CONFIGS["tree_greedy"]
    t = psi_inputs.tree_batch(cfg, N=3, V=3000, index=2)
    N, M = t.node_tokens.shape
    assert (N, M) == (3, cfg.M) and tuple(t.ar.shape) == (3, cfg.M + 1, 3000)
    assert t.ar.dtype == torch.bfloat16
    for n in range(N):
        par, dep, tok = t.parents[n].tolist(), t.depth[n].tolist(), t.node_tokens[n].tolist()
        for k in range(M):
            assert -1 <= par[k] < k  # parents precede children: prefix-closed
            assert dep[k] == (1 if par[k] == -1 else dep[par[k]] + 1)
            assert 0 <= tok[k] < 3000
        assert dep == sorted(dep) and max(dep) <= cfg.depth  # ordered by depth
        assert sum(1 for k in range(M) if par[k] == -1) <= cfg.width
        for node in [-1] + list(range(M)):  # siblings carry distinct tokens
            kids = [tok[k] for k in range(M) if par[k] == node]
            assert len(kids) == len(set(kids)) and len(kids) <= cfg.width
    # deeper levels exist: the best-first expansion goes past the root's children
    assert int(t.depth.max()) >= 3


def test_tree_iid_variant_keeps_the_structure():
    cfg = psi_inputs.TreeConfig("iid", 2, 20, 1000, 5, 3, 11, 1, iid=True)
    t = psi_inputs.tree_batch(cfg)
    assert tuple(t.ar.shape) == (2, 21, 1000)
    assert all(-1 <= p < k for row in t.parents.tolist() for k, p in enumerate(row))


def test_host_views_round_trip():
    x = torch.randn(3, 7).to(torch.bfloat16)
    bits = psi_inputs.to_host_logits(x)
    assert bits.dtype == np.uint16 and torch.equal(psi_inputs.from_bf16_bits(bits), x)
    f = torch.randn(2, 5)
    assert np.array_equal(psi_inputs.to_host_logits(f), f.numpy())


def test_headline_formula_bytes():
    # N (2B + 1) V x 2 bytes at N = 256, B = 8, V = 151,936 bf16
    assert psi_inputs.logits_nbytes(CONFIGS["large_batch_nucleus"]) == 1_322_450_944
