"""Early-exit rounds of the sampled linear verify (no p / q outputs requested):
tokens and counts must equal the oracle's and, exactly, the GPU's own
every-row results on the same inputs."""
import numpy as np
import pytest
import torch

import psi_inputs
from helpers import assert_linear_parity, gpu_linear, oracle_linear

pytestmark = pytest.mark.gpu

CFG = psi_inputs.CONFIGS


def _batch(ar, draft, ids, T, top_p):
    return psi_inputs.LinearBatch(ar, draft, ids, T, top_p)


def _check(b, seed, step, seq_ids=None, oracle_rows=None):
    early = gpu_linear(b, seed, step, seq_ids=seq_ids, want_probs=False)
    full = gpu_linear(b, seed, step, seq_ids=seq_ids, want_probs=True)
    assert np.array_equal(early["tokens"], full["tokens"])
    assert np.array_equal(early["n_emitted"], full["n_emitted"])
    assert early["status"] == full["status"]
    if oracle_rows is None:
        assert_linear_parity(early, oracle_linear(b, seed, step, seq_ids=seq_ids))
    return early


@pytest.mark.parametrize("index", range(3))
def test_early_exit_nucleus_recipe(index):
    cfg = CFG["large_batch_nucleus"]
    b = psi_inputs.linear_batch(cfg, device="cuda", N=16, index=index)
    g = _check(b, cfg.seed, index)
    # some sequences stop in the first round, some run past it
    assert g["n_emitted"].min() <= 3 and g["n_emitted"].max() >= 1


@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 8, 32])
@pytest.mark.parametrize("top_p", [1.0, 0.8])
def test_early_exit_block_sizes(B, top_p):
    rng = torch.Generator().manual_seed(100 + B)
    N, V = 6, 5003
    ar = (1.2 * torch.randn(N, B + 1, V, generator=rng)).to(torch.bfloat16)
    draft = (ar[:, :B].float() + 0.2 * torch.randn(N, B, V, generator=rng)).to(torch.bfloat16)
    ids = psi_inputs.gumbel_max(draft, 1.0, rng)
    _check(_batch(ar, draft, ids, 1.0, top_p), 9, B)


def test_early_exit_single_stream_recipe():
    cfg = CFG["single_stream"]
    b = psi_inputs.linear_batch(cfg, device="cuda", index=1)
    _check(b, cfg.seed, 4)


def test_early_exit_tiny_recipe_many_sequences():
    cfg = CFG["tiny"]
    base = psi_inputs.linear_batch(cfg, device="cpu")
    n = 1000
    rng = np.random.default_rng(3)
    q = torch.softmax(base.draft[0].double(), -1).numpy()
    ids = np.stack([rng.choice(cfg.V, size=n, p=q[i] / q[i].sum()) for i in range(cfg.B)],
                   axis=1).astype(np.int32)
    b = _batch(base.ar.expand(n, -1, -1).contiguous(), base.draft.expand(n, -1, -1).contiguous(),
               torch.tensor(ids), cfg.temperature, cfg.top_p)
    _check(b, cfg.seed, 2)


def test_early_exit_rescanned_and_general_units():
    # rows whose top-p mass reaches below the first window (second scan)
    g = torch.Generator().manual_seed(21)
    N, B, V = 3, 3, 20000
    ar = torch.full((N, B + 1, V), -40.0)
    for n in range(N):
        for i in range(B + 1):
            perm = torch.randperm(V, generator=g)
            ar[n, i, perm[:2]] = 0.0
            ar[n, i, perm[2:1502]] = -13.5 * float(np.log(2.0))
    draft = ar[:, :B] + 0.05 * torch.randn(N, B, V, generator=g)
    ar, draft = ar.to(torch.bfloat16), draft.to(torch.bfloat16)
    ids = psi_inputs.gumbel_max(draft, 1.0, g)
    _check(_batch(ar.cuda(), draft.cuda(), ids, 1.0, 0.95), 6, 0)
    # flat rows: every unit goes to the general path
    for top_p in (0.9, 1.0):
        cfg = psi_inputs.LinearConfig("flat", 24, 4, 40000, "f32", 1.0, top_p, 31, 1, "tiny", 1.0)
        _check(psi_inputs.linear_batch(cfg, device="cuda"), 3, 1)


def test_early_exit_full_size_sampled():
    """The benchmark's workload: every sequence equal to the every-row run,
    a sample checked against the oracle one by one."""
    cfg = CFG["large_batch_nucleus"]
    b = psi_inputs.linear_batch(cfg, device="cuda")
    g = _check(b, cfg.seed, 7, oracle_rows=False)
    pick = np.array([1, 64, 200, 255])
    sub = _batch(b.ar[pick].cpu(), b.draft[pick].cpu(), b.ids[pick].cpu(), cfg.temperature,
                 cfg.top_p)
    o = oracle_linear(sub, cfg.seed, 7, seq_ids=pick.astype(np.uint64))
    gs = {k: (v[pick] if isinstance(v, np.ndarray) else v) for k, v in g.items()}
    gs["status"] = 0
    assert_linear_parity(gs, o)
    assert g["status"] == 0


def test_early_exit_deterministic():
    cfg = CFG["large_batch_nucleus"]
    b = psi_inputs.linear_batch(cfg, device="cuda", N=32, index=5)
    r1 = gpu_linear(b, 1, 2, want_probs=False)
    r2 = gpu_linear(b, 1, 2, want_probs=False)
    assert np.array_equal(r1["tokens"], r2["tokens"])
    assert np.array_equal(r1["n_emitted"], r2["n_emitted"])
