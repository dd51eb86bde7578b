"""Early-exit rounds of the linear verify (no p / q outputs requested, batch
large enough): tokens and counts must equal the oracle's and, exactly, the
GPU's own every-row results on the same inputs."""
import numpy as np
import pytest
import torch

import psi_inputs
from helpers import assert_linear_parity, gpu_linear, oracle_linear

pytestmark = pytest.mark.gpu

CFG = psi_inputs.CONFIGS


def _batch(ar, draft, ids, T, top_p):
    return psi_inputs.LinearBatch(ar, draft, ids, T, top_p)


MIN_N = 64  # PSI_EARLY_EXIT_MIN_N


def _check(b, seed, step):
    """Early exit against the every-row run (all sequences, exactly) and the
    oracle (all sequences)."""
    assert b.ar.shape[0] >= MIN_N
    early = gpu_linear(b, seed, step, want_probs=False)
    full = gpu_linear(b, seed, step, want_probs=True)
    assert np.array_equal(early["tokens"], full["tokens"])
    assert np.array_equal(early["n_emitted"], full["n_emitted"])
    assert early["status"] == full["status"]
    assert_linear_parity(early, oracle_linear(b, seed, step))
    return early


@pytest.mark.parametrize("index", range(3))
def test_early_exit_nucleus_recipe(index):
    cfg = CFG["large_batch_nucleus"]
    b = psi_inputs.linear_batch(cfg, device="cuda", N=MIN_N, index=index)
    g = _check(b, cfg.seed, index)
    # some sequences stop in the first round, some run past it
    assert g["n_emitted"].min() <= 3 and g["n_emitted"].max() > 3


@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 8, 32])
@pytest.mark.parametrize("top_p", [1.0, 0.8])
def test_early_exit_block_sizes(B, top_p):
    rng = torch.Generator().manual_seed(100 + B)
    N, V = MIN_N, 5003
    ar = (1.2 * torch.randn(N, B + 1, V, generator=rng)).to(torch.bfloat16)
    draft = (ar[:, :B].float() + 0.2 * torch.randn(N, B, V, generator=rng)).to(torch.bfloat16)
    ids = psi_inputs.gumbel_max(draft, 1.0, rng)
    _check(_batch(ar, draft, ids, 1.0, top_p), 9, B)


def test_early_exit_single_stream_recipe():
    cfg = CFG["single_stream"]
    b = psi_inputs.linear_batch(cfg, device="cuda", N=MIN_N, index=1)
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
    N, B, V = MIN_N, 3, 20000
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
        cfg = psi_inputs.LinearConfig("flat", MIN_N, 4, 40000, "f32", 1.0, top_p, 31, 1, "tiny",
                                      1.0)
        _check(psi_inputs.linear_batch(cfg, device="cuda"), 3, 1)


def test_early_exit_full_size():
    """The benchmark's workload: every sequence equal to the every-row run
    and to the oracle."""
    cfg = CFG["large_batch_nucleus"]
    b = psi_inputs.linear_batch(cfg, device="cuda")
    g = _check(b, cfg.seed, 7)
    assert g["status"] == 0


def test_small_batches_read_every_row():
    """Below PSI_EARLY_EXIT_MIN_N sequences the tokens-only call is the
    every-row pass (same results either way)."""
    cfg = CFG["single_stream"]
    b = psi_inputs.linear_batch(cfg, device="cuda", index=2)
    early = gpu_linear(b, cfg.seed, 1, want_probs=False)
    full = gpu_linear(b, cfg.seed, 1, want_probs=True)
    assert np.array_equal(early["tokens"], full["tokens"])
    assert_linear_parity(early, oracle_linear(b, cfg.seed, 1))


def test_early_exit_deterministic():
    cfg = CFG["large_batch_nucleus"]
    b = psi_inputs.linear_batch(cfg, device="cuda", N=MIN_N, index=5)
    r1 = gpu_linear(b, 1, 2, want_probs=False)
    r2 = gpu_linear(b, 1, 2, want_probs=False)
    assert np.array_equal(r1["tokens"], r2["tokens"])
    assert np.array_equal(r1["n_emitted"], r2["n_emitted"])


def _greedy_raw(b, with_pq):
    """Greedy verify through the C ABI; with_pq passes p / q buffers (which
    T = 0 never writes) to ask for every row to be read."""
    import rejection_sampling_verify_b200 as psi
    N, B1, V = b.ar.shape
    B = B1 - 1
    code = psi.PSI_DTYPE_BF16 if b.ar.dtype == torch.bfloat16 else psi.PSI_DTYPE_F32
    tok = torch.empty(N, B + 1, dtype=torch.int32, device="cuda")
    cnt = torch.empty(N, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pq = torch.zeros(2, N, B, device="cuda") if with_pq else None
    ws_bytes = psi.psi_verify_linear_workspace_bytes(N, B, V, code, 0.0, 1.0)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    ids = b.ids.to("cuda")
    r = psi.psi_verify_linear(b.ar.data_ptr(), V, 0, V, code, ids.data_ptr(), N, B, V, 0.0, 1.0,
                              0, 0, 0, tok.data_ptr(), cnt.data_ptr(),
                              pq[0].data_ptr() if with_pq else 0,
                              pq[1].data_ptr() if with_pq else 0, st.data_ptr(), ws.data_ptr(),
                              ws_bytes, 0)
    assert r == psi.PSI_OK, psi.psi_last_error()
    torch.cuda.synchronize()
    return tok.cpu().numpy(), cnt.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("B", [1, 2, 3, 5, 16, 32])
def test_greedy_early_exit_equals_every_row(B):
    b = psi_inputs.linear_batch(psi_inputs.LinearConfig("g", MIN_N, B, 30011, "bf16", 0.0, 1.0,
                                                        B, 1, "zipf", 0.6), device="cuda")
    early, full = _greedy_raw(b, False), _greedy_raw(b, True)
    for x, y in zip(early, full):
        assert np.array_equal(x, y)
    o = oracle_linear(b, 0, 0)
    assert np.array_equal(early[0], o["tokens"]) and np.array_equal(early[1], o["n_emitted"])


def test_greedy_early_exit_full_size():
    cfg = CFG["max_batch_greedy"]
    b = psi_inputs.linear_batch(cfg, device="cuda")
    early, full = _greedy_raw(b, False), _greedy_raw(b, True)
    for x, y in zip(early, full):
        assert np.array_equal(x, y)
    o = oracle_linear(b, 0, 0)  # T = 0: the seed and step do not matter
    assert np.array_equal(early[0], o["tokens"]) and np.array_equal(early[1], o["n_emitted"])
    assert early[2] == o["status"] == 0
