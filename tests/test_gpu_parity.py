"""GPU parity: the CUDA library (called through its C ABI) against the CPU
oracle on the same seeded inputs.

Greedy and tree paths: token ids, lengths and paths bit-exact.  Sampled
path: p(x) and q(x) within 1e-5; tokens and lengths identical except on
near-tie steps (the oracle's margin < 1e-5), which are counted.
"""
import numpy as np
import pytest
import torch

import oracle
import psi_inputs
import rejection_sampling_verify_b200 as psi
from helpers import (assert_linear_parity, assert_tree_parity, gpu_linear, gpu_tree,
                     oracle_linear, oracle_tree)

pytestmark = pytest.mark.gpu
CFG = psi_inputs.CONFIGS


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    yield


def _batch(ar, draft, ids, T, top_p):
    return psi_inputs.LinearBatch(ar, draft, ids, T, top_p)


# ---- counter RNG ----------------------------------------------------------------

@pytest.mark.parametrize("seed,step,purpose", [(0, 0, 0), (1, 7, 1), (2**63 + 5, 2**40 + 3, 0)])
def test_rng_bit_exact(seed, step, purpose):
    g = psi.rng_uniforms(seed, 64, step, 33, purpose).cpu().numpy().astype(np.float64)
    o = oracle.uniforms(seed, range(64), step, 33, purpose)
    assert np.array_equal(g, o)


def test_rng_seq_ids_bit_exact():
    sids = np.array([0, 1, 12345, 2**40, 2**63 - 1, 2**63, 2**64 - 1], dtype=np.uint64)
    t = torch.as_tensor(sids.view(np.int64), device="cuda")
    g = psi.rng_uniforms(99, len(sids), 4, 9, 1, seq_ids=t).cpu().numpy().astype(np.float64)
    o = oracle.uniforms(99, [int(s) for s in sids], 4, 9, 1)
    assert np.array_equal(g, o)


# ---- greedy linear ---------------------------------------------------------------

def test_greedy_max_batch_recipe_reduced():
    b = psi_inputs.linear_batch(CFG["max_batch_greedy"], device="cuda", N=48)
    assert_linear_parity(gpu_linear(b, 3, 0), oracle_linear(b, 3, 0), exact=True)


def test_greedy_ties_lowest_index():
    rng = np.random.default_rng(1)
    N, B, V = 16, 8, 5000
    ar = torch.tensor(rng.integers(0, 3, (N, B + 1, V)), dtype=torch.bfloat16)
    ids = torch.zeros(N, B, dtype=torch.int32)
    # half the rows: draft id = first maximal index (accepted), others: a later tie
    for n in range(N):
        for i in range(B):
            row = ar[n, i].float().numpy()
            ties = np.nonzero(row == row.max())[0]
            ids[n, i] = int(ties[0] if (n + i) % 3 else ties[-1])
    b = _batch(ar, None, ids, 0.0, 1.0)
    g, o = gpu_linear(b, 0, 0), oracle_linear(b, 0, 0)
    assert_linear_parity(g, o, exact=True)
    assert o["n_emitted"].min() < B + 1  # some later ties were rejected


@pytest.mark.parametrize("V", [1, 7, 100, 4099, 65537])
@pytest.mark.parametrize("B", [1, 5, 32])
@pytest.mark.parametrize("dtype,pad", [("bf16", 0), ("bf16", 3), ("f32", 0), ("f32", 1)])
def test_greedy_shapes(V, B, dtype, pad):
    """Ragged vocabularies, every block size, padded (and misaligned) rows."""
    g = torch.Generator().manual_seed(V * 131 + B)
    N = 3
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    full = torch.randn(N, B + 1, V + pad, generator=g).to(tdt)
    noisy = full[:, :B, :V].float() + 0.3 * torch.randn(N, B, V, generator=g)
    ids = torch.argmax(noisy, -1).to(torch.int32).contiguous()
    full_dev = full.cuda()
    b = _batch(full_dev[..., :V], None, ids, 0.0, 1.0)  # row stride V + pad on the device
    go = gpu_linear(b, 0, 0)
    oo = oracle.verify_linear(psi_inputs.to_host_logits(full), None, ids.numpy(), 0.0, 1.0, 0, 0,
                              V=V)
    assert_linear_parity(go, oo, exact=True)


def test_greedy_flags_and_neg_inf():
    N, B, V = 4, 3, 300
    ar = torch.randn(N, B + 1, V).to(torch.bfloat16)
    ar[0, 1, 5] = float("-inf")           # allowed
    ar[1, 2, :] = float("-inf")           # all -inf row: argmax 0
    ar[2, 0, 7] = float("nan")
    ar[3, 3, 9] = float("inf")
    ids = torch.argmax(ar[:, :B].float(), -1).to(torch.int32)
    ids[0, 2] = V + 5                      # invalid id
    b = _batch(ar, None, ids, 0.0, 1.0)
    g, o = gpu_linear(b, 0, 0), oracle_linear(b, 0, 0)
    assert o["status"] == oracle.BAD_TOKEN_ID | oracle.NONFINITE
    assert g["status"] == o["status"]
    ok = np.array([True, True, False, False])  # NaN/+inf rows are undefined
    assert np.array_equal(g["tokens"][ok], o["tokens"][ok])
    assert np.array_equal(g["n_emitted"][ok], o["n_emitted"][ok])


# ---- greedy tree -------------------------------------------------------------------

@pytest.mark.parametrize("iid", [False, True])
def test_tree_recipe_full_size(iid):
    cfg = CFG["tree_greedy"]
    if iid:
        cfg = psi_inputs.TreeConfig(**{**cfg.__dict__, "iid": True})
    tb = psi_inputs.tree_batch(cfg, device="cuda")
    g, o = gpu_tree(tb), oracle_tree(tb)
    assert_tree_parity(g, o)
    if not iid:
        assert o["path_len"].max() >= 2  # the recipe produces real matches


def test_tree_handmade_and_flags():
    V = 6

    def rows(am):
        r = torch.zeros(len(am), V)
        for j, a in enumerate(am):
            r[j, a] = 2.0
        return r

    cases = [([1, 3, 0, 5], [1, 3, 0], [-1, 0, 1]),
             ([2, 0, 1, 4, 5], [5, 1, 2, 2], [-1, -1, -1, -1]),
             ([4, 1, 1, 0, 5], [4, 4, 1, 1], [-1, -1, 0, 1]),
             ([4, 1, 3, 2], [4, 1, 9], [-1, 0, 1]),       # bad token
             ([4, 1, 3, 2], [4, 1, 3], [-1, 2, 1])]       # bad parent
    for am, tok, par in cases:
        tb = psi_inputs.TreeBatch(rows(am)[None].to(torch.bfloat16).contiguous(),
                                  torch.tensor([tok], dtype=torch.int32),
                                  torch.tensor([par], dtype=torch.int32), None)
        assert_tree_parity(gpu_tree(tb), oracle_tree(tb))


@pytest.mark.parametrize("N", [1, 40, 100, 200])
def test_tree_cluster_sizes(N):
    """The walk's cluster shrinks as the batch grows (8, 4, 2, 1 CTAs per tree
    on 148 SMs); an odd vocabulary leaves a ragged last chunk."""
    cfg = psi_inputs.TreeConfig(**{**CFG["tree_greedy"].__dict__, "N": N, "V": 5003})
    tb = psi_inputs.tree_batch(cfg, device="cuda", index=N)
    assert_tree_parity(gpu_tree(tb), oracle_tree(tb))


def test_tree_status_covers_the_rows_read():
    """Only the root's and the matched nodes' rows are read: a NaN in an
    unmatched node's row leaves the status clear, one in a matched node's row
    sets it.  Tokens and paths equal the oracle's either way."""
    V = 6

    def batch(nan_row):
        r = torch.zeros(4, V)
        for j, a in enumerate([1, 3, 0, 5]):
            r[j, a] = 2.0
        r[nan_row, 4] = float("nan")
        # node 0 (token 1) matches the root's argmax, node 1 (token 2) does not;
        # node 2 (token 3) is node 0's child and matches
        return psi_inputs.TreeBatch(r[None].contiguous(), torch.tensor([[1, 2, 3]], dtype=torch.int32),
                                    torch.tensor([[-1, -1, 0]], dtype=torch.int32), None)

    for nan_row, read in ((2, False), (1, True)):
        tb = batch(nan_row)
        g, o = gpu_tree(tb), oracle_tree(tb)
        for k in ("path_nodes", "path_len", "tokens"):
            assert np.array_equal(g[k], o[k]), k
        assert o["status"] == oracle.NONFINITE
        assert g["status"] == (oracle.NONFINITE if read else 0), (nan_row, g["status"])


def test_tree_max_nodes():
    """PSI_MAX_TREE_NODES nodes per tree (the walk's largest shared-memory
    footprint), deep random trees and a 2-token vocabulary, so that many
    nodes match and long matched paths occur."""
    rng = np.random.default_rng(9)
    N, M, V = 2, psi.PSI_MAX_TREE_NODES, 2
    par = np.array([[rng.integers(max(-1, k - 8), k) for k in range(M)] for _ in range(N)],
                   dtype=np.int32)
    ar = torch.tensor(rng.integers(0, 6, (N, M + 1, V)), dtype=torch.float32)
    tok = rng.integers(0, V, (N, M)).astype(np.int32)
    tb = psi_inputs.TreeBatch(ar, torch.tensor(tok), torch.tensor(par), None)
    g, o = gpu_tree(tb), oracle_tree(tb)
    assert_tree_parity(g, o)
    assert o["path_len"].max() >= 4


def test_tree_large_random():
    """Many nodes (M = 2000), random valid parents, small vocabulary so that
    matches are frequent."""
    rng = np.random.default_rng(4)
    N, M, V = 3, 2000, 3
    par = np.array([[rng.integers(-1, k) for k in range(M)] for _ in range(N)], dtype=np.int32)
    ar = torch.tensor(rng.integers(0, 4, (N, M + 1, V)), dtype=torch.float32)
    tok = rng.integers(0, V, (N, M)).astype(np.int32)
    tb = psi_inputs.TreeBatch(ar, torch.tensor(tok), torch.tensor(par), None)
    g, o = gpu_tree(tb), oracle_tree(tb)
    assert_tree_parity(g, o)
    assert o["path_len"].max() >= 3


# ---- sampled linear ------------------------------------------------------------------

def test_sampled_tiny_recipe_10k_draws():
    """The tiny recipe (V=32, B=4, float32, T=1): 10,000 independent steps,
    run as 1,000 sequences x 10 steps."""
    cfg = CFG["tiny"]
    base = psi_inputs.linear_batch(cfg, device="cpu")
    n = 1000
    rng = np.random.default_rng(0)
    q = torch.softmax(base.draft[0].double(), -1).numpy()
    near = total = 0
    for step in range(10):
        ids = np.stack([rng.choice(cfg.V, size=n, p=q[i] / q[i].sum()) for i in range(cfg.B)],
                       axis=1).astype(np.int32)
        b = _batch(base.ar.expand(n, -1, -1).contiguous(), base.draft.expand(n, -1, -1).contiguous(),
                   torch.tensor(ids), cfg.temperature, cfg.top_p)
        g, o = gpu_linear(b, cfg.seed, step), oracle_linear(b, cfg.seed, step)
        near += assert_linear_parity(g, o)
        total += n
    assert near <= 0.001 * total, (near, total)


@pytest.mark.parametrize("step", range(6))
def test_sampled_single_stream_recipe(step):
    cfg = CFG["single_stream"]
    b = psi_inputs.linear_batch(cfg, device="cuda", index=step // 3)
    assert_linear_parity(gpu_linear(b, cfg.seed, step), oracle_linear(b, cfg.seed, step))


@pytest.mark.parametrize("step", range(3))
def test_sampled_nucleus_recipe_reduced(step):
    cfg = CFG["large_batch_nucleus"]
    b = psi_inputs.linear_batch(cfg, device="cuda", N=8, index=step)
    assert_linear_parity(gpu_linear(b, cfg.seed, step), oracle_linear(b, cfg.seed, step))


@pytest.mark.parametrize("V", [1, 2, 33, 1000, 12289, 16384, 16392, 65537, 151936])
@pytest.mark.parametrize("top_p", [1.0, 0.9])
def test_sampled_shapes_bf16(V, top_p):
    rng = torch.Generator().manual_seed(V + int(top_p * 10))
    N, B = 3, 4
    ar = (2.0 * torch.randn(N, B + 1, V, generator=rng)).to(torch.bfloat16)
    draft = (ar[:, :B].float() + torch.randn(N, B, V, generator=rng)).to(torch.bfloat16)
    ids = psi_inputs.gumbel_max(draft, 1.3, rng)
    b = _batch(ar, draft, ids, 1.3, top_p)
    assert_linear_parity(gpu_linear(b, 11, V), oracle_linear(b, 11, V))


@pytest.mark.parametrize("B", [1, 32])
@pytest.mark.parametrize("T", [0.05, 5.0])
def test_sampled_block_sizes_and_temperatures(B, T):
    rng = torch.Generator().manual_seed(B * 7 + int(T * 100))
    N, V = 2, 5003
    ar = (1.5 * torch.randn(N, B + 1, V, generator=rng)).to(torch.bfloat16)
    draft = (ar[:, :B].float() + 0.3 * torch.randn(N, B, V, generator=rng)).to(torch.bfloat16)
    ids = psi_inputs.gumbel_max(draft, T, rng)
    for top_p in (1.0, 0.8):
        b = _batch(ar, draft, ids, T, top_p)
        assert_linear_parity(gpu_linear(b, 5, 1), oracle_linear(b, 5, 1))


@pytest.mark.parametrize("V,pad", [(1001, 0), (1001, 1), (40000, 3), (3, 1)])
def test_sampled_float32_and_unaligned_rows(V, pad):
    rng = torch.Generator().manual_seed(V + pad)
    N, B = 3, 3
    full_ar = 2.0 * torch.randn(N, B + 1, V + pad, generator=rng)
    full_dr = full_ar[:, :B] + torch.randn(N, B, V + pad, generator=rng)
    ids = psi_inputs.gumbel_max(full_dr[..., :V].contiguous(), 1.0, rng)
    ar_dev, dr_dev = full_ar.cuda(), full_dr.cuda()
    for top_p in (1.0, 0.7):
        b = _batch(ar_dev[..., :V], dr_dev[..., :V], ids, 1.0, top_p)
        o = oracle.verify_linear(full_ar.numpy(), full_dr.numpy(), ids.numpy(), 1.0, top_p, 2, 0,
                                 V=V)
        assert_linear_parity(gpu_linear(b, 2, 0), o)


def test_sampled_tiny_top_p_is_argmax_group():
    rng = torch.Generator().manual_seed(3)
    N, B, V = 4, 6, 3000
    ar = torch.randn(N, B + 1, V, generator=rng).to(torch.bfloat16)
    draft = (ar[:, :B].float() + 0.2 * torch.randn(N, B, V, generator=rng)).to(torch.bfloat16)
    ids = torch.argmax(draft.float(), -1).to(torch.int32)
    b = _batch(ar, draft, ids, 0.8, 1e-6)
    g, o = gpu_linear(b, 1, 1), oracle_linear(b, 1, 1)
    assert_linear_parity(g, o)


def test_sampled_masked_vocab_and_flags():
    rng = torch.Generator().manual_seed(8)
    N, B, V = 5, 4, 20000
    ar = torch.randn(N, B + 1, V, generator=rng)
    draft = ar[:, :B] + 0.5 * torch.randn(N, B, V, generator=rng)
    ar[:, :, V // 2:] = float("-inf")      # a masked half of the vocabulary
    draft[:, :, V // 2 + 100:] = float("-inf")
    ar, draft = ar.to(torch.bfloat16), draft.to(torch.bfloat16)
    ids = psi_inputs.gumbel_max(draft, 1.0, rng)
    ids[1, 2] = -3                          # invalid id: rejected and flagged
    draft[2, 1, :] = float("-inf")          # an all -inf draft row
    ar[3, 0, 17] = float("nan")             # undefined sequence, flagged
    for top_p in (1.0, 0.9):
        b = _batch(ar, draft, ids, 1.0, top_p)
        g, o = gpu_linear(b, 4, 2), oracle_linear(b, 4, 2)
        assert o["status"] == oracle.BAD_TOKEN_ID | oracle.NONFINITE
        assert g["status"] == o["status"]
        keep = np.array([0, 1, 4])
        gk = {k: (v[keep] if isinstance(v, np.ndarray) else v) for k, v in g.items()}
        ok = {k: (v[keep] if isinstance(v, np.ndarray) else v) for k, v in o.items()}
        assert_linear_parity(gk, ok)
        # the all -inf draft row sequence still emits valid tokens
        assert 1 <= g["n_emitted"][2] <= B + 1 and g["tokens"][2, 0] >= 0


def test_sampled_deterministic_and_batch_invariant():
    cfg = CFG["single_stream"]
    b = psi_inputs.linear_batch(cfg, device="cuda", N=6)
    sids = np.array([10, 11, 12, 13, 14, 15], dtype=np.uint64)
    g1 = gpu_linear(b, 9, 3, seq_ids=sids)
    g2 = gpu_linear(b, 9, 3, seq_ids=sids)
    for k in ("tokens", "n_emitted", "p_draft", "q_draft"):
        assert np.array_equal(g1[k], g2[k])
    pick = np.array([4, 1])
    sub = _batch(b.ar[pick], b.draft[pick], b.ids[pick], cfg.temperature, cfg.top_p)
    g3 = gpu_linear(sub, 9, 3, seq_ids=sids[pick])
    for k in ("tokens", "n_emitted", "p_draft", "q_draft"):
        assert np.array_equal(g1[k][pick], g3[k])


def test_host_argument_errors():
    ar = torch.zeros(2, 3, 10, dtype=torch.bfloat16, device="cuda")
    draft = torch.zeros(2, 2, 10, dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros(2, 2, dtype=torch.int32, device="cuda")
    with pytest.raises(psi.PsiError) as e:
        psi.verify_linear(ar, draft, ids, -1.0, 1.0)
    assert e.value.status == psi.PSI_ERR_INVALID_ARG
    with pytest.raises(psi.PsiError) as e:
        psi.verify_linear(ar, draft, ids, 1.0, 0.0)
    assert e.value.status == psi.PSI_ERR_INVALID_ARG
    big = torch.zeros(1, 2, psi.PSI_MAX_V + 1, dtype=torch.bfloat16, device="cuda")
    big_d = torch.zeros(1, 1, psi.PSI_MAX_V + 1, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(psi.PsiError) as e:
        psi.verify_linear(big, big_d, torch.zeros(1, 1, dtype=torch.int32, device="cuda"), 1.0)
    assert e.value.status == psi.PSI_ERR_UNSUPPORTED


def test_sampled_second_pass_rows():
    """Rows whose top-p mass reaches below the narrow first-pass window (two
    tokens on top, 1500 tokens 2^-13.5 below them, the rest far below): the
    streaming path must settle them on its second pass."""
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
    b = _batch(ar.cuda(), draft.cuda(), ids, 1.0, 0.95)
    assert_linear_parity(gpu_linear(b, 6, 0), oracle_linear(b, 6, 0))


@pytest.mark.parametrize("top_p", [0.9, 1.0])
def test_sampled_general_units_many_per_cluster(top_p):
    """Flat rows (i.i.d. N(0, 2^2) logits at T = 1, V = 40000): nearly every
    element lies within the streaming window, so with top-p every unit goes
    to the cluster kernel's list mode, more units than the list-mode grid
    has clusters (several units per cluster); without top-p every emitting
    row's draw takes the sample mode."""
    cfg = psi_inputs.LinearConfig("flat", 24, 4, 40000, "f32", 1.0, top_p, 31, 1, "tiny", 1.0)
    b = psi_inputs.linear_batch(cfg, device="cuda")
    assert_linear_parity(gpu_linear(b, 3, 1), oracle_linear(b, 3, 1))
