"""psi_verify_linear_noalloc (the entry point without a caller workspace):
called through the C ABI twice in a row, it must give the same results as
psi_verify_linear with a workspace, bit for bit.  This file is collected
last, so it also runs after every other GPU test in the same process."""
import numpy as np
import pytest
import torch

import psi_inputs
import rejection_sampling_verify_b200 as psi

pytestmark = pytest.mark.gpu

CFG = psi_inputs.CONFIGS


def _ptr(t):
    return 0 if t is None else t.data_ptr()


def _outputs(N, B, probs):
    dev = "cuda"
    return dict(tokens=torch.full((N, B + 1), -7, dtype=torch.int32, device=dev),
                n=torch.zeros(N, dtype=torch.int32, device=dev),
                p=torch.full((N, B), -1.0, device=dev) if probs else None,
                q=torch.full((N, B), -1.0, device=dev) if probs else None,
                status=torch.zeros(1, dtype=torch.int32, device=dev))


def _args(b, T, top_p, seed, step, seq_ids, o):
    N, B1, V = b.ar.shape
    code = psi.PSI_DTYPE_BF16 if b.ar.dtype == torch.bfloat16 else psi.PSI_DTYPE_F32
    draft = None if T == 0 else b.draft
    return [_ptr(b.ar), V, _ptr(draft), V, code, _ptr(b.ids), N, B1 - 1, V, float(T),
            float(top_p), seed, _ptr(seq_ids), step, _ptr(o["tokens"]), _ptr(o["n"]),
            _ptr(o["p"]), _ptr(o["q"]), _ptr(o["status"])]


def _host(o):
    return {k: v.cpu().numpy() for k, v in o.items() if v is not None}


def _run_both(b, T, top_p, seed, step, seq_ids=None):
    N, B1, V = b.ar.shape
    B = B1 - 1
    probs = T > 0
    # reference: the entry point with a caller-owned workspace
    ref = _outputs(N, B, probs)
    code = psi.PSI_DTYPE_BF16 if b.ar.dtype == torch.bfloat16 else psi.PSI_DTYPE_F32
    ws_bytes = psi.psi_verify_linear_workspace_bytes(N, B, V, code, float(T), float(top_p))
    assert 0 < ws_bytes <= psi.PSI_NOALLOC_SCRATCH_BYTES
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    st = psi.psi_verify_linear(*_args(b, T, top_p, seed, step, seq_ids, ref), _ptr(ws), ws_bytes, 0)
    assert st == psi.PSI_OK, psi.psi_last_error()
    runs = []
    for _ in range(2):  # two calls in a row reuse the same scratch
        o = _outputs(N, B, probs)
        st = psi.psi_verify_linear_noalloc(*_args(b, T, top_p, seed, step, seq_ids, o), 0)
        assert st == psi.PSI_OK, psi.psi_last_error()
        runs.append(o)
    torch.cuda.synchronize()
    want = _host(ref)
    for o in runs:
        got = _host(o)
        assert sorted(got) == sorted(want)
        for k in want:
            assert np.array_equal(got[k], want[k]), k
    return want


def test_noalloc_sampled_nucleus_matches_workspace_entry():
    cfg = CFG["large_batch_nucleus"]
    b = psi_inputs.linear_batch(cfg, device="cuda", N=6, index=1)
    _run_both(b, cfg.temperature, cfg.top_p, cfg.seed, 4)


def test_noalloc_sampled_single_stream_matches_workspace_entry():
    cfg = CFG["single_stream"]
    b = psi_inputs.linear_batch(cfg, device="cuda", N=2, index=0)
    sids = torch.tensor([5, 9], dtype=torch.int64, device="cuda")
    _run_both(b, cfg.temperature, cfg.top_p, cfg.seed, 1, seq_ids=sids)


def test_noalloc_float32_without_top_p_matches_workspace_entry():
    cfg = psi_inputs.LinearConfig("flat", 3, 5, 3000, "f32", 0.8, 1.0, 11, 1, "tiny", 1.0)
    b = psi_inputs.linear_batch(cfg, device="cuda")
    _run_both(b, cfg.temperature, cfg.top_p, 2, 7)


def test_noalloc_greedy_matches_workspace_entry():
    cfg = CFG["max_batch_greedy"]
    b = psi_inputs.linear_batch(cfg, device="cuda", N=16, index=0)
    _run_both(b, 0.0, 1.0, 0, 0)


def test_noalloc_greedy_early_exit_rounds_match_workspace_entry():
    """128 sequences take the greedy early-exit rounds, whose partials, row
    lists, counters and active flags then live in the library's scratch."""
    cfg = CFG["max_batch_greedy"]
    b = psi_inputs.linear_batch(cfg, device="cuda", N=128, index=1)
    assert b.ar.shape[0] >= psi.PSI_EARLY_EXIT_MIN_N
    _run_both(b, 0.0, 1.0, 0, 0)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # 600 sequences of 17 rows need far more than the scratch holds (the
    # sampled path keeps a candidate list per row); nothing is launched
    N, B, V = 600, 8, 64
    code = psi.PSI_DTYPE_BF16
    assert psi.psi_verify_linear_workspace_bytes(N, B, V, code, 1.0, 0.9) > \
        psi.PSI_NOALLOC_SCRATCH_BYTES
    ar = torch.zeros(N, B + 1, V, dtype=torch.bfloat16, device="cuda")
    draft = torch.zeros(N, B, V, dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros(N, B, dtype=torch.int32, device="cuda")
    b = psi_inputs.LinearBatch(ar, draft, ids, 1.0, 0.9)
    o = _outputs(N, B, True)
    st = psi.psi_verify_linear_noalloc(*_args(b, 1.0, 0.9, 0, 0, None, o), 0)
    assert st == psi.PSI_ERR_UNSUPPORTED
    assert "scratch" in psi.psi_last_error()
    # invalid sizes keep their own status
    st = psi.psi_verify_linear_noalloc(*_args(b, -1.0, 0.9, 0, 0, None, o), 0)
    assert st == psi.PSI_ERR_INVALID_ARG
