"""Top-k linear verify on the GPU (psi_verify_linear_topk through the C ABI)
against the oracle's top_k on the same seeded inputs.

Reading (the run card names top-k beside top-p): top-k on the temperature
softmax first, ties with the k-th kept, the kept mass renormalised, then
top-p.  The bar is the linear verify's: tokens and lengths identical except
at the oracle's near ties (at most 0.1% of the sequences), p(x) and q(x)
within 1e-5 on every drafted position, the status word equal.

k = 1, 20, 50 are usually settled from the scan's candidates; k = 4000 lies
below the candidate window, so those units take the whole-row top-k path.
"""
import numpy as np
import pytest
import torch

import oracle
import psi_inputs
import rejection_sampling_verify_b200 as psi
from helpers import NEAR_TIE, PROB_TOL

pytestmark = pytest.mark.gpu
CFG = psi_inputs.CONFIGS


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    yield


def _gpu(b, k, seed, step, want_probs, top_p=None, temperature=None):
    T = b.temperature if temperature is None else temperature
    tp = b.top_p if top_p is None else top_p
    r = psi.verify_linear(b.ar.cuda(), b.draft.cuda(), b.ids.cuda(), T, tp, seed=seed, step=step,
                          want_probs=want_probs, top_k=k)
    torch.cuda.synchronize()
    out = dict(tokens=r.tokens.cpu().numpy(), n_emitted=r.n_emitted.cpu().numpy(),
               status=int(r.status.item()) & 0xFFFFFFFF)
    if r.p_draft is not None:
        out["p_draft"] = r.p_draft.cpu().numpy().astype(np.float64)
        out["q_draft"] = r.q_draft.cpu().numpy().astype(np.float64)
    return out


def _oracle(b, k, seed, step, top_p=None, temperature=None):
    T = b.temperature if temperature is None else temperature
    tp = b.top_p if top_p is None else top_p
    return oracle.verify_linear_parallel(psi_inputs.to_host_logits(b.ar),
                                         psi_inputs.to_host_logits(b.draft), b.ids.cpu().numpy(),
                                         T, tp, seed, step, top_k=k)


def _compare(g, o):
    """(sequences, sequences that differ); differences only at near ties,
    probabilities within PROB_TOL everywhere, equal status."""
    near = o["margin"] < NEAR_TIE
    differ = (g["n_emitted"] != o["n_emitted"]) | np.any(g["tokens"] != o["tokens"], axis=1)
    assert not np.any(differ & ~near), np.nonzero(differ & ~near)[0][:10]
    assert g["status"] == o["status"], (g["status"], o["status"])
    if "p_draft" in g:
        dp = np.abs(g["p_draft"] - o["p_draft"])
        dq = np.abs(g["q_draft"] - o["q_draft"])
        worst = float(max(dp.max(), dq.max()))
        assert worst <= PROB_TOL, (worst, np.argwhere((dp > PROB_TOL) | (dq > PROB_TOL))[:5])
    return len(near), int(differ.sum())


@pytest.mark.parametrize("top_p", [1.0, 0.95])
@pytest.mark.parametrize("k", [1, 20, 50, 4000])
def test_topk_nucleus_recipe(k, top_p):
    """The large-batch recipe (V = 151936 bf16, T = 0.7) at N = 64: the
    tokens-only call (early-exit rounds) and the call with p / q."""
    cfg = CFG["large_batch_nucleus"]
    total = differ = 0
    for step, want in ((0, False), (1, True)):
        b = psi_inputs.linear_batch(cfg, device="cuda", index=20 + step, N=64)
        g = _gpu(b, k, cfg.seed, step, want, top_p=top_p)
        o = _oracle(b, k, cfg.seed, step, top_p=top_p)
        n, d = _compare(g, o)
        total, differ = total + n, differ + d
    assert differ <= 0.001 * total + 0.5, (differ, total)


@pytest.mark.parametrize("k", [1, 20, 4000])
def test_topk_single_stream(k):
    """single_stream (N = 8, T = 1, no top-p): one pass over every row."""
    cfg = CFG["single_stream"]
    for step in range(3):
        b = psi_inputs.linear_batch(cfg, device="cuda", index=40 + step)
        _compare(_gpu(b, k, cfg.seed, step, True), _oracle(b, k, cfg.seed, step))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("V", [37, 1000])
def test_topk_ties_and_small_vocabularies(dtype, V):
    """Small vocabularies with many tied logits (ties with the k-th stay),
    k from 1 to past V, with and without top-p, several steps.  V = 37 rows do
    not start on 16-byte boundaries, so every unit takes the whole-row path."""
    g = torch.Generator().manual_seed(V)
    N, B = 16, 4
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    ar = torch.randint(-3, 4, (N, B + 1, V), generator=g).float().to(tdt)   # heavy ties
    draft = (ar[:, :B].float() + torch.randint(-1, 2, (N, B, V), generator=g).float()).to(tdt)
    ids = torch.randint(0, V, (N, B), generator=g, dtype=torch.int32)
    b = psi_inputs.LinearBatch(ar=ar, draft=draft, ids=ids, temperature=1.0, top_p=1.0)
    for k in (1, 2, 5, V - 1, V, V + 3):
        for top_p in (1.0, 0.8):
            for step in range(2):
                gg = _gpu(b, k, 11, step, True, top_p=top_p)
                oo = _oracle(b, k, 11, step, top_p=top_p)
                _compare(gg, oo)


def test_topk_off_is_the_plain_verify():
    """top_k = 0 and top_k >= V give psi_verify_linear's results bit for bit."""
    cfg = CFG["large_batch_nucleus"]
    b = psi_inputs.linear_batch(cfg, device="cuda", index=30, N=64)
    base = psi.verify_linear(b.ar.cuda(), b.draft.cuda(), b.ids.cuda(), b.temperature, b.top_p,
                             seed=3, step=1)
    for k in (0, cfg.V, cfg.V + 10):
        r = psi.verify_linear(b.ar.cuda(), b.draft.cuda(), b.ids.cuda(), b.temperature, b.top_p,
                              seed=3, step=1, top_k=k)
        torch.cuda.synchronize()
        assert torch.equal(r.tokens, base.tokens) and torch.equal(r.n_emitted, base.n_emitted)
        assert torch.equal(r.p_draft, base.p_draft) and torch.equal(r.q_draft, base.q_draft)


def test_topk_negative_is_rejected():
    cfg = CFG["single_stream"]
    b = psi_inputs.linear_batch(cfg, device="cuda", index=0)
    with pytest.raises(psi.PsiError):
        psi.verify_linear(b.ar.cuda(), b.draft.cuda(), b.ids.cuda(), 1.0, 1.0, top_k=-1)
