"""Rows with many candidates: 600-2000 elements within the candidate window
of their maximum (above the 512 a finish warp keeps in registers, up to the
2048 it holds in shared memory), so the top-p and top-k searches and the
draws run on the shared-memory lists; some top-k cuts also fall below the
window and take the whole-row path.  The results must equal the oracle's
(tokens outside near ties, p / q within 1e-5)."""
import numpy as np
import pytest
import torch

import oracle
import psi_inputs
import rejection_sampling_verify_b200 as psi
from helpers import NEAR_TIE, PROB_TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    yield


def _rows(g, n_rows, V, n_near):
    """Each row: n_near elements spread over the 6 logits below its maximum
    (inside the 13 log2-unit window at T = 1), the rest 30 logits lower."""
    x = torch.full((n_rows, V), -30.0)
    x += 0.5 * torch.randn(n_rows, V, generator=g)
    for r in range(n_rows):
        idx = torch.randperm(V, generator=g)[:n_near[r]]
        x[r, idx] = -6.0 * torch.rand(len(idx), generator=g)
    return x


@pytest.mark.parametrize("top_p,top_k", [(0.95, 0), (0.5, 0), (1.0, 1500), (0.9, 1200)])
def test_many_candidates(top_p, top_k):
    g = torch.Generator().manual_seed(100 + top_k)
    N, B, V = 12, 3, 16384
    n_near = [600, 900, 1100, 1400, 1800, 2000] * 2
    ar = _rows(g, N * (B + 1), V, [n_near[i % len(n_near)] for i in range(N * (B + 1))])
    ar = ar.reshape(N, B + 1, V).to(torch.bfloat16)
    draft = (ar[:, :B].float() + 0.3 * torch.randn(N, B, V, generator=g)).to(torch.bfloat16)
    ids = torch.argmax(draft.float() + torch.rand(N, B, V, generator=g).log().neg().log().neg(),
                       dim=-1).to(torch.int32)
    for step in range(3):
        r = psi.verify_linear(ar.cuda(), draft.cuda(), ids.cuda(), 1.0, top_p, seed=9, step=step,
                              top_k=top_k)
        torch.cuda.synchronize()
        o = oracle.verify_linear(psi_inputs.to_host_logits(ar), psi_inputs.to_host_logits(draft),
                                 ids.numpy(), 1.0, top_p, 9, step, top_k=top_k)
        near = o["margin"] < NEAR_TIE
        tok = r.tokens.cpu().numpy()
        n = r.n_emitted.cpu().numpy()
        differ = (n != o["n_emitted"]) | np.any(tok != o["tokens"], axis=1)
        assert not np.any(differ & ~near), np.nonzero(differ & ~near)[0]
        dp = np.abs(r.p_draft.cpu().numpy().astype(np.float64) - o["p_draft"]).max()
        dq = np.abs(r.q_draft.cpu().numpy().astype(np.float64) - o["q_draft"]).max()
        assert max(dp, dq) <= PROB_TOL, (dp, dq)
        assert (int(r.status.item()) & 0xFFFFFFFF) == o["status"]
