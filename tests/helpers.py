"""Shared helpers for the parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare them."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import psi_inputs

# Probability tolerance of the sampled path (fp32 on the GPU vs double in
# the oracle).
PROB_TOL = 1e-5
# A step whose acceptance ratio, residual CDF or top-p crossing lies within
# this distance of its uniform / threshold is a near tie: the decision may
# legitimately differ between fp32 and double arithmetic.
NEAR_TIE = 1e-5


def gpu_linear(batch: psi_inputs.LinearBatch, seed: int, step: int, seq_ids=None,
               device="cuda", want_probs: bool = True):
    import rejection_sampling_verify_b200 as psi
    ar = batch.ar.to(device)
    draft = batch.draft.to(device) if batch.draft is not None else None
    ids = batch.ids.to(device)
    sid = None if seq_ids is None else torch.as_tensor(np.asarray(seq_ids, dtype=np.uint64).view(np.int64), device=device)
    r = psi.verify_linear(ar, draft, ids, batch.temperature, batch.top_p, seed=seed, step=step,
                          seq_ids=sid, want_probs=want_probs)
    torch.cuda.synchronize()
    out = dict(tokens=r.tokens.cpu().numpy(), n_emitted=r.n_emitted.cpu().numpy(),
               status=int(r.status.item()) & 0xFFFFFFFF)
    if r.p_draft is not None:
        out["p_draft"] = r.p_draft.cpu().numpy().astype(np.float64)
        out["q_draft"] = r.q_draft.cpu().numpy().astype(np.float64)
    return out


def oracle_linear(batch: psi_inputs.LinearBatch, seed: int, step: int, seq_ids=None):
    ar = psi_inputs.to_host_logits(batch.ar)
    draft = None if batch.temperature == 0 else psi_inputs.to_host_logits(batch.draft)
    return oracle.verify_linear_parallel(ar, draft, batch.ids.cpu().numpy(), batch.temperature,
                                         batch.top_p, seed, step, seq_ids=seq_ids)


def compare_linear(g, o, exact: bool = False):
    """Returns (n_sequences, n_near_ties, n_bad, where_bad, n_differ): a
    sequence is bad if its tokens or length differ outside a near tie, or if
    p(x) or q(x) is off by more than PROB_TOL at any drafted position (near
    tie or not)."""
    N = len(o["n_emitted"])
    near = (o["margin"] < NEAR_TIE) if not exact else np.zeros(N, bool)
    differ = (g["n_emitted"] != o["n_emitted"]) | np.any(g["tokens"] != o["tokens"], axis=1)
    bad = differ & ~near
    if "p_draft" in g and not exact:
        dp = np.abs(g["p_draft"] - o["p_draft"]).max(axis=1)
        dq = np.abs(g["q_draft"] - o["q_draft"]).max(axis=1)
        bad |= (dp > PROB_TOL) | (dq > PROB_TOL)
    return N, int(near.sum()), int(bad.sum()), np.nonzero(bad)[0], int(differ.sum())


def assert_linear_parity(g, o, exact: bool = False, max_differ_frac: float = 0.001):
    """Every difference is at a near tie, and the sequences that differ are at
    most max_differ_frac of the batch.  Returns the number of near ties."""
    N, n_near, n_bad, where, n_differ = compare_linear(g, o, exact)
    assert n_bad == 0, (f"{n_bad}/{N} sequences differ outside near ties: {where[:10]}\n"
                        f"gpu n={g['n_emitted'][where[:5]]} oracle n={o['n_emitted'][where[:5]]}\n"
                        f"gpu tok={g['tokens'][where[:2]]}\noracle tok={o['tokens'][where[:2]]}")
    assert g["status"] == o["status"], (g["status"], o["status"])
    assert n_differ <= max_differ_frac * N, (n_differ, N)
    return n_near


def gpu_tree(tb: psi_inputs.TreeBatch, device="cuda"):
    import rejection_sampling_verify_b200 as psi
    r = psi.verify_tree_greedy(tb.ar.to(device), tb.node_tokens.to(device), tb.parents.to(device))
    torch.cuda.synchronize()
    return dict(path_nodes=r.path_nodes.cpu().numpy(), path_len=r.path_len.cpu().numpy(),
                tokens=r.tokens.cpu().numpy(), status=int(r.status.item()) & 0xFFFFFFFF)


def oracle_tree(tb: psi_inputs.TreeBatch):
    return oracle.verify_tree_greedy(psi_inputs.to_host_logits(tb.ar), tb.node_tokens.cpu().numpy(),
                                     tb.parents.cpu().numpy())


def assert_tree_parity(g, o):
    for k in ("path_nodes", "path_len", "tokens"):
        assert np.array_equal(g[k], o[k]), (k, np.nonzero(np.any(np.atleast_2d(g[k] != o[k]), axis=-1)))
    assert g["status"] == o["status"]
