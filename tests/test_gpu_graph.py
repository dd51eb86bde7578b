"""CUDA-graph capture of whole verify calls.

Each case captures one call into a graph (after an eager call on the capture
stream, which does the library's once-per-device setup), then replays it on
several input sets copied into the captured buffers.  Every replay must equal
an eager call on the same inputs exactly: the launches, their grids and the
device-side work lists do not depend on the host seeing any data.  seed and
step are plain arguments, captured by value: a replay repeats the step it was
captured with.
"""
import pytest
import torch

import psi_inputs
import rejection_sampling_verify_b200 as psi

pytestmark = pytest.mark.gpu

CFG = psi_inputs.CONFIGS
REPLAYS = 3


def _captured(fn):
    """Run fn once eagerly on a side stream, then capture it; returns the
    graph and what the captured call returned."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out = fn()
    return g, out


def _linear_outputs(N, B, want_probs, dev="cuda"):
    pq = (torch.empty(N, B, dtype=torch.float32, device=dev) if want_probs else None)
    return psi.LinearResult(torch.empty(N, B + 1, dtype=torch.int32, device=dev),
                            torch.empty(N, dtype=torch.int32, device=dev), pq,
                            torch.empty_like(pq) if want_probs else None,
                            torch.zeros(1, dtype=torch.int32, device=dev))


def _check_linear(batches, T, top_p, seed, step, want_probs):
    first = batches[0]
    N, B1, V = first.ar.shape
    B = B1 - 1
    ar = first.ar.clone()
    draft = None if first.draft is None else first.draft.clone()
    ids = first.ids.clone()
    out = _linear_outputs(N, B, want_probs and T > 0)
    ws = torch.empty(max(1, psi.psi_verify_linear_workspace_bytes(
        N, B, V, psi.PSI_DTYPE_BF16 if ar.dtype == torch.bfloat16 else psi.PSI_DTYPE_F32,
        T, top_p)), dtype=torch.uint8, device="cuda")

    def call():
        out.status.zero_()
        return psi.verify_linear(ar, draft, ids, T, top_p, seed=seed, step=step,
                                 want_probs=want_probs, workspace=ws, out=out)

    g, _ = _captured(call)
    for b in batches:
        ar.copy_(b.ar)
        if draft is not None:
            draft.copy_(b.draft)
        ids.copy_(b.ids)
        g.replay()
        eager = psi.verify_linear(b.ar, b.draft, b.ids, T, top_p, seed=seed, step=step,
                                  want_probs=want_probs)
        torch.cuda.synchronize()
        assert torch.equal(out.tokens, eager.tokens)
        assert torch.equal(out.n_emitted, eager.n_emitted)
        assert torch.equal(out.status, eager.status)
        if want_probs and T > 0:
            assert torch.equal(out.p_draft, eager.p_draft)
            assert torch.equal(out.q_draft, eager.q_draft)
    return out


def test_graph_sampled_early_exit_rounds():
    """Tokens only at 64 sequences: the early-exit rounds, whose later rounds
    read only the rows the device lists for them."""
    cfg = CFG["large_batch_nucleus"]
    batches = [psi_inputs.linear_batch(cfg, device="cuda", N=64, V=8192, index=i)
               for i in range(REPLAYS)]
    out = _check_linear(batches, cfg.temperature, cfg.top_p, cfg.seed, 3, want_probs=False)
    assert int(out.n_emitted.min()) >= 1


def test_graph_sampled_every_row_with_probs():
    cfg = CFG["single_stream"]
    batches = [psi_inputs.linear_batch(cfg, device="cuda", V=30011, index=i)
               for i in range(REPLAYS)]
    _check_linear(batches, 0.8, 0.9, 5, 1, want_probs=True)


def test_graph_general_path_units():
    """Flat rows send every unit to the second pass and the cluster kernel;
    how many do varies with the data, the captured launches do not."""
    cfg = psi_inputs.LinearConfig("flat", 64, 4, 40000, "f32", 1.0, 0.9, 31, 1, "tiny", 1.0)
    batches = [psi_inputs.linear_batch(cfg, device="cuda", index=i) for i in range(REPLAYS)]
    _check_linear(batches, 1.0, 0.9, 3, 1, want_probs=False)


def test_graph_greedy_linear_early_exit():
    cfg = CFG["max_batch_greedy"]
    batches = []
    for i in range(REPLAYS):
        b = psi_inputs.linear_batch(cfg, device="cuda", N=64, V=8192, index=i)
        batches.append(psi_inputs.LinearBatch(b.ar, None, b.ids, 0.0, 1.0))
    _check_linear(batches, 0.0, 1.0, 0, 0, want_probs=False)


def test_graph_tree_greedy():
    cfg = CFG["tree_greedy"]
    batches = [psi_inputs.tree_batch(cfg, device="cuda", N=4, index=i) for i in range(REPLAYS)]
    first = batches[0]
    ar, tok, par = first.ar.clone(), first.node_tokens.clone(), first.parents.clone()
    N, M1, V = ar.shape
    M = M1 - 1
    out = psi.TreeResult(torch.empty(N, M, dtype=torch.int32, device="cuda"),
                         torch.empty(N, dtype=torch.int32, device="cuda"),
                         torch.empty(N, M + 1, dtype=torch.int32, device="cuda"),
                         torch.zeros(1, dtype=torch.int32, device="cuda"))
    ws = torch.empty(max(1, psi.psi_verify_tree_greedy_workspace_bytes(
        N, M, V, psi.PSI_DTYPE_BF16)), dtype=torch.uint8, device="cuda")

    def call():
        out.status.zero_()
        return psi.verify_tree_greedy(ar, tok, par, workspace=ws, out=out)

    g, _ = _captured(call)
    for b in batches:
        ar.copy_(b.ar)
        tok.copy_(b.node_tokens)
        par.copy_(b.parents)
        g.replay()
        eager = psi.verify_tree_greedy(b.ar, b.node_tokens, b.parents)
        torch.cuda.synchronize()
        assert torch.equal(out.tokens, eager.tokens)
        assert torch.equal(out.path_len, eager.path_len)
        assert torch.equal(out.path_nodes, eager.path_nodes)
        assert torch.equal(out.status, eager.status)
