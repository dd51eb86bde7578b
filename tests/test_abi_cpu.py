"""CPU checks of the C ABI (no GPU needed): the library loads, exports every
function the public header declares, and rejects bad arguments on the host
before launching anything."""
import os
import re

import pytest

import rejection_sampling_verify_b200 as psi

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "psi_verify.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(psi_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    lib = psi.load_library()
    names = declared_functions()
    assert len(names) >= 7, names
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(psi.EXPORTED) == names


def test_header_constants_match_binding():
    text = open(HEADER).read()
    consts = dict(re.findall(r"#define\s+(PSI_[A-Z_]+)\s+(\d+)u?", text))
    for k, v in consts.items():
        assert getattr(psi, k) == int(v), k
    enums = dict(re.findall(r"\b(PSI_[A-Z_0-9]+)\s*=\s*(\d+)", text))
    for k, v in enums.items():
        assert getattr(psi, k) == int(v), k


def test_status_strings():
    for code in range(7):
        assert psi.psi_status_string(code).startswith("PSI_")
    assert psi.psi_status_string(99) == "PSI_ERR_UNKNOWN"


def test_workspace_queries():
    ws = psi.psi_verify_linear_workspace_bytes(256, 8, 151936, psi.PSI_DTYPE_BF16, 0.7, 0.95)
    assert ws >= 256 * 9 * 8 and ws % 256 == 0
    wg = psi.psi_verify_linear_workspace_bytes(1024, 16, 151936, psi.PSI_DTYPE_BF16, 0.0, 1.0)
    assert wg >= 1024 * 17 * 8 and wg % 256 == 0
    assert psi.psi_verify_linear_workspace_bytes(0, 8, 10, 1, 1.0, 1.0) == 0
    assert psi.psi_verify_linear_workspace_bytes(1, 33, 10, 1, 1.0, 1.0) == 0
    assert psi.psi_verify_linear_workspace_bytes(1, 8, psi.PSI_MAX_V + 1, 1, 1.0, 1.0) == 0
    assert psi.psi_verify_linear_workspace_bytes(1, 8, psi.PSI_MAX_V // 2 + 1, 0, 1.0, 1.0) == 0
    assert psi.psi_verify_tree_greedy_workspace_bytes(16, 64, 151936, 1) > 0
    assert psi.psi_verify_tree_greedy_workspace_bytes(16, psi.PSI_MAX_TREE_NODES + 1, 10, 1) == 0


FAKE = 0x10000  # a 64 KB-aligned fake device address: never dereferenced


def _linear(**over):
    args = dict(ar_logits=FAKE, ar_row_stride=100, draft_logits=FAKE, draft_row_stride=100,
                dtype=psi.PSI_DTYPE_BF16, draft_ids=FAKE, N=2, B=4, V=100, temperature=1.0,
                top_p=1.0, seed=0, seq_ids=None, step=0, out_tokens=FAKE, out_n_emitted=FAKE,
                out_p_draft=None, out_q_draft=None, dev_status=None, workspace=FAKE,
                workspace_bytes=1 << 20, stream=None)
    args.update(over)
    return psi.psi_verify_linear(**args)


@pytest.mark.parametrize("over,want", [
    (dict(N=0), psi.PSI_ERR_INVALID_ARG),
    (dict(B=0), psi.PSI_ERR_INVALID_ARG),
    (dict(B=33), psi.PSI_ERR_INVALID_ARG),
    (dict(V=0), psi.PSI_ERR_INVALID_ARG),
    (dict(V=psi.PSI_MAX_V + 1, ar_row_stride=psi.PSI_MAX_V + 1,
          draft_row_stride=psi.PSI_MAX_V + 1), psi.PSI_ERR_UNSUPPORTED),
    (dict(temperature=-0.5), psi.PSI_ERR_INVALID_ARG),
    (dict(temperature=float("nan")), psi.PSI_ERR_INVALID_ARG),
    (dict(temperature=float("inf")), psi.PSI_ERR_INVALID_ARG),
    (dict(top_p=0.0), psi.PSI_ERR_INVALID_ARG),
    (dict(top_p=1.5), psi.PSI_ERR_INVALID_ARG),
    (dict(top_p=float("nan")), psi.PSI_ERR_INVALID_ARG),
    (dict(ar_logits=None), psi.PSI_ERR_INVALID_ARG),
    (dict(draft_logits=None), psi.PSI_ERR_INVALID_ARG),
    (dict(draft_ids=None), psi.PSI_ERR_INVALID_ARG),
    (dict(out_tokens=None), psi.PSI_ERR_INVALID_ARG),
    (dict(ar_row_stride=99), psi.PSI_ERR_INVALID_ARG),
    (dict(dtype=7), psi.PSI_ERR_INVALID_ARG),
    (dict(ar_logits=FAKE + 1), psi.PSI_ERR_MISALIGNED),
    (dict(draft_ids=FAKE + 2), psi.PSI_ERR_MISALIGNED),
    (dict(seq_ids=FAKE + 4), psi.PSI_ERR_MISALIGNED),
    (dict(workspace=None), psi.PSI_ERR_WORKSPACE),
    (dict(workspace_bytes=8), psi.PSI_ERR_WORKSPACE),
])
def test_linear_rejects_bad_arguments_before_launch(over, want):
    assert _linear(**over) == want
    assert psi.psi_last_error()


def test_greedy_allows_null_draft():
    # greedy with a null draft pointer passes validation up to the workspace
    assert _linear(temperature=0.0, draft_logits=None, workspace=None) == psi.PSI_ERR_WORKSPACE


@pytest.mark.parametrize("over,want", [
    (dict(N=0), psi.PSI_ERR_INVALID_ARG),
    (dict(M=0), psi.PSI_ERR_INVALID_ARG),
    (dict(M=psi.PSI_MAX_TREE_NODES + 1), psi.PSI_ERR_INVALID_ARG),
    (dict(parents=None), psi.PSI_ERR_INVALID_ARG),
    (dict(node_tokens=FAKE + 1), psi.PSI_ERR_MISALIGNED),
    (dict(workspace_bytes=0), psi.PSI_ERR_WORKSPACE),
])
def test_tree_rejects_bad_arguments_before_launch(over, want):
    args = dict(ar_logits=FAKE, ar_row_stride=50, dtype=psi.PSI_DTYPE_BF16, node_tokens=FAKE,
                parents=FAKE, N=2, M=8, V=50, out_path_nodes=FAKE, out_path_len=FAKE,
                out_tokens=FAKE, dev_status=None, workspace=FAKE, workspace_bytes=1 << 20,
                stream=None)
    args.update(over)
    assert psi.psi_verify_tree_greedy(**args) == want


def test_rng_rejects_bad_arguments():
    assert psi.psi_rng_uniforms(0, None, 0, 0, 4, 0, FAKE, None) == psi.PSI_ERR_INVALID_ARG
    assert psi.psi_rng_uniforms(0, None, 4, 0, 4, 0, None, None) == psi.PSI_ERR_INVALID_ARG
    assert psi.psi_rng_uniforms(0, None, 4, 0, 4, 0, FAKE + 2, None) == psi.PSI_ERR_MISALIGNED


def test_binding_refuses_tensors_off_the_gpu():
    """The library has no CPU path: host tensors are refused before any
    launch (never handed to a kernel as device pointers)."""
    import torch
    ar = torch.zeros(2, 3, 64, dtype=torch.bfloat16)
    draft = torch.zeros(2, 2, 64, dtype=torch.bfloat16)
    ids = torch.zeros(2, 2, dtype=torch.int32)
    for T in (0.7, 0.0):
        with pytest.raises(ValueError, match="CUDA"):
            psi.verify_linear(ar, draft, ids, T, 0.9)
    tok = torch.zeros(2, 2, dtype=torch.int32)
    par = torch.full((2, 2), -1, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        psi.verify_tree_greedy(ar, tok, par)
    with pytest.raises(ValueError, match="CUDA"):
        psi.rng_uniforms(0, 4, 0, 3, 0, device="cpu")


def test_binding_checks_caller_output_buffers():
    """A caller-supplied `out` must have the shapes and dtypes the kernels
    write (checked before anything else, so a wrong buffer is never written
    past its end)."""
    import torch
    N, B, V = 2, 3, 64
    ar = torch.zeros(N, B + 1, V, dtype=torch.bfloat16)
    draft = torch.zeros(N, B, V, dtype=torch.bfloat16)
    ids = torch.zeros(N, B, dtype=torch.int32)

    def out(tokens=(N, B + 1), n=(N,), pq=(N, B), dt=torch.int32):
        return psi.LinearResult(torch.zeros(tokens, dtype=dt), torch.zeros(n, dtype=torch.int32),
                                torch.zeros(pq), torch.zeros(pq), torch.zeros(1, dtype=torch.int32))

    for bad in (out(tokens=(N, B)), out(n=(N + 1,)), out(pq=(N, B + 1)), out(dt=torch.int64)):
        with pytest.raises(ValueError, match="out\\."):
            psi.verify_linear(ar, draft, ids, 0.7, out=bad)
    with pytest.raises(ValueError, match="CUDA"):  # well-formed buffers reach the device check
        psi.verify_linear(ar, draft, ids, 0.7, out=out())
    M = 4
    tr = psi.TreeResult(torch.zeros(N, M, dtype=torch.int32), torch.zeros(N, dtype=torch.int32),
                        torch.zeros(N, M, dtype=torch.int32), torch.zeros(1, dtype=torch.int32))
    with pytest.raises(ValueError, match="out.tokens"):
        psi.verify_tree_greedy(torch.zeros(N, M + 1, V, dtype=torch.bfloat16),
                               torch.zeros(N, M, dtype=torch.int32),
                               torch.full((N, M), -1, dtype=torch.int32), out=tr)


def test_workspace_size_claims_of_the_header():
    """The header's sizing notes: the sampled path needs about 65.7 KB per
    logit row (N (2B + 1) rows), and the no-allocation scratch fits N <= 7
    sequences at B = 8."""
    for N, B in ((256, 8), (1024, 16), (64, 3)):
        ws = psi.psi_verify_linear_workspace_bytes(N, B, 151936, psi.PSI_DTYPE_BF16, 0.7, 0.95)
        per_row = ws / (N * (2 * B + 1))
        assert 65536 <= per_row <= 66000, (N, B, per_row)
    cap = psi.PSI_NOALLOC_SCRATCH_BYTES
    at = lambda n: psi.psi_verify_linear_workspace_bytes(n, 8, 151936, psi.PSI_DTYPE_BF16, 0.7, 0.95)
    assert at(7) <= cap < at(8)
    # the greedy path needs far less: one packed maximum per (row, split), plus the rounds' lists
    g = psi.psi_verify_linear_workspace_bytes(7, 8, 151936, psi.PSI_DTYPE_BF16, 0.0, 1.0)
    assert g < at(7) // 10


def test_binding_checks_sequence_ids():
    """seq_ids are read as N uint64 values: a short or 32-bit tensor is refused."""
    import torch
    ar = torch.zeros(2, 3, 64, dtype=torch.bfloat16)
    draft = torch.zeros(2, 2, 64, dtype=torch.bfloat16)
    ids = torch.zeros(2, 2, dtype=torch.int32)
    for bad in (torch.zeros(1, dtype=torch.int64), torch.zeros(2, dtype=torch.int32)):
        with pytest.raises(ValueError, match="seq_ids"):
            psi.verify_linear(ar, draft, ids, 0.7, seq_ids=bad)
        with pytest.raises(ValueError, match="seq_ids"):
            psi.rng_uniforms(0, 2, 0, 3, 0, seq_ids=bad)
    with pytest.raises(ValueError, match="CUDA"):  # well-formed ids reach the device check
        psi.verify_linear(ar, draft, ids, 0.7, seq_ids=torch.zeros(2, dtype=torch.int64))
