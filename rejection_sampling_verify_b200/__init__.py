"""Psi-Spec verify step on NVIDIA B200 (sm_100a): Python binding.

The work happens in ``libpsi_verify.so`` (hand-written CUDA kernels behind a
C ABI, declared in ``include/psi_verify.h``).  This module only marshals
arguments: the raw functions below carry the ABI's names and arguments
one-for-one (device pointers as integers), and the tensor helpers
(:func:`verify_linear`, :func:`verify_tree_greedy`, :func:`rng_uniforms`)
take ``torch`` CUDA tensors, allocate outputs and workspace with torch, and
call the raw functions on the current stream.

There is no fallback: if the library is missing or cannot load, every call
raises.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpsi_verify.so")

# psi_status
PSI_OK = 0
PSI_ERR_INVALID_ARG = 1
PSI_ERR_MISALIGNED = 2
PSI_ERR_UNSUPPORTED = 3
PSI_ERR_CUDA = 4
PSI_ERR_WORKSPACE = 5
PSI_ERR_TIMEOUT = 6
# psi_dtype
PSI_DTYPE_F32 = 0
PSI_DTYPE_BF16 = 1
# device status bits
PSI_DEV_BAD_TOKEN_ID = 1
PSI_DEV_BAD_PARENT = 2
PSI_DEV_NONFINITE = 4
PSI_DEV_TIMEOUT = 8
# RNG purposes
PSI_PURPOSE_ACCEPT = 0
PSI_PURPOSE_RESID = 1
# limits
PSI_MAX_B = 32
PSI_MAX_V = 393216
PSI_MAX_TREE_NODES = 4096
PSI_NOALLOC_SCRATCH_BYTES = 8 << 20
PSI_SAMPLED_ROUND_POSITIONS = 2
PSI_GREEDY_ROUND_POSITIONS = 3
PSI_SAMPLED_SHORT_ROUNDS = 2
PSI_GREEDY_SHORT_ROUNDS = 3
PSI_EARLY_EXIT_MIN_N = 64

EXPORTED = (
    "psi_verify_linear_workspace_bytes",
    "psi_verify_linear",
    "psi_verify_linear_noalloc",
    "psi_verify_linear_topk_workspace_bytes",
    "psi_verify_linear_topk",
    "psi_verify_tree_greedy_workspace_bytes",
    "psi_verify_tree_greedy",
    "psi_verify_tree_sampled_workspace_bytes",
    "psi_verify_tree_sampled",
    "psi_rng_uniforms",
    "psi_profile_main_kernel",
    "psi_status_string",
    "psi_last_error",
)


class PsiError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {psi_status_string(status)} ({psi_last_error()})")


_lib = None


def load_library():
    """Load ``libpsi_verify.so`` (building it first if only sources exist and
    nvcc is available).  Raises if it cannot be loaded."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        from . import build as _build
        _build.build()
    lib = C.CDLL(LIB_PATH)
    vp, i32, i64, u32, u64, f32, sz = (C.c_void_p, C.c_int32, C.c_int64, C.c_uint32,
                                       C.c_uint64, C.c_float, C.c_size_t)
    lib.psi_verify_linear_workspace_bytes.restype = sz
    lib.psi_verify_linear_workspace_bytes.argtypes = [i32, i32, i32, C.c_int, f32, f32]
    lib.psi_verify_linear.restype = C.c_int
    lib.psi_verify_linear.argtypes = [vp, i64, vp, i64, C.c_int, vp, i32, i32, i32, f32, f32,
                                      u64, vp, u64, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.psi_verify_linear_noalloc.restype = C.c_int
    lib.psi_verify_linear_noalloc.argtypes = [vp, i64, vp, i64, C.c_int, vp, i32, i32, i32, f32,
                                              f32, u64, vp, u64, vp, vp, vp, vp, vp, vp]
    lib.psi_verify_linear_topk_workspace_bytes.restype = sz
    lib.psi_verify_linear_topk_workspace_bytes.argtypes = [i32, i32, i32, C.c_int, f32, f32, i32]
    lib.psi_verify_linear_topk.restype = C.c_int
    lib.psi_verify_linear_topk.argtypes = [vp, i64, vp, i64, C.c_int, vp, i32, i32, i32, f32, f32,
                                           i32, u64, vp, u64, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.psi_verify_tree_greedy_workspace_bytes.restype = sz
    lib.psi_verify_tree_greedy_workspace_bytes.argtypes = [i32, i32, i32, C.c_int]
    lib.psi_verify_tree_greedy.restype = C.c_int
    lib.psi_verify_tree_greedy.argtypes = [vp, i64, C.c_int, vp, vp, i32, i32, i32, vp, vp, vp,
                                           vp, vp, sz, vp]
    lib.psi_verify_tree_sampled_workspace_bytes.restype = sz
    lib.psi_verify_tree_sampled_workspace_bytes.argtypes = [i32, i32, i32, C.c_int, f32, f32]
    lib.psi_verify_tree_sampled.restype = C.c_int
    lib.psi_verify_tree_sampled.argtypes = [vp, i64, C.c_int, vp, vp, i32, i32, i32, f32, f32,
                                            u64, vp, u64, vp, vp, vp, vp, vp, sz, vp]
    lib.psi_rng_uniforms.restype = C.c_int
    lib.psi_rng_uniforms.argtypes = [u64, vp, i32, u64, i32, u32, vp, vp]
    lib.psi_profile_main_kernel.restype = C.c_int
    lib.psi_profile_main_kernel.argtypes = [vp, vp]
    lib.psi_status_string.restype = C.c_char_p
    lib.psi_status_string.argtypes = [C.c_int]
    lib.psi_last_error.restype = C.c_char_p
    lib.psi_last_error.argtypes = []
    _lib = lib
    return lib


# ---- raw ABI (device pointers as ints, stream as an int handle) --------------

def psi_status_string(status: int) -> str:
    return load_library().psi_status_string(status).decode()


def psi_last_error() -> str:
    return load_library().psi_last_error().decode()


def psi_verify_linear_workspace_bytes(N, B, V, dtype, temperature, top_p) -> int:
    return int(load_library().psi_verify_linear_workspace_bytes(N, B, V, dtype, temperature,
                                                                top_p))


def psi_verify_linear_topk_workspace_bytes(N, B, V, dtype, temperature, top_p, top_k) -> int:
    return int(load_library().psi_verify_linear_topk_workspace_bytes(N, B, V, dtype, temperature,
                                                                     top_p, top_k))


def psi_verify_linear_topk(ar_logits, ar_row_stride, draft_logits, draft_row_stride, dtype,
                           draft_ids, N, B, V, temperature, top_p, top_k, seed, seq_ids, step,
                           out_tokens, out_n_emitted, out_p_draft, out_q_draft, dev_status,
                           workspace, workspace_bytes, stream) -> int:
    return int(load_library().psi_verify_linear_topk(
        ar_logits, ar_row_stride, draft_logits, draft_row_stride, dtype, draft_ids, N, B, V,
        temperature, top_p, top_k, seed, seq_ids, step, out_tokens, out_n_emitted, out_p_draft,
        out_q_draft, dev_status, workspace, workspace_bytes, stream))


def psi_verify_linear(ar_logits, ar_row_stride, draft_logits, draft_row_stride, dtype,
                      draft_ids, N, B, V, temperature, top_p, seed, seq_ids, step, out_tokens,
                      out_n_emitted, out_p_draft, out_q_draft, dev_status, workspace,
                      workspace_bytes, stream) -> int:
    return int(load_library().psi_verify_linear(
        ar_logits, ar_row_stride, draft_logits, draft_row_stride, dtype, draft_ids, N, B, V,
        temperature, top_p, seed, seq_ids, step, out_tokens, out_n_emitted, out_p_draft,
        out_q_draft, dev_status, workspace, workspace_bytes, stream))


def psi_verify_linear_noalloc(ar_logits, ar_row_stride, draft_logits, draft_row_stride, dtype,
                              draft_ids, N, B, V, temperature, top_p, seed, seq_ids, step,
                              out_tokens, out_n_emitted, out_p_draft, out_q_draft, dev_status,
                              stream) -> int:
    return int(load_library().psi_verify_linear_noalloc(
        ar_logits, ar_row_stride, draft_logits, draft_row_stride, dtype, draft_ids, N, B, V,
        temperature, top_p, seed, seq_ids, step, out_tokens, out_n_emitted, out_p_draft,
        out_q_draft, dev_status, stream))


def psi_verify_tree_greedy_workspace_bytes(N, M, V, dtype) -> int:
    return int(load_library().psi_verify_tree_greedy_workspace_bytes(N, M, V, dtype))


def psi_verify_tree_greedy(ar_logits, ar_row_stride, dtype, node_tokens, parents, N, M, V,
                           out_path_nodes, out_path_len, out_tokens, dev_status, workspace,
                           workspace_bytes, stream) -> int:
    return int(load_library().psi_verify_tree_greedy(
        ar_logits, ar_row_stride, dtype, node_tokens, parents, N, M, V, out_path_nodes,
        out_path_len, out_tokens, dev_status, workspace, workspace_bytes, stream))


def psi_verify_tree_sampled_workspace_bytes(N, M, V, dtype, temperature, top_p) -> int:
    return int(load_library().psi_verify_tree_sampled_workspace_bytes(N, M, V, dtype,
                                                                      temperature, top_p))


def psi_verify_tree_sampled(ar_logits, ar_row_stride, dtype, node_tokens, parents, N, M, V,
                            temperature, top_p, seed, seq_ids, step, out_path_nodes,
                            out_path_len, out_tokens, dev_status, workspace, workspace_bytes,
                            stream) -> int:
    return int(load_library().psi_verify_tree_sampled(
        ar_logits, ar_row_stride, dtype, node_tokens, parents, N, M, V, temperature, top_p,
        seed, seq_ids, step, out_path_nodes, out_path_len, out_tokens, dev_status, workspace,
        workspace_bytes, stream))


def psi_rng_uniforms(seed, seq_ids, n_seq, step, n_rows, purpose, out, stream) -> int:
    return int(load_library().psi_rng_uniforms(seed, seq_ids, n_seq, step, n_rows, purpose, out,
                                               stream))


def psi_profile_main_kernel(before, after) -> int:
    """before/after: cudaEvent_t handles as ints (torch.cuda.Event.cuda_event),
    or None, None to stop."""
    return int(load_library().psi_profile_main_kernel(before, after))


# ---- torch tensor helpers --------------------------------------------------------

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return PSI_DTYPE_BF16
    if t.dtype == torch.float32:
        return PSI_DTYPE_F32
    raise TypeError(f"logits must be bfloat16 or float32, got {t.dtype}")


def _rows(t, lead: int, name: str):
    """(row stride in elements, V) of a [..., V] tensor whose rows are evenly
    spaced (contiguous last dim)."""
    if t.dim() != lead + 1 or t.stride(-1) != 1:
        raise ValueError(f"{name}: expected {lead + 1} dims with a contiguous last dim")
    stride = t.stride(-2)
    for d in range(lead - 1):
        if t.stride(d) != t.stride(d + 1) * t.shape[d + 1]:
            raise ValueError(f"{name}: rows must be evenly spaced")
    return stride, t.shape[-1]


def _ptr(t):
    return None if t is None else t.data_ptr()


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _check_out(name, t, dtype, shape, optional=False):
    """A caller-supplied output buffer must match what the kernels write."""
    if t is None:
        if optional:
            return
        raise ValueError(f"out.{name} is required")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"out.{name} must be a contiguous {dtype} tensor of shape "
                         f"{tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


def _check_seq_ids(t, n):
    """Sequence ids: n 64-bit integers (the kernels read them as uint64)."""
    torch = _torch()
    if t is None:
        return
    if t.dtype not in (torch.int64, torch.uint64) or tuple(t.shape) != (n,) or not t.is_contiguous():
        raise ValueError(f"seq_ids must be a contiguous 64-bit integer tensor of shape ({n},), "
                         f"got {t.dtype} {tuple(t.shape)}")


def _check_workspace(t):
    if t is not None and not t.is_contiguous():
        raise ValueError("workspace must be contiguous")


def _device_of(ref, **tensors):
    """The CUDA device of `ref`, after checking that every other given tensor
    is on it and that it is the current device (the library launches on the
    current device and stream; it has no CPU path)."""
    torch = _torch()
    dev = ref.device
    if dev.type != "cuda":
        raise ValueError(f"tensors must be CUDA tensors (got {dev}): the library has no CPU path")
    for name, t in tensors.items():
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the logits on {dev}")
    cur = torch.cuda.current_device()
    if dev.index != cur:
        raise ValueError(f"the tensors are on {dev} but the current device is cuda:{cur}; "
                         f"call under torch.cuda.device({dev.index})")
    return dev


def _stream(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check(status, where):
    if status != PSI_OK:
        raise PsiError(status, where)


@dataclass
class LinearResult:
    tokens: "torch.Tensor"      # int32 [N, B+1]
    n_emitted: "torch.Tensor"   # int32 [N]
    p_draft: "torch.Tensor | None"  # float32 [N, B]
    q_draft: "torch.Tensor | None"
    status: "torch.Tensor"      # uint32-as-int32 [1] device status word


def verify_linear(ar, draft, ids, temperature: float, top_p: float = 1.0, seed: int = 0,
                  step: int = 0, seq_ids=None, want_probs: bool = True, workspace=None,
                  stream=None, out: LinearResult | None = None, top_k: int = 0) -> LinearResult:
    """Linear verify of a batch (see ``psi_verify_linear`` in the header; with
    ``top_k`` != 0, ``psi_verify_linear_topk``).

    ar [N, B+1, V], draft [N, B, V] (may be None when temperature == 0),
    ids int32 [N, B], seq_ids uint64-as-int64 [N] or None; CUDA tensors.

    With ``out`` and a large enough ``workspace`` passed in, the call only
    launches work on the stream, so it can be captured into a CUDA graph
    (after one call on the device outside capture).  seed and step are then
    fixed in the graph.
    """
    torch = _torch()
    N, B1 = ar.shape[0], ar.shape[1]
    B = B1 - 1
    ar_stride, V = _rows(ar, 2, "ar")
    code = _dtype_code(ar)
    greedy = temperature == 0
    if draft is not None and not greedy:
        if draft.dtype != ar.dtype or tuple(draft.shape[:2]) != (N, B) or draft.shape[-1] != V:
            raise ValueError("draft must be [N, B, V] with the AR dtype")
        dr_stride, _ = _rows(draft, 2, "draft")
    else:
        dr_stride = ar_stride
    if ids.dtype != torch.int32 or tuple(ids.shape) != (N, B) or not ids.is_contiguous():
        raise ValueError("ids must be a contiguous int32 [N, B] tensor")
    _check_seq_ids(seq_ids, N)
    if out is not None:
        _check_out("tokens", out.tokens, torch.int32, (N, B + 1))
        _check_out("n_emitted", out.n_emitted, torch.int32, (N,))
        _check_out("p_draft", out.p_draft, torch.float32, (N, B), optional=True)
        _check_out("q_draft", out.q_draft, torch.float32, (N, B), optional=True)
        _check_out("status", out.status, torch.int32, (1,))
    _check_workspace(workspace)
    dev = _device_of(ar, draft=None if greedy else draft, ids=ids, seq_ids=seq_ids,
                     workspace=workspace,
                     **({} if out is None else dict(tokens=out.tokens, n_emitted=out.n_emitted,
                                                    p_draft=out.p_draft, q_draft=out.q_draft,
                                                    status=out.status)))
    if out is None:
        out = LinearResult(
            torch.empty(N, B + 1, dtype=torch.int32, device=dev),
            torch.empty(N, dtype=torch.int32, device=dev),
            torch.empty(N, B, dtype=torch.float32, device=dev) if want_probs and not greedy else None,
            torch.empty(N, B, dtype=torch.float32, device=dev) if want_probs and not greedy else None,
            torch.zeros(1, dtype=torch.int32, device=dev))
    ws_bytes = psi_verify_linear_workspace_bytes(N, B, V, code, float(temperature), float(top_p))
    if ws_bytes == 0:  # invalid sizes: let the ABI report the precise status
        workspace = None
    elif workspace is None or _nbytes(workspace) < ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    if top_k:
        st = psi_verify_linear_topk(
            _ptr(ar), ar_stride, None if greedy else _ptr(draft), dr_stride, code, _ptr(ids), N,
            B, V, float(temperature), float(top_p), int(top_k), int(seed) & (2**64 - 1),
            _ptr(seq_ids), int(step) & (2**64 - 1), _ptr(out.tokens), _ptr(out.n_emitted),
            _ptr(out.p_draft), _ptr(out.q_draft), _ptr(out.status), _ptr(workspace),
            _nbytes(workspace), _stream(stream))
        _check(st, "psi_verify_linear_topk")
        return out
    st = psi_verify_linear(
        _ptr(ar), ar_stride, None if greedy else _ptr(draft), dr_stride, code, _ptr(ids), N, B,
        V, float(temperature), float(top_p), int(seed) & (2**64 - 1),
        _ptr(seq_ids), int(step) & (2**64 - 1), _ptr(out.tokens), _ptr(out.n_emitted),
        _ptr(out.p_draft), _ptr(out.q_draft), _ptr(out.status), _ptr(workspace),
        _nbytes(workspace), _stream(stream))
    _check(st, "psi_verify_linear")
    return out


@dataclass
class TreeResult:
    path_nodes: "torch.Tensor"  # int32 [N, M]
    path_len: "torch.Tensor"    # int32 [N]
    tokens: "torch.Tensor"      # int32 [N, M+1]
    status: "torch.Tensor"


def verify_tree_greedy(ar, node_tokens, parents, workspace=None, stream=None,
                       out: TreeResult | None = None) -> TreeResult:
    """Greedy tree verify.  ar [N, M+1, V]; node_tokens, parents int32 [N, M]."""
    torch = _torch()
    N, M1 = ar.shape[0], ar.shape[1]
    M = M1 - 1
    stride, V = _rows(ar, 2, "ar")
    code = _dtype_code(ar)
    for name, t in (("node_tokens", node_tokens), ("parents", parents)):
        if t.dtype != torch.int32 or tuple(t.shape) != (N, M) or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous int32 [N, M] tensor")
    if out is not None:
        _check_out("path_nodes", out.path_nodes, torch.int32, (N, M))
        _check_out("path_len", out.path_len, torch.int32, (N,))
        _check_out("tokens", out.tokens, torch.int32, (N, M + 1))
        _check_out("status", out.status, torch.int32, (1,))
    _check_workspace(workspace)
    dev = _device_of(ar, node_tokens=node_tokens, parents=parents, workspace=workspace,
                     **({} if out is None else dict(path_nodes=out.path_nodes,
                                                    path_len=out.path_len, tokens=out.tokens,
                                                    status=out.status)))
    if out is None:
        out = TreeResult(torch.empty(N, M, dtype=torch.int32, device=dev),
                         torch.empty(N, dtype=torch.int32, device=dev),
                         torch.empty(N, M + 1, dtype=torch.int32, device=dev),
                         torch.zeros(1, dtype=torch.int32, device=dev))
    ws_bytes = psi_verify_tree_greedy_workspace_bytes(N, M, V, code)
    if ws_bytes == 0:  # invalid sizes: let the ABI report the precise status
        workspace = None
    elif workspace is None or _nbytes(workspace) < ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = psi_verify_tree_greedy(_ptr(ar), stride, code, _ptr(node_tokens), _ptr(parents), N, M,
                                V, _ptr(out.path_nodes), _ptr(out.path_len), _ptr(out.tokens),
                                _ptr(out.status), _ptr(workspace),
                                _nbytes(workspace), _stream(stream))
    _check(st, "psi_verify_tree_greedy")
    return out


def verify_tree_sampled(ar, node_tokens, parents, temperature: float, top_p: float = 1.0,
                        seed: int = 0, step: int = 0, seq_ids=None, workspace=None, stream=None,
                        out: TreeResult | None = None) -> TreeResult:
    """Sampled tree verify (recursive rejection over each reached node's
    children).  ar [N, M+1, V]; node_tokens, parents int32 [N, M]; seq_ids
    int64 [N] (read as uint64) or None."""
    torch = _torch()
    N, M1 = ar.shape[0], ar.shape[1]
    M = M1 - 1
    stride, V = _rows(ar, 2, "ar")
    code = _dtype_code(ar)
    for name, t in (("node_tokens", node_tokens), ("parents", parents)):
        if t.dtype != torch.int32 or tuple(t.shape) != (N, M) or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous int32 [N, M] tensor")
    if seq_ids is not None:
        _check_seq_ids(seq_ids, N)
    if out is not None:
        _check_out("path_nodes", out.path_nodes, torch.int32, (N, M))
        _check_out("path_len", out.path_len, torch.int32, (N,))
        _check_out("tokens", out.tokens, torch.int32, (N, M + 1))
        _check_out("status", out.status, torch.int32, (1,))
    _check_workspace(workspace)
    dev = _device_of(ar, node_tokens=node_tokens, parents=parents, workspace=workspace,
                     seq_ids=seq_ids,
                     **({} if out is None else dict(path_nodes=out.path_nodes,
                                                    path_len=out.path_len, tokens=out.tokens,
                                                    status=out.status)))
    if out is None:
        out = TreeResult(torch.empty(N, M, dtype=torch.int32, device=dev),
                         torch.empty(N, dtype=torch.int32, device=dev),
                         torch.empty(N, M + 1, dtype=torch.int32, device=dev),
                         torch.zeros(1, dtype=torch.int32, device=dev))
    ws_bytes = psi_verify_tree_sampled_workspace_bytes(N, M, V, code, float(temperature),
                                                       float(top_p))
    if ws_bytes == 0:  # invalid sizes: let the ABI report the precise status
        workspace = None
    elif workspace is None or _nbytes(workspace) < ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = psi_verify_tree_sampled(_ptr(ar), stride, code, _ptr(node_tokens), _ptr(parents), N, M,
                                 V, float(temperature), float(top_p), int(seed) & (2**64 - 1),
                                 _ptr(seq_ids), int(step) & (2**64 - 1), _ptr(out.path_nodes),
                                 _ptr(out.path_len), _ptr(out.tokens), _ptr(out.status),
                                 _ptr(workspace), _nbytes(workspace), _stream(stream))
    _check(st, "psi_verify_tree_sampled")
    return out


def rng_uniforms(seed: int, n_seq: int, step: int, n_rows: int, purpose: int, seq_ids=None,
                 device="cuda", stream=None):
    """float32 [n_seq, n_rows] of the verify step's uniforms."""
    torch = _torch()
    if torch.device(device).type != "cuda":
        raise ValueError(f"device must be a CUDA device (got {device}): the library has no CPU path")
    _check_seq_ids(seq_ids, n_seq)
    out = torch.empty(n_seq, n_rows, dtype=torch.float32, device=device)
    _device_of(out, seq_ids=seq_ids)
    st = psi_rng_uniforms(int(seed) & (2**64 - 1), _ptr(seq_ids), n_seq, int(step) & (2**64 - 1),
                          n_rows, purpose, _ptr(out), _stream(stream))
    _check(st, "psi_rng_uniforms")
    return out


__all__ = [n for n in dir() if n.startswith(("psi_", "PSI_"))] + [
    "verify_linear", "verify_tree_greedy", "rng_uniforms", "LinearResult", "TreeResult",
    "PsiError", "load_library", "EXPORTED", "verify_tree_sampled"]
