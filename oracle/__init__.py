"""Double-precision CPU oracle of the Psi-Spec verify step (ctypes binding).

TEST INFRASTRUCTURE ONLY.  The product library never imports, links or calls
anything here; the tests, ``__graft_entry__.smoke`` and the CPU-baseline leg
of ``bench.py`` are the only users.  The arithmetic lives in ``psi_oracle.c``
(plain C, double precision); this module only marshals numpy arrays.

Logit arrays are numpy ``float32`` (IEEE binary32 rows) or ``uint16``
(raw bfloat16 bit patterns).  Shapes follow the CUDA library: AR logits
``[N, B+1, S]``, draft logits ``[N, B, S]`` with row stride ``S >= V``.

Every function here follows a passage of the method's pages; the citations
are in ``psi_oracle.c``.  Parity status per function:
  - counter RNG, row softmax/top-p, linear sampled verify, greedy linear,
    greedy tree, sampled tree: pinned by the CPU tests in
    ``tests/test_oracle_*.py``;
    ``tests/test_oracle_mutants.py`` plants single mistakes in copies of
    ``psi_oracle.c`` and requires those pins to catch every one.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "psi_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libpsi_oracle.so")

F32 = 0
BF16 = 1
BAD_TOKEN_ID = 1
BAD_PARENT = 2
NONFINITE = 4
PURPOSE_ACCEPT = 0
PURPOSE_RESID = 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math: IEEE double throughout)."""
    up_to_date = (
        os.path.exists(_LIB_PATH)
        and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)
        and os.path.getmtime(_LIB_PATH)
        >= os.path.getmtime(os.path.join(_HERE, "psi_oracle.h"))
    )
    if force or not up_to_date:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra",
             "-fno-fast-math", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _load():
    global _lib
    if _lib is None:
        # PSI_ORACLE_LIB names a prebuilt copy to load instead (the mutation
        # check builds deliberately broken copies and runs the pins on them).
        path = os.environ.get("PSI_ORACLE_LIB") or build()
        lib = C.CDLL(path)
        u64, i64, i32, u32, dbl, vp = (C.c_uint64, C.c_int64, C.c_int32,
                                       C.c_uint32, C.c_double, C.c_void_p)
        lib.orc_splitmix64_mix.restype = u64
        lib.orc_splitmix64_mix.argtypes = [u64]
        lib.orc_counter_hash.restype = u64
        lib.orc_counter_hash.argtypes = [u64] * 5
        lib.orc_uniform.restype = dbl
        lib.orc_uniform.argtypes = [u64] * 5
        lib.orc_row_probs.restype = u32
        lib.orc_row_probs.argtypes = [vp, C.c_int, i32, dbl, i32, dbl, vp, vp]
        lib.orc_row_argmax.restype = i32
        lib.orc_row_argmax.argtypes = [vp, C.c_int, i32, vp]
        lib.orc_verify_one.restype = u32
        lib.orc_verify_one.argtypes = [vp, i64, vp, i64, C.c_int, vp, i32, i32,
                                       dbl, i32, dbl, vp, vp, vp, vp, vp, vp, vp]
        lib.orc_verify_linear.restype = u32
        lib.orc_verify_linear.argtypes = [vp, i64, vp, i64, C.c_int, vp, i32,
                                          i32, i32, dbl, i32, dbl, u64, vp, u64,
                                          vp, vp, vp, vp, vp]
        lib.orc_verify_tree_greedy.restype = u32
        lib.orc_verify_tree_greedy.argtypes = [vp, i64, C.c_int, vp, vp, i32,
                                               i32, i32, vp, vp, vp]
        lib.orc_verify_tree_sampled_one.restype = u32
        lib.orc_verify_tree_sampled_one.argtypes = [vp, i64, C.c_int, vp, vp, i32,
                                                    i32, dbl, i32, dbl, vp, vp, vp,
                                                    vp, vp, vp]
        lib.orc_verify_tree_sampled.restype = u32
        lib.orc_verify_tree_sampled.argtypes = [vp, i64, C.c_int, vp, vp, i32, i32,
                                                i32, dbl, i32, dbl, u64, vp, u64, vp,
                                                vp, vp, vp]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"logits must be float32 or uint16 (bf16 bits), got {a.dtype}")


def _contig(a, dtype=None):
    return np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))


# ---- counter RNG ---------------------------------------------------------

def splitmix64_mix(x: int) -> int:
    return int(_load().orc_splitmix64_mix(x))


def counter_hash(seed: int, seq: int, step: int, row: int, purpose: int) -> int:
    return int(_load().orc_counter_hash(seed, seq, step, row, purpose))


def uniform(seed: int, seq: int, step: int, row: int, purpose: int) -> float:
    return float(_load().orc_uniform(seed, seq, step, row, purpose))


def uniforms(seed: int, seq_ids, step: int, n_rows: int, purpose: int) -> np.ndarray:
    """[len(seq_ids), n_rows] table of uniforms (float64, exactly 24-bit)."""
    lib = _load()
    out = np.empty((len(seq_ids), n_rows), dtype=np.float64)
    for a, s in enumerate(seq_ids):
        for r in range(n_rows):
            out[a, r] = lib.orc_uniform(seed, int(s), step, r, purpose)
    return out


# ---- single rows -----------------------------------------------------------

def row_probs(row: np.ndarray, temperature: float, top_p: float = 1.0, top_k: int = 0):
    """(probabilities float64[V], status bits, top-p margin) of one row."""
    row = _contig(row)
    V = row.shape[-1]
    out = np.empty(V, dtype=np.float64)
    margin = np.empty(1, dtype=np.float64)
    st = _load().orc_row_probs(_ptr(row), _dtype_code(row), V, temperature, int(top_k),
                               top_p, _ptr(out), _ptr(margin))
    return out, int(st), float(margin[0])


def row_argmax(row: np.ndarray) -> int:
    row = _contig(row)
    st = np.zeros(1, dtype=np.uint32)
    return int(_load().orc_row_argmax(_ptr(row), _dtype_code(row), row.shape[-1],
                                      _ptr(st)))


# ---- linear verify ----------------------------------------------------------

def verify_one(ar, draft, ids, temperature, top_p, u_accept, u_resid, V=None, top_k=0):
    """One sequence with explicit uniforms.  ar [B+1, S], draft [B, S]."""
    ar = _contig(ar)
    code = _dtype_code(ar)
    B = ar.shape[0] - 1
    S = ar.shape[-1]
    V = S if V is None else V
    if draft is not None:
        draft = _contig(draft)
        assert draft.dtype == ar.dtype and draft.shape[0] == B
    ids = _contig(np.asarray(ids), np.int32)
    u_accept = _contig(np.asarray(u_accept, dtype=np.float64))
    u_resid = _contig(np.asarray(u_resid, dtype=np.float64))
    assert u_accept.size >= B and u_resid.size >= B + 1
    tokens = np.empty(B + 1, dtype=np.int32)
    n = np.empty(1, dtype=np.int32)
    p = np.full(B, np.nan)
    q = np.full(B, np.nan)
    margin = np.empty(1)
    st = _load().orc_verify_one(
        _ptr(ar), S, _ptr(draft), draft.shape[-1] if draft is not None else S,
        code, _ptr(ids), B, V, temperature, int(top_k), top_p, _ptr(u_accept),
        _ptr(u_resid), _ptr(tokens), _ptr(n), _ptr(p), _ptr(q), _ptr(margin))
    return dict(tokens=tokens, n_emitted=int(n[0]), p_draft=p, q_draft=q,
                margin=float(margin[0]), status=int(st))


def verify_linear(ar, draft, ids, temperature, top_p, seed, step, seq_ids=None,
                  V=None, top_k=0):
    """Batch verify with the counter RNG.  ar [N, B+1, S], draft [N, B, S]."""
    ar = _contig(ar)
    code = _dtype_code(ar)
    N, B1, S = ar.shape
    B = B1 - 1
    V = S if V is None else V
    if draft is not None:
        draft = _contig(draft)
        assert draft.dtype == ar.dtype and draft.shape[:2] == (N, B)
    ids = _contig(np.asarray(ids), np.int32).reshape(N, B)
    sid = None if seq_ids is None else _contig(np.asarray(seq_ids), np.uint64)
    tokens = np.empty((N, B + 1), dtype=np.int32)
    n_em = np.empty(N, dtype=np.int32)
    p = np.full((N, B), np.nan)
    q = np.full((N, B), np.nan)
    margin = np.empty(N)
    st = _load().orc_verify_linear(
        _ptr(ar), S, _ptr(draft), draft.shape[-1] if draft is not None else S,
        code, _ptr(ids), N, B, V, temperature, int(top_k), top_p, seed, _ptr(sid), step,
        _ptr(tokens), _ptr(n_em), _ptr(p), _ptr(q), _ptr(margin))
    return dict(tokens=tokens, n_emitted=n_em, p_draft=p, q_draft=q,
                margin=margin, status=int(st))


def verify_linear_parallel(ar, draft, ids, temperature, top_p, seed, step, seq_ids=None,
                           V=None, top_k=0, threads=None):
    """verify_linear over a pool of host threads: the batch is cut into
    contiguous groups of sequences, each verified by one plain
    ``orc_verify_linear`` call on its own rows (ctypes releases the GIL while
    the C code runs).  Sequence n keeps its RNG key (seq_ids[n], default n),
    so the result equals one verify_linear call over the whole batch."""
    ar = _contig(ar)
    N = ar.shape[0]
    sid = (np.arange(N, dtype=np.uint64) if seq_ids is None
           else _contig(np.asarray(seq_ids), np.uint64).reshape(N))
    threads = max(1, min(N, threads or os.cpu_count() or 1))
    cuts = np.linspace(0, N, min(N, 4 * threads) + 1).astype(int)
    parts = [(a, b) for a, b in zip(cuts[:-1], cuts[1:]) if b > a]

    def run(ab):
        a, b = ab
        return verify_linear(ar[a:b], None if draft is None else draft[a:b], np.asarray(ids)[a:b],
                             temperature, top_p, seed, step, seq_ids=sid[a:b], V=V, top_k=top_k)

    with ThreadPoolExecutor(max_workers=threads) as ex:
        outs = list(ex.map(run, parts))
    res = {k: np.concatenate([o[k] for o in outs]) for k in
           ("tokens", "n_emitted", "p_draft", "q_draft", "margin")}
    res["status"] = 0
    for o in outs:
        res["status"] |= o["status"]
    return res


# ---- greedy tree --------------------------------------------------------------

def verify_tree_greedy(ar, node_tokens, parents, V=None):
    """ar [N, M+1, S]; node_tokens, parents [N, M] int32."""
    ar = _contig(ar)
    code = _dtype_code(ar)
    N, M1, S = ar.shape
    M = M1 - 1
    V = S if V is None else V
    tok = _contig(np.asarray(node_tokens), np.int32).reshape(N, M)
    par = _contig(np.asarray(parents), np.int32).reshape(N, M)
    path = np.empty((N, M), dtype=np.int32)
    plen = np.empty(N, dtype=np.int32)
    toks = np.empty((N, M + 1), dtype=np.int32)
    st = _load().orc_verify_tree_greedy(_ptr(ar), S, code, _ptr(tok), _ptr(par),
                                        N, M, V, _ptr(path), _ptr(plen),
                                        _ptr(toks))
    return dict(path_nodes=path, path_len=plen, tokens=toks, status=int(st))


# ---- sampled tree ---------------------------------------------------------------

def verify_tree_sampled_one(ar, node_tokens, parents, temperature, top_p, u_accept, u_resid,
                            V=None, top_k=0):
    """One tree with explicit uniforms.  ar [M+1, S]; node_tokens, parents
    [M]; u_accept [M+1] (entry k+1 tests node k), u_resid [M+1] (by row)."""
    ar = _contig(ar)
    code = _dtype_code(ar)
    M1, S = ar.shape
    M = M1 - 1
    V = S if V is None else V
    tok = _contig(np.asarray(node_tokens), np.int32).reshape(M)
    par = _contig(np.asarray(parents), np.int32).reshape(M)
    ua = _contig(np.asarray(u_accept, dtype=np.float64))
    ur = _contig(np.asarray(u_resid, dtype=np.float64))
    assert ua.size >= M + 1 and ur.size >= M + 1
    path = np.empty(max(M, 1), dtype=np.int32)
    plen = np.empty(1, dtype=np.int32)
    toks = np.empty(M + 1, dtype=np.int32)
    margin = np.empty(1)
    st = _load().orc_verify_tree_sampled_one(_ptr(ar), S, code, _ptr(tok), _ptr(par), M, V,
                                             temperature, int(top_k), top_p, _ptr(ua),
                                             _ptr(ur),
                                             _ptr(path), _ptr(plen), _ptr(toks), _ptr(margin))
    return dict(path_nodes=path[:M], path_len=int(plen[0]), tokens=toks,
                margin=float(margin[0]), status=int(st))


def verify_tree_sampled(ar, node_tokens, parents, temperature, top_p, seed, step,
                        seq_ids=None, V=None, top_k=0):
    """Batch sampled tree verify with the counter RNG.  ar [N, M+1, S];
    node_tokens, parents int32 [N, M]."""
    ar = _contig(ar)
    code = _dtype_code(ar)
    N, M1, S = ar.shape
    M = M1 - 1
    V = S if V is None else V
    tok = _contig(np.asarray(node_tokens), np.int32).reshape(N, M)
    par = _contig(np.asarray(parents), np.int32).reshape(N, M)
    sid = None if seq_ids is None else _contig(np.asarray(seq_ids), np.uint64)
    path = np.empty((N, M), dtype=np.int32)
    plen = np.empty(N, dtype=np.int32)
    toks = np.empty((N, M + 1), dtype=np.int32)
    margin = np.empty(N)
    st = _load().orc_verify_tree_sampled(_ptr(ar), S, code, _ptr(tok), _ptr(par), N, M, V,
                                         temperature, int(top_k), top_p, seed, _ptr(sid), step,
                                         _ptr(path),
                                         _ptr(plen), _ptr(toks), _ptr(margin))
    return dict(path_nodes=path, path_len=plen, tokens=toks, margin=margin, status=int(st))
