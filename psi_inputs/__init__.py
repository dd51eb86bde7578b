"""Seeded synthetic inputs for the Psi-Spec verify step.

This module is shared by the tests, the smoke check and the benchmark: it
feeds the SAME bytes to the CUDA library and to the CPU oracle.  It holds
none of the verify step's arithmetic (no acceptance test, no residual, no
top-p); it only draws logits, draft ids and draft trees.

The workloads stand in for the pages' serving setup (a Qwen3-8B model,
vocabulary 151,936, blocks of 4-16 drafted tokens, batch 1-1024); no
prompt, dataset or weight is involved.  Recipes:

* ``tiny``: AR logits i.i.d. N(0, 2^2) float32; draft logits = AR rows
  0..B-1 + N(0, 1); draft ids sampled from softmax(draft / T) by the
  Gumbel-max construction.
* ``zipf``: each row is -1.1 * ln(rank + 1) over a per-row random permutation
  of the vocabulary plus N(0, 0.5^2); draft rows = AR rows + N(0, sigma^2);
  rows are rounded to bfloat16; draft ids are sampled from the draft
  softmax at the step's temperature (Gumbel-max), or are the draft row's
  argmax when the temperature is 0.
* trees: see :func:`tree_batch`.

All draws use ``torch.Generator`` objects seeded from (config seed, batch
index), on the requested device; the same call on the same device returns
the same bytes.
"""
from __future__ import annotations

import heapq
import math
from dataclasses import dataclass, field

import numpy as np
import torch

V_QWEN3 = 151936


@dataclass(frozen=True)
class LinearConfig:
    name: str
    N: int
    B: int
    V: int
    dtype: str          # "f32" or "bf16"
    temperature: float
    top_p: float
    seed: int
    steps: int
    kind: str           # "tiny" or "zipf"
    draft_sigma: float


@dataclass(frozen=True)
class TreeConfig:
    name: str
    N: int
    M: int
    V: int
    depth: int
    width: int
    seed: int
    steps: int
    iid: bool = False
    temperature: float = 0.0   # > 0: the sampled tree verify
    top_p: float = 1.0


CONFIGS = {
    "tiny": LinearConfig("tiny", 1, 4, 32, "f32", 1.0, 1.0, 0, 10_000, "tiny", 1.0),
    "single_stream": LinearConfig("single_stream", 8, 8, V_QWEN3, "bf16", 1.0, 1.0,
                                  1, 1_000, "zipf", 0.7),
    "large_batch_nucleus": LinearConfig("large_batch_nucleus", 256, 8, V_QWEN3,
                                        "bf16", 0.7, 0.95, 2, 200, "zipf", 0.5),
    "max_batch_greedy": LinearConfig("max_batch_greedy", 1024, 16, V_QWEN3, "bf16",
                                     0.0, 1.0, 3, 50, "zipf", 0.6),
    "tree_greedy": TreeConfig("tree_greedy", 16, 64, V_QWEN3, 8, 4, 4, 500),
    # the same trees and logits, verified by the sampled tree rule
    "tree_sampled": TreeConfig("tree_sampled", 16, 64, V_QWEN3, 8, 4, 4, 500,
                               temperature=0.7, top_p=0.95),
}


@dataclass
class LinearBatch:
    ar: torch.Tensor        # [N, B+1, V]
    draft: torch.Tensor     # [N, B, V]
    ids: torch.Tensor       # [N, B] int32
    temperature: float
    top_p: float


@dataclass
class TreeBatch:
    ar: torch.Tensor        # [N, M+1, V] bf16, row 0 = root, row k+1 = node k
    node_tokens: torch.Tensor  # [N, M] int32
    parents: torch.Tensor      # [N, M] int32, -1 = root, parent < child
    depth: torch.Tensor        # [N, M] int32 (bookkeeping only)


def _gen(device, seed: int, index: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + int(index)) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def zipf_rows(n_rows: int, V: int, noise_sigma: float, gen: torch.Generator,
              device, chunk: int = 256) -> torch.Tensor:
    """Float32 rows: -1.1*ln(rank+1) over a random permutation + N(0, s^2)."""
    base = -1.1 * torch.log(torch.arange(V, device=device, dtype=torch.float32) + 1.0)
    out = torch.empty(n_rows, V, device=device, dtype=torch.float32)
    for r0 in range(0, n_rows, chunk):
        r1 = min(n_rows, r0 + chunk)
        keys = torch.rand(r1 - r0, V, device=device, generator=gen)
        perm = torch.argsort(keys, dim=1)
        vals = base.expand(r1 - r0, V) + noise_sigma * torch.randn(
            r1 - r0, V, device=device, generator=gen)
        out[r0:r1].scatter_(1, perm, vals)
    return out


def gumbel_max(logits: torch.Tensor, temperature: float, gen: torch.Generator,
               chunk: int = 256) -> torch.Tensor:
    """Index sampled from softmax(logits / T) along the last dim (T > 0), or
    the first maximal index when T == 0."""
    flat = logits.reshape(-1, logits.shape[-1])
    out = torch.empty(flat.shape[0], dtype=torch.int64, device=flat.device)
    for r0 in range(0, flat.shape[0], chunk):
        x = flat[r0:r0 + chunk].float()
        if temperature > 0:
            u = torch.rand(x.shape, device=x.device, generator=gen,
                           dtype=torch.float64).clamp_(min=1e-300)
            x = x.double() / temperature - torch.log(-torch.log(u))
        out[r0:r0 + chunk] = torch.argmax(x, dim=-1)
    return out.reshape(logits.shape[:-1]).to(torch.int32)


def linear_batch(cfg: LinearConfig, device="cpu", index: int = 0, N: int | None = None,
                 V: int | None = None) -> LinearBatch:
    """One batch of inputs for the linear verify (override N or V for
    smaller parity cases of the same recipe)."""
    N = cfg.N if N is None else N
    V = cfg.V if V is None else V
    B = cfg.B
    g = _gen(device, cfg.seed, index)
    if cfg.kind == "tiny":
        ar = 2.0 * torch.randn(N, B + 1, V, device=device, generator=g)
        draft = ar[:, :B] + cfg.draft_sigma * torch.randn(N, B, V, device=device, generator=g)
    else:
        ar = zipf_rows(N * (B + 1), V, 0.5, g, device).reshape(N, B + 1, V)
        if cfg.dtype == "bf16":
            ar = ar.to(torch.bfloat16).float()
        draft = ar[:, :B] + cfg.draft_sigma * torch.randn(N, B, V, device=device, generator=g)
    tdt = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
    ar = ar.to(tdt).contiguous()
    draft = draft.to(tdt).contiguous()
    ids = gumbel_max(draft, cfg.temperature, g)
    return LinearBatch(ar, draft, ids.contiguous(), cfg.temperature, cfg.top_p)


def tree_batch(cfg: TreeConfig, device="cpu", index: int = 0, N: int | None = None,
               V: int | None = None) -> TreeBatch:
    """Greedy tree-verify inputs.

    Chain rows C_0..C_depth follow the zipf recipe; the draft's marginal at
    depth d (1..depth) is C_{d-1} + N(0, 0.7^2) and contributes its top
    ``width`` tokens.  A node is a tuple of candidate ranks (r_1..r_d) with
    score = sum of draft log-probabilities along it; the M best nodes are
    kept (ties: shallower first, then lexicographic ranks), which keeps the
    set prefix-closed.  Nodes are ordered by (depth, ranks).  The AR row of
    a depth-d node is C_d + N(0, 0.3^2); the root row is C_0.  With
    ``cfg.iid`` every AR row is instead an independent zipf row.
    """
    N = cfg.N if N is None else N
    V = cfg.V if V is None else V
    M, D, W = cfg.M, cfg.depth, cfg.width
    g = _gen(device, cfg.seed, index)
    ars, toks, pars, deps = [], [], [], []
    for _ in range(N):
        chain = zipf_rows(D + 1, V, 0.5, g, device).to(torch.bfloat16).float()
        draft = chain[:D] + 0.7 * torch.randn(D, V, device=device, generator=g)
        logp = torch.log_softmax(draft.double(), dim=-1)
        top = torch.topk(draft, W, dim=-1)
        cand_tok = top.indices.cpu().numpy()                     # [D, W]
        cand_lp = torch.gather(logp, 1, top.indices).cpu().numpy()  # [D, W]
        nodes = _best_first(cand_lp, M)
        nodes.sort(key=lambda r: (len(r), r))
        index_of = {r: k for k, r in enumerate(nodes)}
        tok = np.array([cand_tok[len(r) - 1, r[-1]] for r in nodes], dtype=np.int32)
        par = np.array([index_of[r[:-1]] if len(r) > 1 else -1 for r in nodes],
                       dtype=np.int32)
        dep = np.array([len(r) for r in nodes], dtype=np.int32)
        if cfg.iid:
            rows = zipf_rows(M + 1, V, 0.5, g, device)
        else:
            dep_t = torch.as_tensor(dep, device=device, dtype=torch.int64)
            rows = torch.empty(M + 1, V, device=device, dtype=torch.float32)
            rows[0] = chain[0]
            rows[1:] = chain[dep_t] + 0.3 * torch.randn(M, V, device=device, generator=g)
        ars.append(rows.to(torch.bfloat16))
        toks.append(torch.as_tensor(tok))
        pars.append(torch.as_tensor(par))
        deps.append(torch.as_tensor(dep))
    return TreeBatch(torch.stack(ars).contiguous(),
                     torch.stack(toks).to(device).contiguous(),
                     torch.stack(pars).to(device).contiguous(),
                     torch.stack(deps).to(device).contiguous())


def _best_first(cand_lp: np.ndarray, M: int):
    """The M highest-scoring rank tuples, expanded best-first."""
    D, W = cand_lp.shape
    heap = [(-float(cand_lp[0, r]), 1, (r,)) for r in range(W)]
    heapq.heapify(heap)
    kept = []
    while heap and len(kept) < M:
        neg, d, ranks = heapq.heappop(heap)
        kept.append(ranks)
        if d < D:
            for r in range(W):
                heapq.heappush(heap, (neg - float(cand_lp[d, r]), d + 1, ranks + (r,)))
    return kept


# ---- host views for the oracle -----------------------------------------------

def to_host_logits(t: torch.Tensor) -> np.ndarray:
    """numpy view for the oracle: float32 stays float32, bfloat16 becomes its
    uint16 bit patterns."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)


def from_bf16_bits(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def logits_nbytes(cfg: LinearConfig) -> int:
    es = 4 if cfg.dtype == "f32" else 2
    return cfg.N * (2 * cfg.B + 1) * cfg.V * es


__all__ = ["CONFIGS", "LinearConfig", "TreeConfig", "LinearBatch", "TreeBatch",
           "linear_batch", "tree_batch", "zipf_rows", "gumbel_max",
           "to_host_logits", "from_bf16_bits", "logits_nbytes", "V_QWEN3"]
