"""Benchmark of the Psi-Spec verify step (one JSON line on rank 0).

Default workload: the large-batch nucleus verify -- batch 256, block B=8,
vocabulary 151,936, bf16 logits, temperature 0.7, top-p 0.95 -- i.e. the
configuration the headline metric (verified blocks/s and logits HBM GB/s vs
peak) is quoted on.  One step = one call of ``psi_verify_linear`` over the
whole batch (all kernels of the path).  Inputs are synthetic (seeded), 1.32
GB per step, larger than the 126 MB L2, and resident in HBM before timing.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--config NAME]

Multi-GPU (torchrun, one rank per GPU): each rank verifies its own batch of
the same shape with sequence ids offset by rank (batch sharding, no
collective on the data path); ``value`` counts the blocks of all ranks over
the slowest rank's device time.
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import psi_inputs  # noqa: E402

METRIC = "Ψ-Spec verify blocks/s & logits HBM GB/s vs peak at bs=256,B=8,V=151936"
FALLBACK_HBM_GBS = 6650.0  # used only if MEASURED_PEAKS.json is absent


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="large_batch_nucleus",
                    choices=[k for k, v in psi_inputs.CONFIGS.items()])
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the batch size (smaller profiling cases)")
    ap.add_argument("--max-repeats", type=int, default=200,
                    help="most timed passes of K steps (passes continue until ~0.5 s)")
    return ap.parse_args()


# ---- peaks, profiles, clocks ------------------------------------------------------

def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def strip_c_comments(text: str) -> str:
    """C / CUDA source as the compiler sees it: comments removed (string and
    character literals kept whole), trailing spaces and blank lines dropped."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    lines = [ln.rstrip() for ln in "".join(out).splitlines()]
    return "\n".join(ln for ln in lines if ln)


def kernel_source_files():
    files = sorted(glob.glob(os.path.join(ROOT, "rejection_sampling_verify_b200", "csrc", "*")))
    return files + [os.path.join(ROOT, "include", "psi_verify.h")]


def kernel_source_hash() -> str:
    """First 16 hex digits of SHA-256 over the kernel sources' code (comments
    and blank lines removed): a comment-only edit keeps it, any code change
    does not."""
    h = hashlib.sha256()
    for f in kernel_source_files():
        with open(f, encoding="utf-8") as fh:
            h.update(os.path.basename(f).encode())
            h.update(strip_c_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel and
    workload, or None if absent or taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", f"{kernel}__{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    src = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    val = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    if not src or not val or src.group(1) != kernel_source_hash():
        return None
    return int(val.group(1))


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every ~20 ms."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device: torch.device):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            pr = torch.cuda.get_device_properties(device)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: clocks unknown
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.nv:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---- distributed plumbing ------------------------------------------------------------

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus and world > 1:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    return rank, local, world, pg


def max_over_ranks(x: float, pg, device) -> float:
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg):
    if pg is not None:
        pg.barrier()


# ---- workloads ----------------------------------------------------------------------

def algorithmic_bytes(cfg) -> int:
    """Bytes of logits one step must read once: every AR row and, for T > 0,
    every draft row (the formula batch*(2B+1)*V*elem); the greedy paths read
    the AR rows only."""
    es = 4 if getattr(cfg, "dtype", "bf16") == "f32" else 2
    if isinstance(cfg, psi_inputs.TreeConfig):
        return cfg.N * (cfg.M + 1) * cfg.V * es
    rows = cfg.N * (cfg.B + 1) + (cfg.N * cfg.B if cfg.temperature > 0 else 0)
    return rows * cfg.V * es


def make_inputs(cfg, device, rank):
    if isinstance(cfg, psi_inputs.TreeConfig):
        return psi_inputs.tree_batch(cfg, device=device, index=rank)
    return psi_inputs.linear_batch(cfg, device=device, index=rank)


def call_verify(psi, cfg, batch, step, seq_ids, ws, out):
    """One verify step as a server calls it: tokens and counts only (no p / q
    diagnostics), which lets the sampled path read rows in early-exit rounds."""
    if isinstance(cfg, psi_inputs.TreeConfig):
        if cfg.temperature > 0:
            return psi.verify_tree_sampled(batch.ar, batch.node_tokens, batch.parents,
                                           cfg.temperature, cfg.top_p, seed=cfg.seed, step=step,
                                           workspace=ws, out=out)
        return psi.verify_tree_greedy(batch.ar, batch.node_tokens, batch.parents, workspace=ws,
                                      out=out)
    return psi.verify_linear(batch.ar, batch.draft, batch.ids, cfg.temperature, cfg.top_p,
                             seed=cfg.seed, step=step, seq_ids=seq_ids, want_probs=False,
                             workspace=ws, out=out)


def sampled_rounds(cfg):
    """Position rounds of the linear paths' early exit: [(first, end), ...]
    (the schedule of include/psi_verify.h); one round of every position
    below PSI_EARLY_EXIT_MIN_N sequences."""
    import rejection_sampling_verify_b200 as psi
    if cfg.N < psi.PSI_EARLY_EXIT_MIN_N:
        return [(0, cfg.B + 1)]
    if cfg.temperature == 0:
        short, rs = psi.PSI_GREEDY_SHORT_ROUNDS, psi.PSI_GREEDY_ROUND_POSITIONS
    else:
        short, rs = psi.PSI_SAMPLED_SHORT_ROUNDS, psi.PSI_SAMPLED_ROUND_POSITIONS
    begins = [min(k * rs, cfg.B + 1) for k in range(short + 1)] + [cfg.B + 1]
    return [(a, b) for a, b in zip(begins, begins[1:]) if a < b]


def rows_in_round(cfg, r):
    """AR rows of the round's positions, plus draft rows when T > 0 (none for
    the bonus row)."""
    i0, i1 = r
    return (i1 - i0) + ((min(i1, cfg.B) - i0) if cfg.temperature > 0 else 0)


def main_launch_bytes(cfg) -> int:
    """Algorithmic bytes of one launch of the timed main kernel: the first
    round's row scan (sampled) or argmax (greedy linear) over every
    sequence's rows of the first round's positions; every node row of a
    sampled tree (the greedy tree walk's bytes are counted from its matches
    in main())."""
    if isinstance(cfg, psi_inputs.TreeConfig):
        return algorithmic_bytes(cfg)
    es = 4 if cfg.dtype == "f32" else 2
    return cfg.N * rows_in_round(cfg, sampled_rounds(cfg)[0]) * cfg.V * es


def rows_read(cfg, n_emitted) -> int:
    """Logit rows the linear paths read for these results: a sequence takes
    part in the rounds up to the one holding its emitting position."""
    rounds = sampled_rounds(cfg)
    total = 0
    for n in n_emitted:
        L = int(n) - 1
        for r in rounds:
            total += rows_in_round(cfg, r)
            if L < r[1]:
                break
    return total


def tree_rows_read(argmax, node_tokens, parents) -> int:
    """Rows the greedy tree walk reads: per tree the root's and every matched
    node's (node k is matched when its token is its parent row's argmax and
    its parent is matched).  argmax [N, M+1], node_tokens / parents [N, M]."""
    total = 0
    for am, tok, par in zip(argmax, node_tokens, parents):
        matched = []
        for k in range(len(tok)):
            p = int(par[k])
            ok = -1 <= p < k and (p < 0 or matched[p])
            matched.append(bool(ok and int(tok[k]) == int(am[p + 1])))
        total += 1 + sum(matched)
    return total


def units(cfg) -> int:
    return cfg.N  # one verified block per sequence per step


# ---- oracle (CPU) -------------------------------------------------------------------------

def oracle_sample_rate(cfg, batch_cpu, target_seconds, one=None, threads=1):
    """Times the CPU oracle on a bounded sample of the workload; returns
    (blocks/s, sequences timed, seconds).  `one` is the seconds one sequence
    takes on one thread, if already known (else one sequence is timed first
    to size the sample).  threads > 1 runs the oracle's thread pool over
    sequences (oracle.verify_linear_parallel)."""
    import oracle
    n_have = batch_cpu.ar.shape[0]
    if isinstance(cfg, psi_inputs.TreeConfig):
        ar = psi_inputs.to_host_logits(batch_cpu.ar)
        tok, par = batch_cpu.node_tokens.numpy(), batch_cpu.parents.numpy()

        def tree(n):
            if cfg.temperature > 0:
                oracle.verify_tree_sampled(ar[:n], tok[:n], par[:n], cfg.temperature, cfg.top_p,
                                           cfg.seed, 0)
            else:
                oracle.verify_tree_greedy(ar[:n], tok[:n], par[:n])
        if one is None:
            t0 = time.perf_counter()
            tree(1)
            one = time.perf_counter() - t0
        n = max(1, min(cfg.N, n_have, int(target_seconds / max(one, 1e-6))))
        t0 = time.perf_counter()
        tree(n)
        dt = time.perf_counter() - t0
        return n / dt, n, dt
    ar = psi_inputs.to_host_logits(batch_cpu.ar)
    draft = psi_inputs.to_host_logits(batch_cpu.draft) if cfg.temperature > 0 else None
    ids = batch_cpu.ids.numpy()
    if one is None:
        t0 = time.perf_counter()
        oracle.verify_linear(ar[:1], None if draft is None else draft[:1], ids[:1],
                             cfg.temperature, cfg.top_p, cfg.seed, 0)
        one = time.perf_counter() - t0
    n = max(1, min(cfg.N, n_have, int(threads * target_seconds / max(one, 1e-6))))
    if threads > 1:  # whole rounds of the pool
        n = max(1, min(n_have, (n // threads) * threads or threads))
    t0 = time.perf_counter()
    if threads > 1:
        oracle.verify_linear_parallel(ar[:n], None if draft is None else draft[:n], ids[:n],
                                      cfg.temperature, cfg.top_p, cfg.seed, 0, threads=threads)
    else:
        oracle.verify_linear(ar[:n], None if draft is None else draft[:n], ids[:n],
                             cfg.temperature, cfg.top_p, cfg.seed, 0)
    dt = time.perf_counter() - t0
    return n / dt, n, dt


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def sample_inputs(cfg, n):
    """The first n sequences of the workload's recipe, generated on the host."""
    if isinstance(cfg, psi_inputs.TreeConfig):
        return psi_inputs.tree_batch(cfg, device="cpu", N=n)
    return psi_inputs.linear_batch(cfg, device="cpu", N=n)


def config_block(cfg, name, world):
    c = {"workload": name}
    if isinstance(cfg, psi_inputs.TreeConfig):
        c.update(batch=cfg.N, tree_nodes=cfg.M, vocab=cfg.V, depth=cfg.depth, width=cfg.width,
                 temperature=cfg.temperature, top_p=cfg.top_p)
    else:
        c.update(batch=cfg.N, block=cfg.B, vocab=cfg.V, temperature=cfg.temperature,
                 top_p=cfg.top_p, logits_dtype=cfg.dtype,
                 outputs="tokens and counts (no p/q diagnostics)")
        c.update(schedule=(f"early-exit rounds {sampled_rounds(cfg)}; roofline = the first round's "
                           "main kernel" if cfg.N >= 64 else "one pass over every row"))
    c.update(global_batch=cfg.N * world, parallelism=f"batch-sharded x{world} (no collective)",
             l2="inputs larger than L2 (no flush needed)",
             inputs="seeded synthetic logits resident in HBM")
    return c


def run_reference(args, cfg, name):
    """The reference arm: the CPU oracle as it stands, on a pool of the host's
    cores (one plain oracle call per group of sequences), each step a bounded
    sample of the workload (whole run ~2 minutes).  ms_per_step is the time a
    step's sample actually took."""
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    cores = host_cores()
    per_step = max(0.2, 120.0 / max(1, args.steps + args.warmup))
    probe = make_inputs(cfg, "cpu", 0) if cfg.N * cfg.V < 4e6 else sample_inputs(cfg, 1)
    _, _, one = oracle_sample_rate(cfg, probe, 0.0)
    n_seq = max(1, min(cfg.N, cores * max(1, int(per_step / max(one, 1e-6)))))
    batch = probe if n_seq <= (probe.ar.shape[0]) else sample_inputs(cfg, n_seq)
    rates, times = [], []
    seqs = 0
    for s in range(args.warmup + args.steps):
        r, n, dt = oracle_sample_rate(cfg, batch, per_step, one=one, threads=cores)
        if s >= args.warmup:
            rates.append(r)
            times.append(dt)
            seqs = n
    value = float(statistics.median(rates))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "blocks/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * float(statistics.median(times)),
        "sequences_per_step": seqs,
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(config_block(cfg, name, 1), schedule="every row (the oracle as it stands)"),
        "cpu_baseline": {"value": value, "unit": "blocks/s", "cores": cores, "kind": "oracle",
                         "sample": (f"{seqs} of the {cfg.N} sequences of the workload per step, "
                                    f"on a pool of {cores} host threads")},
        "e2e": {"value": value, "unit": "blocks/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    cfg = psi_inputs.CONFIGS[args.config]
    name = args.config
    if args.batch is not None:
        cfg = type(cfg)(**{**cfg.__dict__, "N": args.batch})
        name = f"{name}_batch{args.batch}"
    if args.impl == "reference":
        return run_reference(args, cfg, name)

    import rejection_sampling_verify_b200 as psi
    psi.load_library()
    rank, local, world, pg = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    batch = make_inputs(cfg, dev, rank)
    is_tree = isinstance(cfg, psi_inputs.TreeConfig)
    seq_ids = None
    if not is_tree and world > 1:
        seq_ids = torch.arange(rank * cfg.N, (rank + 1) * cfg.N, device=dev, dtype=torch.int64)
    if is_tree and cfg.temperature > 0:
        ws_bytes = psi.psi_verify_tree_sampled_workspace_bytes(cfg.N, cfg.M, cfg.V,
                                                               psi.PSI_DTYPE_BF16,
                                                               cfg.temperature, cfg.top_p)
    elif is_tree:
        ws_bytes = psi.psi_verify_tree_greedy_workspace_bytes(cfg.N, cfg.M, cfg.V,
                                                              psi.PSI_DTYPE_BF16)
    else:
        ws_bytes = psi.psi_verify_linear_workspace_bytes(
            cfg.N, cfg.B, cfg.V, psi.PSI_DTYPE_BF16 if cfg.dtype == "bf16" else psi.PSI_DTYPE_F32,
            cfg.temperature, cfg.top_p)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    out = call_verify(psi, cfg, batch, 0, seq_ids, ws, None)
    torch.cuda.synchronize()

    # warm-up
    for w in range(args.warmup):
        call_verify(psi, cfg, batch, w, seq_ids, ws, out)
    torch.cuda.synchronize()

    # timed region: K steps, bracketed by a barrier and a synchronize, main-kernel
    # events recorded per step; repeated so that the clock record spans at
    # least ~0.5 s (the per-step time reported is the median over the repeats)
    K = args.steps
    # the same number of passes on every rank (each pass has its own barriers)
    est = max_over_ranks(max(step_ms_estimate(psi, cfg, batch, seq_ids, ws, out, stream), 1e-3),
                         pg, dev)
    repeats = max(1, min(args.max_repeats, math.ceil(500.0 / (est * K))))
    ev_main = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(K)] for _ in range(repeats)]
    for rep in ev_main:  # torch creates the CUDA events lazily, on first record
        for a, b in rep:
            a.record(stream)
            b.record(stream)
    spans = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(repeats)]
    torch.cuda.synchronize()
    elapsed = []
    with ClockSampler(dev) as clocks:
        for rep in range(repeats):
            barrier(pg)
            torch.cuda.synchronize()
            start, stop = spans[rep]
            start.record(stream)
            for k in range(K):
                psi.psi_profile_main_kernel(ev_main[rep][k][0].cuda_event,
                                            ev_main[rep][k][1].cuda_event)
                call_verify(psi, cfg, batch, args.warmup + rep * K + k, seq_ids, ws, out)
            stop.record(stream)
            psi.psi_profile_main_kernel(None, None)
            torch.cuda.synchronize()
            barrier(pg)
            elapsed.append(max_over_ranks(start.elapsed_time(stop), pg, dev))
    elapsed_ms = float(statistics.median(elapsed))
    main_ms = statistics.mean(a.elapsed_time(b) for rep in ev_main for a, b in rep)
    status = int(out.status.item()) & 0xFFFFFFFF
    if status:
        print(f"warning: device status bits {status:#x}", file=sys.stderr)

    ms_per_step = elapsed_ms / K
    blocks = units(cfg) * world * K
    value = blocks / (elapsed_ms / 1000.0)
    alg = main_launch_bytes(cfg)
    formula = algorithmic_bytes(cfg)
    es = 4 if getattr(cfg, "dtype", "bf16") == "f32" else 2
    if is_tree and cfg.temperature > 0:
        read = formula
    elif is_tree:  # the walk reads the root's and the matched nodes' rows
        am = batch.ar.float().argmax(dim=-1).cpu().numpy()
        read = tree_rows_read(am, batch.node_tokens.cpu().numpy(),
                              batch.parents.cpu().numpy()) * cfg.V * es
        alg = read  # one launch: the walk
    else:
        read = rows_read(cfg, out.n_emitted.cpu().numpy()) * cfg.V * es
    peak, peak_kind = hbm_peak()
    achieved = alg / (main_ms / 1000.0) / 1e9
    if is_tree:
        kernel = "psi_row_scan" if cfg.temperature > 0 else "psi_tree_walk"
    else:
        kernel = "psi_row_scan" if cfg.temperature > 0 else "psi_row_argmax"

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(psi, cfg, batch, seq_ids, ws, min(K, 10), dev, pg, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores = host_cores()
        bc = make_inputs(cfg, "cpu", 0) if cfg.N * cfg.V < 4e6 else cpu_copy(batch, cfg, 4 * cores)
        r1, n1, dt1 = oracle_sample_rate(cfg, bc, args.cpu_seconds / 2)
        rp, npool, dtp = oracle_sample_rate(cfg, bc, args.cpu_seconds / 2, one=dt1 / n1,
                                            threads=cores)
        cpu = {"value": rp, "unit": "blocks/s", "cores": cores, "kind": "oracle",
               "sample": (f"{npool} of the {cfg.N} sequences of one step on a pool of {cores} "
                          f"host threads ({dtp:.1f} s)"),
               "single_thread": {"value": r1, "unit": "blocks/s", "cores": 1,
                                 "sample": f"{n1} sequences ({dt1:.1f} s)"}}

    if rank == 0:
        # our kernels per call: greedy tree: the walk; sampled tree: row
        # scan, row finish, walk; greedy linear: argmax and emit, or per
        # early-exit round list building and argmax, then emit; sampled: per
        # round list building, row scan, row finish and unit decision, then
        # one second pass of the three, the general-path list, fast_emit and
        # the draws (over the nucleus with top-p, else over the whole row)
        rounds = 0 if is_tree else len(sampled_rounds(cfg))
        if is_tree and cfg.temperature == 0:
            launches_per_step = 1  # the level-by-level walk
        elif is_tree:
            launches_per_step = 3  # row scan, row finish, sampled walk
        elif cfg.temperature == 0 and cfg.N < 64:
            launches_per_step = 2  # argmax + emit
        elif cfg.temperature == 0:  # per round: list building and argmax; then emit
            launches_per_step = 2 * rounds + 1
        elif cfg.N < 64:  # one pass: scan, finish, unit, their second passes, lists, emit, draw
            launches_per_step = 9
        else:
            launches_per_step = 4 * rounds + 6
        line = {
            "metric": METRIC, "value": value, "unit": "blocks/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if getattr(cfg, "dtype", "bf16") == "bf16" else "f32",
            "data": "synthetic", "config": config_block(cfg, name, world),
            "formula_bytes_per_step": formula * world,
            "bytes_read_per_step": read * world,
            "read_gbs": read * world / (elapsed_ms / K / 1000.0) / 1e9,
            "roofline": {"kernel": kernel, "bound": "hbm", "achieved": achieved, "peak": peak,
                         "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind,
                         "algorithmic_bytes_per_launch": alg, "launch_ms": main_ms,
                         "traffic": profiled_traffic(kernel, name)},
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks.summary(),
            "timed_repeats": repeats,
            "gpu_launches": launches_per_step * K, "device_status": status,
        }
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()
    return 0


def step_ms_estimate(psi, cfg, batch, seq_ids, ws, out, stream) -> float:
    """Milliseconds of one verify call (three calls timed with CUDA events)."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for k in range(3):
        call_verify(psi, cfg, batch, k, seq_ids, ws, out)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / 3.0


def cpu_copy(batch, cfg, n=64):
    """Host copy of the first n sequences (enough for the oracle sample)."""
    n = min(cfg.N, n)
    if isinstance(cfg, psi_inputs.TreeConfig):
        return psi_inputs.TreeBatch(batch.ar[:n].cpu(), batch.node_tokens[:n].cpu(),
                                    batch.parents[:n].cpu(), None)
    return psi_inputs.LinearBatch(batch.ar[:n].cpu(), batch.draft[:n].cpu(), batch.ids[:n].cpu(),
                                  batch.temperature, batch.top_p)


def measure_e2e(psi, cfg, batch, seq_ids, ws, K, dev, pg, world):
    """Same metric through the public API from pinned host buffers: every step
    copies its inputs host->device, verifies, and copies the emitted tokens
    and counts back."""
    is_tree = isinstance(cfg, psi_inputs.TreeConfig)
    if is_tree:
        host = [batch.ar.cpu().pin_memory(), batch.node_tokens.cpu().pin_memory(),
                batch.parents.cpu().pin_memory()]
    elif cfg.temperature == 0:  # greedy: the draft logits are not an input
        host = [batch.ar.cpu().pin_memory(), batch.ids.cpu().pin_memory()]
    else:
        host = [batch.ar.cpu().pin_memory(), batch.draft.cpu().pin_memory(),
                batch.ids.cpu().pin_memory()]
    dev_bufs = [torch.empty_like(h, device=dev) for h in host]
    out = call_verify(psi, cfg, batch, 0, seq_ids, ws, None)
    res_host = [torch.empty_like(out.tokens, device="cpu").pin_memory(),
                torch.empty_like(out.path_len if is_tree else out.n_emitted,
                                 device="cpu").pin_memory()]
    h2d = sum(h.numel() * h.element_size() for h in host)
    d2h = sum(h.numel() * h.element_size() for h in res_host)
    stream = torch.cuda.current_stream(dev)

    def step(k):
        for d, h in zip(dev_bufs, host):
            d.copy_(h, non_blocking=True)
        if is_tree:
            b = psi_inputs.TreeBatch(*dev_bufs, None)
        elif cfg.temperature == 0:
            b = psi_inputs.LinearBatch(dev_bufs[0], None, dev_bufs[1], cfg.temperature, cfg.top_p)
        else:
            b = psi_inputs.LinearBatch(dev_bufs[0], dev_bufs[1], dev_bufs[2], cfg.temperature,
                                       cfg.top_p)
        o = call_verify(psi, cfg, b, k, seq_ids, ws, out)
        res_host[0].copy_(o.tokens, non_blocking=True)
        res_host[1].copy_(o.path_len if is_tree else o.n_emitted, non_blocking=True)

    step(0)
    torch.cuda.synchronize()
    barrier(pg)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for k in range(K):
        step(k + 1)
    e.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e), pg, dev)
    return {"value": units(cfg) * world * K / (ms / 1000.0), "unit": "blocks/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": K}


if __name__ == "__main__":
    sys.exit(main())
