"""The multi-GPU path on CPU: two gloo ranks, world size 2.

Batch sharding needs no collective on the data path: each rank verifies its
own sequences, and the counter RNG is keyed by the global sequence id, so the
union of the ranks' results equals one verify of the whole batch.  The only
collectives are the benchmark's barrier and its max-over-ranks timing, which
run here on gloo.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import psi_inputs

WORLD = 2
N_PER_RANK = 3


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _global_batch():
    cfg = psi_inputs.LinearConfig("shard", WORLD * N_PER_RANK, 4, 64, "f32", 0.9, 0.8, 5, 1,
                                  "tiny", 1.0)
    return cfg, psi_inputs.linear_batch(cfg, device="cpu")


def _rank_main(rank, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        import bench
        cfg, b = _global_batch()
        lo, hi = rank * N_PER_RANK, (rank + 1) * N_PER_RANK
        ar = psi_inputs.to_host_logits(b.ar[lo:hi])
        draft = psi_inputs.to_host_logits(b.draft[lo:hi])
        ids = b.ids[lo:hi].numpy()
        seq = np.arange(lo, hi, dtype=np.uint64)  # global sequence ids
        r = oracle.verify_linear(ar, draft, ids, cfg.temperature, cfg.top_p, 11, 2, seq_ids=seq)
        gathered = [None] * WORLD
        dist.all_gather_object(gathered, {k: np.asarray(v) for k, v in r.items()})
        # the benchmark's timing: barrier, then the max over ranks
        bench.barrier(dist)
        t = bench.max_over_ranks(1.0 + rank, dist, torch.device("cpu"))
        if rank == 0:
            np.save(os.path.join(out_dir, "shards.npy"), np.array(gathered, dtype=object),
                    allow_pickle=True)
            np.save(os.path.join(out_dir, "max.npy"), np.array([t]))
    finally:
        dist.destroy_process_group()


def test_batch_sharding_needs_no_exchange(tmp_path):
    mp.start_processes(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=WORLD,
                       start_method="spawn", join=True)
    shards = np.load(tmp_path / "shards.npy", allow_pickle=True)
    assert float(np.load(tmp_path / "max.npy")[0]) == float(WORLD)
    cfg, b = _global_batch()
    whole = oracle.verify_linear(psi_inputs.to_host_logits(b.ar),
                                 psi_inputs.to_host_logits(b.draft), b.ids.numpy(),
                                 cfg.temperature, cfg.top_p, 11, 2,
                                 seq_ids=np.arange(WORLD * N_PER_RANK, dtype=np.uint64))
    for k, v in whole.items():
        v = np.asarray(v)
        if v.ndim == 0:
            continue
        joined = np.concatenate([np.asarray(s[k]) for s in shards])
        assert np.array_equal(joined, v), k


def test_sequence_ids_decide_the_draws_not_the_rank():
    """Moving a sequence to another position or shard with its id keeps its
    result; changing only its id changes the draws (the RNG is keyed by it)."""
    cfg, b = _global_batch()
    ar = psi_inputs.to_host_logits(b.ar)
    draft = psi_inputs.to_host_logits(b.draft)
    ids = b.ids.numpy()
    seq = np.arange(WORLD * N_PER_RANK, dtype=np.uint64) + 100
    base = oracle.verify_linear(ar, draft, ids, cfg.temperature, cfg.top_p, 3, 9, seq_ids=seq)
    perm = np.array([5, 2, 0, 4, 1, 3])
    moved = oracle.verify_linear(ar[perm], draft[perm], ids[perm], cfg.temperature, cfg.top_p,
                                 3, 9, seq_ids=seq[perm])
    assert np.array_equal(moved["tokens"], np.asarray(base["tokens"])[perm])
    other = oracle.verify_linear(ar, draft, ids, cfg.temperature, cfg.top_p, 3, 9,
                                 seq_ids=seq + 1000)
    assert not np.array_equal(other["tokens"], base["tokens"])
