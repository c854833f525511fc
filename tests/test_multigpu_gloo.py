"""The N > 1 bench path, on CPU with the gloo backend (world size 2): ranks
rendezvous on 127.0.0.1, every rank takes part in the same collectives, the
reported time is the max over ranks, and each rank draws its own request."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import ffd_workloads as fw


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    r, lr, w = bench.dist_env()
    assert (r, lr, w) == (rank, rank, world)
    bench.dist_init("gloo", world)
    try:
        bench.dist_barrier(world)
        mx = bench.dist_max(10.0 * (rank + 1), world)
        total = bench.dist_sum(rank + 1, world)
        wl = fw.WORKLOADS["tiny"]
        w_rank = fw.scaled_workload(wl, seed=wl.seed + 1000 * rank) if rank else wl
        q = fw.make_inputs(w_rank)["q"]
        out[rank] = (mx, total, int(q.astype(np.int64).sum()))
        bench.dist_barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_reductions_and_replica_seeding():
    world = 2
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 20.0  # max over ranks
    assert out[0][1] == out[1][1] == 3.0
    assert out[0][2] != out[1][2]  # each replica serves a different request


def test_single_rank_helpers_are_identity():
    assert bench.dist_max(3.5, 1) == 3.5
    assert bench.dist_sum(2.0, 1) == 2.0
    bench.dist_barrier(1)


def test_algorithmic_bytes_accounting():
    w = fw.WORKLOADS["long128k"]
    lengths = np.array([131072], np.int32)
    nblk = w.capacity // w.block_size
    dense = bench.algorithmic_bytes(w, lengths, w.num_kv_heads * 131072, dense=True)
    assert dense["scan"] == 0
    assert dense["kv"] == 8 * 131072 * 512
    sparse = bench.algorithmic_bytes(w, lengths, 0, dense=False)
    assert sparse["scan"] == 8 * (131072 * 64 + nblk * 256) == 71303168
    assert sparse["partials"] == 8 * 32 * 4 * 130 * 4 * 2
    # kept-token count from a mask: a ragged last block counts its valid tokens only
    w2 = fw.Workload("m", 1, 4, 1, 512, 64, 4, 1.0, 0, context=200)
    mask = np.zeros((1, 1, 1), np.uint32)
    mask[0, 0, 0] = 0b1001  # blocks 0 and 3 (3 holds tokens 192..199)
    kb, vb, kt = bench.kept_tokens_from_mask(w2, np.array([200]), mask)
    assert (kb, vb, kt) == (2, 4, 64 + 8)
