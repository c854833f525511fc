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
import oracle


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


# ------------------------------------------------ context sharding (host) --

def _partials_numpy(q, k, v, mask_blocks, lengths_local, T, S, G):
    """Per-split softmax partials (m in base 2, l, acc) of one shard, computed
    from the selected blocks -- the quantity ffd_decode_partials exchanges."""
    B, Hq, D = q.shape
    nsplit = -(-(k.shape[2] // T) // S)
    m = np.full((B, Hq, nsplit), -np.inf)
    l = np.zeros((B, Hq, nsplit))
    acc = np.zeros((B, Hq, nsplit, D))
    qf = fw.bf16_bits_to_f32(q).astype(np.float64)
    kf = fw.bf16_bits_to_f32(k).astype(np.float64)
    vf = fw.bf16_bits_to_f32(v).astype(np.float64)
    for b in range(B):
        n = int(lengths_local[b])
        for h in range(Hq):
            g = h // G
            for t in range(n):
                j = t // T
                if not mask_blocks[b, g, j]:
                    continue
                s = j // S
                x = qf[b, h] @ kf[b, g, t] / np.sqrt(D) * np.log2(np.e)
                mn = max(m[b, h, s], x)
                scale = 0.0 if m[b, h, s] == -np.inf else 2.0 ** (m[b, h, s] - mn)
                l[b, h, s] = l[b, h, s] * scale + 2.0 ** (x - mn)
                acc[b, h, s] = acc[b, h, s] * scale + 2.0 ** (x - mn) * vf[b, g, t]
                m[b, h, s] = mn
    return m, l, acc


def _shard_worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    from sparse_long_context_ffd_b200 import sharded
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    bench.dist_init("gloo", world)
    try:
        T, S, G, Hkv, B = 64, 2, 2, 1, 2
        cap_local = T * S * 2
        cap = world * cap_local
        w = fw.Workload("shard", B, G * Hkv, Hkv, cap, T, S, 1.0, 5, ragged=(cap_local // 2, cap),
                        needles=1)
        inp = fw.make_inputs(w)  # every rank draws the same global inputs
        lengths = inp["lengths"]
        packed, scales = oracle.quantize_keys(inp["k"], lengths, T)
        sc = oracle.block_scores(inp["q"], packed, scales, lengths, T)
        _, gmask = oracle.select(sc, lengths, Hkv, cap, T, S, 1.0)
        nblk = cap // T
        blocks = np.array([[oracle.mask_to_blocks(gmask[b, g], nblk) for g in range(Hkv)]
                           for b in range(B)])
        sharded.check_shard_capacity(cap_local, T, S)
        ll = sharded.local_lengths(lengths, rank, cap_local)
        sl = slice(rank * cap_local, (rank + 1) * cap_local)
        m, l, acc = _partials_numpy(inp["q"], inp["k"][:, :, sl], inp["v"][:, :, sl],
                                    blocks[:, :, rank * (cap_local // T):(rank + 1) * (cap_local // T)],
                                    ll, T, S, G)
        mine = torch.from_numpy(np.concatenate([m.ravel(), l.ravel(), acc.ravel()]))
        gathered = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(gathered, mine)
        # log-sum-exp merge over every split of every shard
        parts = []
        for t in gathered:
            a = t.numpy()
            n1 = m.size
            parts.append((a[:n1].reshape(m.shape), a[n1:2 * n1].reshape(m.shape),
                          a[2 * n1:].reshape(acc.shape)))
        M = np.max(np.stack([p[0].max(axis=2) for p in parts]), axis=0)
        L = sum((p[1] * np.exp2(np.where(np.isinf(p[0]), -np.inf, p[0] - M[..., None]))).sum(axis=2)
                for p in parts)
        O = sum((p[2] * np.exp2(np.where(np.isinf(p[0]), -np.inf, p[0] - M[..., None]))[..., None]).sum(axis=2)
                for p in parts) / L[..., None]
        want, _ = oracle.attend(inp["q"], inp["k"], inp["v"], lengths, gmask, T)
        out[rank] = float(np.abs(O - want).max())
    finally:
        dist.destroy_process_group()


def test_two_rank_context_sharding_reproduces_unsharded_attention():
    world = 2
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0] < 1e-9 and out[1] < 1e-9


def _gather_worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    from sparse_long_context_ffd_b200 import sharded
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    bench.dist_init("gloo", world)
    try:
        region = torch.arange(37, dtype=torch.int64).to(torch.uint8) + 100 * rank
        got = sharded.gather_regions(region)
        out[rank] = got.numpy().copy()
    finally:
        dist.destroy_process_group()


def test_gather_regions_concatenates_in_rank_order_over_gloo():
    # the exchange step of the context-sharded decode (sharded.sharded_decode)
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_gather_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    want = np.concatenate([np.arange(37, dtype=np.uint8) + 100 * r for r in range(world)])
    assert np.array_equal(out[0], want) and np.array_equal(out[1], want)


def test_shard_bookkeeping():
    from sparse_long_context_ffd_b200 import sharded
    ll = [sharded.local_lengths([0, 100, 256, 700], r, 256) for r in range(3)]
    assert [list(x) for x in ll] == [[0, 100, 256, 256], [0, 0, 0, 256], [0, 0, 0, 188]]
    with pytest.raises(ValueError):
        sharded.check_shard_capacity(300, 64, 2)
    assert sharded.global_mask_words(3, 256, 64) == 1
