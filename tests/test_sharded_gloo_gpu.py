"""Context sharding through the library's own exchange path: two gloo ranks
(processes) on the one GPU each decode their shard of every sequence with
ffd_decode_partials, all-gather the workspace region that ffd_partials_region
names (sharded.gather_regions, staged through host memory for gloo), and merge
every shard's splits with ffd_merge_partials (sharded.sharded_decode).  Both
ranks must reproduce the unsharded oracle: the global mask bit for bit and the
output within tolerance.  The ranks' kernels never wait on one another; they
meet only in the host-side collective."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import ffd_workloads as fw
import oracle
from gpu_util import MAX_ABS_TOL, MEAN_ABS_TOL

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, cfg, out):
    import torch
    import torch.distributed as dist
    from gpu_util import bf16_to_np_f32, to_dev_bf16
    from sparse_long_context_ffd_b200 import ffd, sharded
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        T, S, G, Hkv, B, delta, seed = cfg
        cap_local = T * S * 3
        cap = world * cap_local
        w = fw.random_small_workload(seed, B, G, Hkv, cap, T, S, delta, 1, cap, needles=2)
        inp = fw.make_inputs(w)  # every rank draws the same global inputs
        lengths = inp["lengths"]
        local = ffd.make_shape(B, G * Hkv, Hkv, cap_local, T, S)
        sl = slice(rank * cap_local, (rank + 1) * cap_local)
        q = to_dev_bf16(inp["q"])
        k_r = to_dev_bf16(np.ascontiguousarray(inp["k"][:, :, sl]))
        v_r = to_dev_bf16(np.ascontiguousarray(inp["v"][:, :, sl]))
        ln_r = torch.from_numpy(sharded.local_lengths(lengths, rank, cap_local)).cuda()
        bufs = ffd.DecodeBuffers(local)
        ffd.quantize_keys(local, k_r, ln_r, 0, bufs.k_packed, bufs.k_scales)
        res = torch.full((B, G * Hkv, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        mask = torch.full((B, Hkv, sharded.global_mask_words(world, cap_local, T)), -1,
                          dtype=torch.int32, device="cuda")
        sharded.sharded_decode(local, q, k_r, v_r, bufs.k_packed, bufs.k_scales, ln_r,
                               torch.from_numpy(lengths).cuda(), delta, res, mask, bufs.workspace,
                               requant_last=(rank == 1))
        torch.cuda.synchronize()
        flags = ffd.check_device_status(bufs.workspace)
        out[rank] = (bf16_to_np_f32(res).astype(np.float64), mask.cpu().numpy().view(np.uint32),
                     flags)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cfg", [(64, 4, 4, 2, 3, 1.0, 95), (64, 2, 8, 1, 2, 0.5, 96),
                                 (128, 3, 2, 2, 2, float("inf"), 97)],
                         ids=["T64S4G4", "T64S2G8", "T128S3G2dense"])
def test_two_gloo_ranks_exchange_the_library_region(cfg):
    world = 2
    manager = mp.get_context("spawn").Manager()  # (this process already holds a CUDA context)
    out = manager.dict()
    mp.spawn(_rank, args=(world, _free_port(), cfg, out), nprocs=world, join=True)
    T, S, G, Hkv, B, delta, seed = cfg
    cap = world * T * S * 3
    w = fw.random_small_workload(seed, B, G, Hkv, cap, T, S, delta, 1, cap, needles=2)
    inp = fw.make_inputs(w)
    packed, scales = oracle.quantize_keys(inp["k"], inp["lengths"], T)
    want_out, want_mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], packed, scales,
                                           inp["lengths"], T, S, delta)
    for rank in range(world):
        got_out, got_mask, flags = out[rank]
        assert flags == 0
        assert np.array_equal(got_mask, want_mask), f"rank {rank}: global mask"
        assert np.isfinite(got_out).all()
        err = np.abs(got_out - want_out)
        assert err.max() <= MAX_ABS_TOL and err.mean() <= MEAN_ABS_TOL, (rank, err.max(), err.mean())
