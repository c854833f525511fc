"""Context (sequence) sharding of the decode step across GPUs.

Rank r of W holds global tokens [r * cap_local, (r + 1) * cap_local) of every
sequence; cap_local is a multiple of block_size * split_blocks, so every
split lies in one shard and its Top-delta selection equals the unsharded one.
A step is: ffd_decode_partials on the local shard, an all-gather of the
partials region over NCCL (NVLink / NVSwitch; a gloo group stages it through
host memory), and ffd_merge_partials.  The
exchange is B * Hkv * nsplit * G * 528 bytes per rank, so sharding pays only
when a single GPU's step is long (about 1M tokens and more).
"""
from __future__ import annotations

import numpy as np

from . import ffd


def local_lengths(global_lengths, rank: int, cap_local: int) -> np.ndarray:
    """Valid tokens of each sequence in shard `rank`."""
    g = np.asarray(global_lengths, dtype=np.int64)
    return np.clip(g - rank * cap_local, 0, cap_local).astype(np.int32)


def check_shard_capacity(cap_local: int, block_size: int, split_blocks: int) -> None:
    if cap_local <= 0 or cap_local % (block_size * split_blocks) != 0:
        raise ValueError("the shard capacity must be a positive multiple of "
                         "block_size * split_blocks (shards start at split boundaries)")


def global_mask_words(num_shards: int, cap_local: int, block_size: int) -> int:
    return (num_shards * (cap_local // block_size) + 31) // 32


def gather_regions(region, group=None):
    """All-gather one rank's partials region (a uint8 tensor) from every rank
    of `group`, concatenated in rank order, on the region's device.  NCCL
    gathers device memory directly (NVLink / NVSwitch); a gloo group, which
    moves host memory only, stages the region through host memory."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    n = region.numel()
    if dist.get_backend(group) == "nccl":
        gathered = torch.empty(world * n, dtype=torch.uint8, device=region.device)
        dist.all_gather_into_tensor(gathered, region, group=group)
        return gathered
    host = region.detach().to("cpu")
    gathered = torch.empty(world * n, dtype=torch.uint8)
    dist.all_gather_into_tensor(gathered, host, group=group)
    return gathered.to(region.device)


def sharded_decode(local_shape, q, k_local, v_local, packed_local, scales_local,
                   local_lengths_dev, global_lengths_dev, delta: float, out, mask_global,
                   workspace, group=None, requant_last: bool = False) -> None:
    """One decode step over context shards (one rank per GPU): the local
    split partials, their all-gather (gather_regions: NCCL, or gloo through
    host memory) and the merge of every shard's splits into `out` and the
    global mask."""
    import torch.distributed as dist
    check_shard_capacity(local_shape.capacity, local_shape.block_size, local_shape.split_blocks)
    world = dist.get_world_size(group)
    ffd.decode_partials(local_shape, q, k_local, v_local, packed_local, scales_local,
                        local_lengths_dev, delta, workspace, requant_last=requant_last)
    off, nbytes = ffd.partials_region(local_shape)
    gathered = gather_regions(workspace[off:off + nbytes], group)
    ffd.merge_partials(local_shape, world, gathered, global_lengths_dev, out, mask_global)
