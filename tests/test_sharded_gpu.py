"""Context sharding (sequence parallelism) on one GPU: each shard is decoded
by an independent launch of ffd_decode_partials on its slice of the cache,
the shards' partial regions are concatenated as an all-gather would, and
ffd_merge_partials must reproduce the unsharded step: the same selection
mask bit for bit, and the output within tolerance of the oracle."""
import numpy as np
import pytest
import torch

import ffd_workloads as fw
import oracle
from gpu_util import assert_mask_equal, assert_output_close, bf16_to_np_f32, to_dev_bf16
from sparse_long_context_ffd_b200 import ffd, sharded

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("W,T,S,G", [(2, 64, 4, 4), (4, 64, 3, 8), (3, 128, 2, 2), (3, 64, 1, 4)])
@pytest.mark.parametrize("delta", [0.5, 2.0, float("inf")])
def test_sharded_decode_matches_unsharded(W, T, S, G, delta):
    cap_local = T * S * (3 if S == 1 else 4)  # S = 1: 3 splits per shard, 9 in all (odd)
    cap = W * cap_local
    B, Hkv = 3, 2
    w = fw.random_small_workload(90 + W, B, G, Hkv, cap, T, S, delta, 1, cap, needles=2)
    inp = fw.make_inputs(w)
    lengths = inp["lengths"].copy()
    lengths[0] = cap_local // 2  # a sequence that lives in shard 0 only
    inp = fw.make_inputs(w, lengths=lengths)
    packed, scales = oracle.quantize_keys(inp["k"], lengths, T)
    want_out, want_mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], packed, scales, lengths,
                                           T, S, delta)
    local = ffd.make_shape(B, G * Hkv, Hkv, cap_local, T, S)
    q = to_dev_bf16(inp["q"])
    off, nbytes = ffd.partials_region(local)
    regions = []
    for r in range(W):
        k_r = to_dev_bf16(np.ascontiguousarray(inp["k"][:, :, r * cap_local:(r + 1) * cap_local]))
        v_r = to_dev_bf16(np.ascontiguousarray(inp["v"][:, :, r * cap_local:(r + 1) * cap_local]))
        ln_r = torch.from_numpy(sharded.local_lengths(lengths, r, cap_local)).cuda()
        bufs = ffd.DecodeBuffers(local)
        ffd.quantize_keys(local, k_r, ln_r, 0, bufs.k_packed, bufs.k_scales)
        ffd.decode_partials(local, q, k_r, v_r, bufs.k_packed, bufs.k_scales, ln_r, delta,
                            bufs.workspace, requant_last=(r % 2 == 1))
        regions.append(bufs.workspace[off:off + nbytes].clone())
        assert ffd.check_device_status(bufs.workspace) == 0
    gathered = torch.cat(regions)
    out = torch.full((B, G * Hkv, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    mask = torch.full((B, Hkv, sharded.global_mask_words(W, cap_local, T)), -1, dtype=torch.int32,
                      device="cuda")
    ffd.merge_partials(local, W, gathered, torch.from_numpy(lengths).cuda(), out, mask)
    torch.cuda.synchronize()
    got_mask = mask.cpu().numpy().view(np.uint32)
    assert_mask_equal(got_mask, want_mask, f"W{W} T{T} S{S} delta {delta}")
    assert_output_close(bf16_to_np_f32(out).astype(np.float64), want_out, f"W{W} delta {delta}")


@pytest.mark.parametrize("W,T,S", [(2, 64, 4), (3, 128, 2)])
@pytest.mark.parametrize("delta", [1.0, float("inf")])
def test_sharded_thumb_resid_decode_matches_unsharded(W, T, S, delta):
    # the same exchange on the 2-bit thumbnail + 8-bit residual key format
    cap_local = T * S * 4
    cap = W * cap_local
    B, Hkv, G = 3, 2, 4
    w = fw.random_small_workload(97 + W, B, G, Hkv, cap, T, S, delta, 1, cap, needles=2)
    inp = fw.make_inputs(w)
    lengths = inp["lengths"].copy()
    lengths[1] = cap_local // 3
    inp = fw.make_inputs(w, lengths=lengths)
    thumb, resid, scales = oracle.quantize_keys_tr(inp["k"], lengths, T)
    want_out, want_mask, _ = oracle.decode_tr(inp["q"], inp["v"], thumb, resid, scales, lengths, T,
                                              S, delta)
    local = ffd.make_shape(B, G * Hkv, Hkv, cap_local, T, S)
    q = to_dev_bf16(inp["q"])
    off, nbytes = ffd.partials_region(local)
    regions = []
    for r in range(W):
        sl = slice(r * cap_local, (r + 1) * cap_local)
        k_r = to_dev_bf16(np.ascontiguousarray(inp["k"][:, :, sl]))
        v_r = to_dev_bf16(np.ascontiguousarray(inp["v"][:, :, sl]))
        ln_r = torch.from_numpy(sharded.local_lengths(lengths, r, cap_local)).cuda()
        bufs = ffd.ThumbResidBuffers(local)
        ffd.quantize_keys_tr(local, k_r, ln_r, 0, bufs.k_thumb, bufs.k_resid, bufs.k_scales)
        ffd.decode_partials_tr(local, q, k_r, v_r, bufs.k_thumb, bufs.k_resid, bufs.k_scales, ln_r,
                               delta, bufs.workspace, requant_last=(r == 0))
        regions.append(bufs.workspace[off:off + nbytes].clone())
        assert ffd.check_device_status(bufs.workspace) == 0
    out = torch.full((B, G * Hkv, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    mask = torch.full((B, Hkv, sharded.global_mask_words(W, cap_local, T)), -1, dtype=torch.int32,
                      device="cuda")
    ffd.merge_partials(local, W, torch.cat(regions), torch.from_numpy(lengths).cuda(), out, mask)
    torch.cuda.synchronize()
    assert_mask_equal(mask.cpu().numpy().view(np.uint32), want_mask, f"tr W{W} delta {delta}")
    assert_output_close(bf16_to_np_f32(out).astype(np.float64), want_out, f"tr W{W} delta {delta}")


def test_sharded_entry_points_reject_bad_shapes():
    import ctypes
    lib = ffd.load_library()
    a = 1 << 20
    s = ffd.make_shape(1, 4, 1, 64 * 6, 64, 4)  # capacity not a multiple of T * S
    opts = ffd.DecodeOptions(0, 0)
    assert lib.ffd_decode_partials(ctypes.byref(s), ctypes.byref(opts), a, a, a, a, a, a, 1.0, a,
                                   1 << 20, None) == ffd.FFD_ERR_INVALID_ARG
    s = ffd.make_shape(1, 4, 1, 64 * 8, 64, 4)
    pseudo = ffd.DecodeOptions(1, 0)
    assert lib.ffd_decode_partials(ctypes.byref(s), ctypes.byref(pseudo), a, a, a, a, a, a, 1.0, a,
                                   1 << 20, None) == ffd.FFD_ERR_UNSUPPORTED
    assert lib.ffd_merge_partials(ctypes.byref(s), 0, a, 1 << 20, a, a, a, None) == ffd.FFD_ERR_INVALID_ARG
    assert lib.ffd_merge_partials(ctypes.byref(s), 2, a, 16, a, a, a, None) == ffd.FFD_ERR_WORKSPACE
