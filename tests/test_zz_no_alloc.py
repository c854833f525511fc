"""ffd_decode_no_alloc: the decode step for callers that cannot allocate
device memory (plug-ins given only input/output buffers, loops that must not
call cudaMalloc while running).  It must give the oracle's selection mask and
output, and the same results as ffd_decode with a caller workspace, call after
call, although all calls share one built-in scratch array that keeps what the
previous call left.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import ffd_workloads as fw
import oracle
from gpu_util import GpuCase, MAX_ABS_TOL, MEAN_ABS_TOL, bf16_to_np_f32
from sparse_long_context_ffd_b200 import ffd

pytestmark = pytest.mark.gpu

INF = float("inf")


def _no_alloc_call(gc, delta, out, mask):
    lib = ffd.load_library()
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.ffd_decode_no_alloc(ctypes.byref(gc.shape), gc.q.data_ptr(), gc.k.data_ptr(),
                                 gc.v.data_ptr(), gc.bufs.k_packed.data_ptr(),
                                 gc.bufs.k_scales.data_ptr(), gc.lengths.data_ptr(), float(delta),
                                 out.data_ptr(), mask.data_ptr(), stream)
    assert rc == ffd.FFD_OK, ffd.status_string(rc)
    torch.cuda.synchronize()
    return (bf16_to_np_f32(out).astype(np.float64), mask.cpu().numpy().view(np.uint32).copy())


def _case(seed, B, G, Hkv, cap, T, S, lo, hi, lengths=None):
    w = fw.random_small_workload(seed, B, G, Hkv, cap, T, S, 2.0, lo, hi, needles=2)
    inp = fw.make_inputs(w, lengths=lengths)
    gc = GpuCase(w, inp)
    gc.quantize(0)
    gc.inp = inp
    return gc


def _oracle(gc, delta):
    w, inp = gc.w, gc.inp
    packed, scales = oracle.quantize_keys(inp["k"], inp["lengths"], w.block_size)
    out, mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], packed, scales, inp["lengths"],
                                 w.block_size, w.split_blocks, delta)
    return out, mask


def _check(gc, delta, got_out, got_mask, tag):
    want_out, want_mask = _oracle(gc, delta)
    assert np.array_equal(got_mask, want_mask), f"{tag}: mask differs from the oracle"
    assert np.isfinite(got_out).all(), tag
    err = np.abs(got_out - want_out)
    assert err.max() <= MAX_ABS_TOL and err.mean() <= MEAN_ABS_TOL, (tag, err.max(), err.mean())
    # and the workspace entry point on the same inputs
    ws_out, ws_mask = gc.decode(delta)
    assert np.array_equal(got_mask, ws_mask), tag
    err = np.abs(got_out - ws_out)
    assert err.max() <= MAX_ABS_TOL and err.mean() <= MEAN_ABS_TOL, (tag, err.max(), err.mean())


def _dirty_call(gc, delta, tag):
    out = torch.full_like(gc.bufs.out, float("nan"))
    mask = torch.full_like(gc.bufs.mask, -1)
    got_out, got_mask = _no_alloc_call(gc, delta, out, mask)
    assert ffd.no_alloc_device_status() == 0, tag
    _check(gc, delta, got_out, got_mask, tag)


def test_no_alloc_matches_oracle_and_workspace_entry_point_call_after_call():
    T = 64
    cases = [
        (_case(40, 3, 4, 2, 4096, 64, 7, 1, 4096), 0.75, "ragged S7"),
        (_case(41, 2, 8, 2, 8192, 128, 5, 900, 8192), 2.0, "T128 S5"),
        # a bigger array footprint first, then splits of 32 blocks (each split
        # writes whole mask words, the last one clears the words past it) on
        # what the earlier calls left behind
        (_case(42, 4, 4, 4, 16384, 64, 3, 8000, 16384), 1.0, "wide S3"),
        (_case(43, 3, 4, 2, 8192, 64, 32, 100, 8192), 1.5, "ragged S32"),
        (_case(44, 2, 4, 2, 4096, 64, 16, 1, 4096), INF, "dense"),
        (_case(45, 5, 4, 2, 8 * T, T, 3, 1, 8 * T,
               lengths=np.array([0, 1, T, T + 1, 8 * T], np.int32)), 1.0, "edge lengths"),
    ]
    for gc, delta, tag in cases:  # calls in a row, different shapes and deltas
        _dirty_call(gc, delta, tag)
    # and again on the first cases: leftovers of the later calls must not leak in
    for gc, delta, tag in cases[:2]:
        _dirty_call(gc, delta, tag + " again")


def test_no_alloc_clears_what_precedes_the_split_bits():
    # each call clears the scratch prefix before the split bits; the error word
    # (offset 0) and one arrival counter per (sequence, kv-head) must lie in it
    for B, Hkv, cap, T, S in ((3, 2, 4096, 64, 7), (16, 8, 65536, 64, 32), (64, 8, 4096, 64, 1)):
        s = ffd.make_shape(B, 4 * Hkv, Hkv, cap, T, S)
        off, _ = ffd.partials_region(s)
        assert off >= 4 + B * Hkv * 4, (B, Hkv, off)


def test_no_alloc_reports_device_flags():
    # a length beyond the capacity: zero rows and an empty mask for that
    # sequence, and the flag read from the built-in array; the next good call
    # starts clean
    gc = _case(46, 3, 4, 2, 4096, 64, 7, 1, 4096)
    good = gc.lengths.clone()
    gc.lengths[1] = 4096 + 64
    out = torch.full_like(gc.bufs.out, float("nan"))
    mask = torch.full_like(gc.bufs.mask, -1)
    got_out, got_mask = _no_alloc_call(gc, 1.0, out, mask)
    assert ffd.no_alloc_device_status() == ffd.FFD_DEVICE_FLAG_BAD_LENGTH
    assert not got_out[1].any() and not got_mask[1].any()
    assert ffd.no_alloc_device_status() == 0  # read and cleared
    gc.lengths.copy_(good)
    _dirty_call(gc, 1.0, "after a flagged call")


def test_no_alloc_rejected_call_leaves_the_array_alone():
    # a call that fails its host checks launches nothing and clears nothing:
    # the flag of the previous call is still there to read
    gc = _case(47, 2, 4, 2, 4096, 64, 7, 1, 4096)
    gc.lengths[0] = 4096 + 1
    out = torch.empty_like(gc.bufs.out)
    mask = torch.empty_like(gc.bufs.mask)
    _no_alloc_call(gc, 1.0, out, mask)
    lib = ffd.load_library()
    rc = lib.ffd_decode_no_alloc(ctypes.byref(gc.shape), gc.q.data_ptr(), gc.k.data_ptr(),
                                 gc.v.data_ptr(), gc.bufs.k_packed.data_ptr(),
                                 gc.bufs.k_scales.data_ptr(), gc.lengths.data_ptr(), -1.0,
                                 out.data_ptr(), mask.data_ptr(), None)
    assert rc == ffd.FFD_ERR_INVALID_ARG  # negative delta
    assert ffd.no_alloc_device_status() == ffd.FFD_DEVICE_FLAG_BAD_LENGTH


def test_no_alloc_rejects_shapes_beyond_its_scratch():
    # 64 sequences x 8 kv-heads x 256K tokens in splits of 1 block needs far
    # more than 16 MiB of scratch: refused on the host, nothing launched
    s = ffd.make_shape(64, 64, 8, 262144, 64, 1)
    assert ffd.decode_workspace_bytes(s) > ffd.FFD_NO_ALLOC_SCRATCH_BYTES
    lib = ffd.load_library()
    a = 1 << 20
    rc = lib.ffd_decode_no_alloc(ctypes.byref(s), a, a, a, a, a, a, 1.0, a, a, None)
    assert rc == ffd.FFD_ERR_WORKSPACE
