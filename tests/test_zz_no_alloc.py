"""ffd_decode_no_alloc: the decode step for callers that cannot allocate
device memory (plug-ins given only input/output buffers, loops that must not
call cudaMalloc while running).  It must give the same output and selection
mask as ffd_decode with a caller workspace, call after call, although all
calls share one built-in scratch array.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import ffd_workloads as fw
from gpu_util import GpuCase, MAX_ABS_TOL, MEAN_ABS_TOL, bf16_to_np_f32
from sparse_long_context_ffd_b200 import ffd

pytestmark = pytest.mark.gpu


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


def _case(seed, B, G, Hkv, cap, T, S, lo, hi):
    w = fw.random_small_workload(seed, B, G, Hkv, cap, T, S, 2.0, lo, hi, needles=2)
    gc = GpuCase(w, fw.make_inputs(w))
    gc.quantize(0)
    return gc


def test_no_alloc_matches_workspace_entry_point_twice_in_a_row():
    cases = [(_case(40, 3, 4, 2, 4096, 64, 7, 1, 4096), 0.75),
             (_case(41, 2, 8, 2, 8192, 128, 5, 900, 8192), 2.0)]
    for gc, delta in cases:  # two calls in a row, different shapes and deltas
        out = torch.full_like(gc.bufs.out, float("nan"))
        mask = torch.full_like(gc.bufs.mask, -1)
        got_out, got_mask = _no_alloc_call(gc, delta, out, mask)
        want_out, want_mask = gc.decode(delta)  # ffd_decode with its own workspace
        assert np.array_equal(got_mask, want_mask)
        err = np.abs(got_out - want_out)
        assert np.isfinite(got_out).all()
        assert err.max() <= MAX_ABS_TOL and err.mean() <= MEAN_ABS_TOL
    # and again on the first case: leftovers of the second call must not leak in
    gc, delta = cases[0]
    out = torch.empty_like(gc.bufs.out)
    mask = torch.empty_like(gc.bufs.mask)
    got_out, got_mask = _no_alloc_call(gc, delta, out, mask)
    want_out, want_mask = gc.decode(delta)
    assert np.array_equal(got_mask, want_mask)
    assert np.abs(got_out - want_out).max() <= MAX_ABS_TOL


def test_no_alloc_rejects_shapes_beyond_its_scratch():
    # 64 sequences x 8 kv-heads x 256K tokens in splits of 1 block needs far
    # more than 16 MiB of scratch: refused on the host, nothing launched
    s = ffd.make_shape(64, 64, 8, 262144, 64, 1)
    assert ffd.decode_workspace_bytes(s) > ffd.FFD_NO_ALLOC_SCRATCH_BYTES
    lib = ffd.load_library()
    a = 1 << 20
    rc = lib.ffd_decode_no_alloc(ctypes.byref(s), a, a, a, a, a, a, 1.0, a, a, None)
    assert rc == ffd.FFD_ERR_WORKSPACE
