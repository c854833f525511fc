"""Failure detection without a GPU fault.

Every pipeline wait of the decode kernel is bounded.  Here the bound is made
short (1 us, far below the time the selector needs for its first decision), so
the waits run out on their own: the kernel must flag FFD_DEVICE_FLAG_TIMEOUT,
finish (no hang, no fault: its own copies in flight are still drained under the
default limit), ffd_check_device_status must report FFD_ERR_TIMEOUT, and the
same context, workspace and buffers must then give the oracle's result."""
import ctypes

import numpy as np
import pytest
import torch

import ffd_workloads as fw
import oracle
from gpu_util import GpuCase, assert_mask_equal, assert_output_close
from sparse_long_context_ffd_b200 import ffd

pytestmark = pytest.mark.gpu


def _case():
    T, S, cap = 64, 16, 64 * 96
    lengths = np.array([cap, cap - 100], np.int32)
    w = fw.Workload("timeout", 2, 8, 2, cap, T, S, 2.0, 48, context=cap, needles=2)
    inp = fw.make_inputs(w, lengths=lengths)
    return w, inp


@pytest.mark.parametrize("fmt", ["int4", "tr"])
def test_short_wait_limit_times_out_and_the_context_recovers(fmt):
    w, inp = _case()
    gc = GpuCase(w, inp)
    T, S = w.block_size, w.split_blocks
    if fmt == "int4":
        gc.quantize(0)
        b = gc.bufs

        def run(limit):
            ffd.decode_ex(gc.shape, gc.q, gc.k, gc.v, b.k_packed, b.k_scales, gc.lengths, 2.0, b.out,
                          b.mask, b.workspace, requant_last=True, wait_limit_us=limit)
    else:
        b = ffd.ThumbResidBuffers(gc.shape)
        ffd.quantize_keys_tr(gc.shape, gc.k, gc.lengths, 0, b.k_thumb, b.k_resid, b.k_scales)

        def run(limit):
            ffd.decode_tr(gc.shape, gc.q, gc.k, gc.v, b.k_thumb, b.k_resid, b.k_scales, gc.lengths,
                          2.0, b.out, b.mask, b.workspace, requant_last=True, wait_limit_us=limit)
    assert ffd.check_device_status(b.workspace) == 0
    run(1)
    flags = ctypes.c_uint32(0)
    st = ffd.load_library().ffd_check_device_status(b.workspace.data_ptr(), ctypes.byref(flags),
                                                    torch.cuda.current_stream().cuda_stream)
    assert st == ffd.FFD_ERR_TIMEOUT
    assert flags.value & ffd.FFD_DEVICE_FLAG_TIMEOUT
    # the same context and buffers, the default limit: the oracle's result
    run(0)
    torch.cuda.synchronize()
    assert ffd.check_device_status(b.workspace) == 0
    if fmt == "int4":
        p, sc = oracle.quantize_keys(inp["k"], inp["lengths"], T)
        want_out, want_mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], p, sc, inp["lengths"],
                                               T, S, 2.0)
    else:
        th, re, sc = oracle.quantize_keys_tr(inp["k"], inp["lengths"], T)
        want_out, want_mask, _ = oracle.decode_tr(inp["q"], inp["v"], th, re, sc, inp["lengths"], T,
                                                  S, 2.0)
    mask = b.mask.cpu().numpy().view(np.uint32)
    out = b.out.float().cpu().numpy().astype(np.float64)
    assert_mask_equal(mask, want_mask, fmt)
    assert_output_close(out, want_out, fmt)
