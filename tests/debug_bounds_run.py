"""Run in a process of its own (see test_debug_bounds_gpu.py).

Loads the bounds-checking debug build of the library and runs the small
parity cases on both key formats, the fused append and the pseudo-max
reference.  After each call the device flags must be clear (no index left the
extent the shape implies) and the results must match the oracle.  Exits
non-zero on the first failure; prints one summary line on success."""
import ctypes
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
sys.path.insert(0, os.path.dirname(HERE))

import ffd_workloads as fw  # noqa: E402
import oracle  # noqa: E402
from gpu_util import GpuCase, assert_mask_equal, assert_output_close  # noqa: E402
from sparse_long_context_ffd_b200 import ffd  # noqa: E402
from test_parity_gpu import SMALL, _small  # noqa: E402


def flags_clear(ws, what):
    f = ffd.check_device_status(ws)
    if f:
        raise AssertionError(f"{what}: device flags {f:#x}")


def main():
    ffd.use_debug_library()
    assert ffd.library_path().endswith("libffd_b200_debug.so")
    lib = ffd.load_library()
    # the flag path itself: a failing check reports FFD_DEVICE_FLAG_BOUNDS
    ws = torch.zeros(64, dtype=torch.int32, device="cuda")
    lib.ffd_debug_bounds_selftest.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    assert lib.ffd_debug_bounds_selftest(ws.data_ptr(), None) == ffd.FFD_OK
    assert ffd.check_device_status(ws) == ffd.FFD_DEVICE_FLAG_BOUNDS
    runs = 0
    for case in SMALL:
        w, inp = _small(case)
        T, S = w.block_size, w.split_blocks
        for delta in (0.75, 2.0, float("inf")):
            gc = GpuCase(w, inp)
            gc.quantize(0)
            out, mask = gc.decode(delta)
            flags_clear(gc.bufs.workspace, f"int4 case {case[0]} delta {delta}")
            p, sc = oracle.quantize_keys(inp["k"], inp["lengths"], T)
            want_out, want_mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], p, sc,
                                                   inp["lengths"], T, S, delta)
            assert_mask_equal(mask, want_mask, f"int4 {case[0]}")
            assert_output_close(out, want_out, f"int4 {case[0]}")
            # pseudo-max reference and the fused re-quantisation on the same buffers
            ffd.decode_ex(gc.shape, gc.q, gc.k, gc.v, gc.bufs.k_packed, gc.bufs.k_scales,
                          gc.lengths, delta, gc.bufs.out, gc.bufs.mask, gc.bufs.workspace,
                          reference=ffd.FFD_REFERENCE_SINK_LOCAL, requant_last=True)
            flags_clear(gc.bufs.workspace, f"int4 pseudo case {case[0]}")
            # the thumbnail + residual format
            b = ffd.ThumbResidBuffers(gc.shape)
            ffd.quantize_keys_tr(gc.shape, gc.k, gc.lengths, 0, b.k_thumb, b.k_resid, b.k_scales)
            ffd.decode_tr(gc.shape, gc.q, gc.k, gc.v, b.k_thumb, b.k_resid, b.k_scales, gc.lengths,
                          delta, b.out, b.mask, b.workspace, requant_last=True)
            flags_clear(b.workspace, f"tr case {case[0]} delta {delta}")
            th, re, sc2 = oracle.quantize_keys_tr(inp["k"], inp["lengths"], T)
            want_out2, want_mask2, _ = oracle.decode_tr(inp["q"], inp["v"], th, re, sc2,
                                                        inp["lengths"], T, S, delta)
            assert_mask_equal(b.mask.cpu().numpy().view(np.uint32), want_mask2, f"tr {case[0]}")
            assert_output_close(b.out.float().cpu().numpy().astype(np.float64), want_out2,
                                f"tr {case[0]}")
            runs += 4
        # the fused append: each sequence's last row written again in place
        n = inp["lengths"].astype(np.int64)
        rows = [max(int(x) - 1, 0) for x in n]
        k_new = torch.stack([gc.k[bb, :, rows[bb]] for bb in range(w.batch)]).contiguous()
        v_new = torch.stack([gc.v[bb, :, rows[bb]] for bb in range(w.batch)]).contiguous()
        ffd.decode_append(gc.shape, gc.q, k_new, v_new, gc.k, gc.v, gc.bufs.k_packed,
                          gc.bufs.k_scales, gc.lengths, 2.0, gc.bufs.out, gc.bufs.mask,
                          gc.bufs.workspace)
        flags_clear(gc.bufs.workspace, f"append case {case[0]}")
        runs += 1
    torch.cuda.synchronize()
    print(f"debug bounds run: {runs} launches on {len(SMALL)} cases, no flags", flush=True)


if __name__ == "__main__":
    main()
