"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
CUDA path through the C ABI, and compare with the oracle."""
import numpy as np
import torch

import ffd_workloads as fw
from sparse_long_context_ffd_b200 import ffd

MAX_ABS_TOL = 1e-2   # bf16 output, fp32 accumulation
MEAN_ABS_TOL = 1e-3


def to_dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_to_np_f32(t):
    return fw.bf16_bits_to_f32(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class GpuCase:
    """Device copies of one workload's inputs plus the buffers the path needs."""

    def __init__(self, w, inp, lengths=None):
        self.w = w
        self.shape = ffd.make_shape(w.batch, w.num_q_heads, w.num_kv_heads, w.capacity,
                                    w.block_size, w.split_blocks)
        self.q = to_dev_bf16(inp["q"])
        self.k = to_dev_bf16(inp["k"])
        self.v = to_dev_bf16(inp["v"])
        ln = inp["lengths"] if lengths is None else lengths
        self.lengths = torch.from_numpy(np.ascontiguousarray(ln, dtype=np.int32)).cuda()
        self.bufs = ffd.DecodeBuffers(self.shape)
        self.bufs.k_packed.fill_(fw.PACKED_POISON_BYTE)
        self.bufs.k_scales.view(torch.int16).fill_(fw.SCALE_POISON_BF16)
        self.bufs.out.view(torch.int16).fill_(0x7FC1)  # NaN canary: must be overwritten
        self.bufs.mask.fill_(-1)

    def quantize(self, block_begin=0):
        ffd.quantize_keys(self.shape, self.k, self.lengths, block_begin, self.bufs.k_packed,
                          self.bufs.k_scales)

    def decode(self, delta):
        ffd.decode(self.shape, self.q, self.k, self.v, self.bufs.k_packed, self.bufs.k_scales,
                   self.lengths, delta, self.bufs.out, self.bufs.mask, self.bufs.workspace)
        torch.cuda.synchronize()
        return (bf16_to_np_f32(self.bufs.out).astype(np.float64),
                self.bufs.mask.cpu().numpy().view(np.uint32))

    def packed(self):
        return self.bufs.k_packed.cpu().numpy()

    def scales(self):
        return u16(self.bufs.k_scales)


def assert_mask_equal(got, want, tag=""):
    if not np.array_equal(got, want):
        idx = np.argwhere(got != want)[0]
        raise AssertionError(f"{tag}: mask differs at {tuple(idx)}: got {got[tuple(idx)]:#010x} "
                             f"want {want[tuple(idx)]:#010x} ({len(np.argwhere(got != want))} words)")


def assert_output_close(got, want, tag=""):
    assert np.isfinite(got).all(), f"{tag}: non-finite output"
    err = np.abs(got - want)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (
        f"{tag}: max-abs {mx:.3e} (tol {MAX_ABS_TOL}), mean-abs {mean:.3e} (tol {MEAN_ABS_TOL}), "
        f"worst at {np.unravel_index(err.argmax(), err.shape)}")
    return mx, mean
