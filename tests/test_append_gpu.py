"""The decode step with the KV append fused in (ffd_decode_append and its
thumbnail + residual form) against the same step on an already appended cache,
and against the oracle.

The fused launch must write the new rows into the caches and give bit-identical
output, mask and key copies to "store the rows, then decode with the last-block
re-quantisation"; the final state must match the oracle (mask bit-exact, output
within 1e-2 / 1e-3).
"""
import numpy as np
import pytest
import torch

import ffd_workloads as fw
import oracle
from gpu_util import assert_mask_equal, assert_output_close, bf16_to_np_f32, to_dev_bf16
from sparse_long_context_ffd_b200 import ffd

pytestmark = pytest.mark.gpu
INF = float("inf")
GARBAGE_BF16 = 0x40E0  # 7.0: what the append must overwrite


class Side:
    """One cache (K, V, key copies) and its output buffers."""

    def __init__(self, shape, k, v, fmt):
        self.shape, self.fmt = shape, fmt
        self.k, self.v = k, v
        self.bufs = ffd.ThumbResidBuffers(shape) if fmt == "tr" else ffd.DecodeBuffers(shape)

    def quantize(self, lengths, block_begin=0):
        if self.fmt == "tr":
            ffd.quantize_keys_tr(self.shape, self.k, lengths, block_begin, self.bufs.k_thumb,
                                 self.bufs.k_resid, self.bufs.k_scales)
        else:
            ffd.quantize_keys(self.shape, self.k, lengths, block_begin, self.bufs.k_packed,
                              self.bufs.k_scales)

    def copies(self):
        b = self.bufs
        c = [b.k_scales.view(torch.int16)]
        c += [b.k_thumb, b.k_resid] if self.fmt == "tr" else [b.k_packed]
        return c


def _run_case(w, inp, fmt, reference, delta, first_back=4, lengths_final=None):
    final = inp["lengths"] if lengths_final is None else lengths_final
    shape = ffd.make_shape(w.batch, w.num_q_heads, w.num_kv_heads, w.capacity, w.block_size,
                           w.split_blocks)
    q = to_dev_bf16(inp["q"])
    k_ref, v_ref = to_dev_bf16(inp["k"]), to_dev_bf16(inp["v"])
    start = np.maximum(final - first_back, 0).astype(np.int32)
    # the fused side's cache holds garbage from each sequence's start length on
    k_app, v_app = k_ref.clone(), v_ref.clone()
    for b in range(w.batch):
        k_app[b, :, int(start[b]):].view(torch.int16).fill_(GARBAGE_BF16)
        v_app[b, :, int(start[b]):].view(torch.int16).fill_(GARBAGE_BF16)
    a = Side(shape, k_app, v_app, fmt)
    r = Side(shape, k_ref, v_ref, fmt)
    ln = torch.from_numpy(start.copy()).cuda()
    a.quantize(ln)
    r.quantize(ln)
    for step in range(first_back):
        # a sequence already at its final length re-appends its last row
        cur = np.minimum(start + step + 1, final).astype(np.int32)
        ln.copy_(torch.from_numpy(cur))
        pos = np.maximum(cur - 1, 0)
        k_new = torch.stack([k_ref[b, :, int(pos[b])] for b in range(w.batch)]).contiguous()
        v_new = torch.stack([v_ref[b, :, int(pos[b])] for b in range(w.batch)]).contiguous()
        if fmt == "tr":
            ffd.decode_append_tr(shape, q, k_new, v_new, a.k, a.v, a.bufs.k_thumb, a.bufs.k_resid,
                                 a.bufs.k_scales, ln, delta, a.bufs.out, a.bufs.mask,
                                 a.bufs.workspace, reference=reference)
            ffd.decode_tr(shape, q, r.k, r.v, r.bufs.k_thumb, r.bufs.k_resid, r.bufs.k_scales, ln,
                          delta, r.bufs.out, r.bufs.mask, r.bufs.workspace, reference=reference,
                          requant_last=True)
        else:
            ffd.decode_append(shape, q, k_new, v_new, a.k, a.v, a.bufs.k_packed, a.bufs.k_scales,
                              ln, delta, a.bufs.out, a.bufs.mask, a.bufs.workspace,
                              reference=reference)
            ffd.decode_ex(shape, q, r.k, r.v, r.bufs.k_packed, r.bufs.k_scales, ln, delta,
                          r.bufs.out, r.bufs.mask, r.bufs.workspace, reference=reference,
                          requant_last=True)
        torch.cuda.synchronize()
        assert torch.equal(a.bufs.out.view(torch.int16), r.bufs.out.view(torch.int16)), step
        assert torch.equal(a.bufs.mask, r.bufs.mask), step
        for ca, cr in zip(a.copies(), r.copies()):
            for b in range(w.batch):
                nb = -(-int(cur[b]) // w.block_size)
                rows = nb if ca.shape[2] == w.capacity // w.block_size else nb * w.block_size
                assert torch.equal(ca[b, :, :rows], cr[b, :, :rows]), step
    # the appended rows are in the cache
    for b in range(w.batch):
        n = int(final[b])
        assert torch.equal(a.k[b, :, :n].view(torch.int16), k_ref[b, :, :n].view(torch.int16))
        assert torch.equal(a.v[b, :, :n].view(torch.int16), v_ref[b, :, :n].view(torch.int16))
        assert (a.k[b, :, n:].view(torch.int16) == GARBAGE_BF16).all() or n == int(start[b])
    assert ffd.check_device_status(a.bufs.workspace) == 0
    return a


def _oracle(w, inp, fmt, reference, delta, lengths):
    # (FFD_REFERENCE_* and the oracle's reference codes share their numbering)
    T, S = w.block_size, w.split_blocks
    if fmt == "tr":
        th, re, sc = oracle.quantize_keys_tr(inp["k"], lengths, T)
        out, mask, _ = oracle.decode_tr(inp["q"], inp["v"], th, re, sc, lengths, T, S, delta,
                                        reference=reference)
    else:
        p, sc = oracle.quantize_keys(inp["k"], lengths, T)
        out, mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], p, sc, lengths, T, S, delta,
                                     reference=reference)
    return out, mask


@pytest.mark.parametrize("fmt", ["int4", "tr"])
@pytest.mark.parametrize("T,delta,reference", [
    (64, 2.0, ffd.FFD_REFERENCE_RUNNING_MAX), (128, 0.75, ffd.FFD_REFERENCE_RUNNING_MAX),
    (64, INF, ffd.FFD_REFERENCE_RUNNING_MAX), (64, 0.5, ffd.FFD_REFERENCE_SINK_LOCAL),
    (128, 1.5, ffd.FFD_REFERENCE_SINK_LOCAL), (64, 1.0, ffd.FFD_REFERENCE_SINK_LOCAL_FIXED)])
def test_decode_append_equals_store_then_step(fmt, T, delta, reference):
    w = fw.random_small_workload(80 + T, 3, 4, 2, 32 * T, T, 3, 2.0, 12 * T, 32 * T, needles=2)
    inp = fw.make_inputs(w)
    a = _run_case(w, inp, fmt, reference, delta)
    want_out, want_mask = _oracle(w, inp, fmt, reference, delta, inp["lengths"])
    assert_mask_equal(a.bufs.mask.cpu().numpy().view(np.uint32), want_mask, f"append {fmt}")
    assert_output_close(bf16_to_np_f32(a.bufs.out).astype(np.float64), want_out, f"append {fmt}")


@pytest.mark.parametrize("fmt", ["int4", "tr"])
def test_decode_append_edge_lengths(fmt):
    # final lengths 0 (nothing appended), 1 (first token), block boundaries and a
    # full cache; the sequences append their last 3 tokens (fewer when shorter)
    T = 64
    cap = 8 * T
    final = np.array([0, 1, T, T + 1, cap], np.int32)
    w = fw.Workload("edge", len(final), 4, 2, cap, T, 3, 1.0, 43, context=cap, needles=1)
    inp = fw.make_inputs(w, lengths=final)
    a = _run_case(w, inp, fmt, ffd.FFD_REFERENCE_RUNNING_MAX, 1.0, first_back=3, lengths_final=final)
    want_out, want_mask = _oracle(w, inp, fmt, ffd.FFD_REFERENCE_RUNNING_MAX, 1.0, final)
    out = bf16_to_np_f32(a.bufs.out).astype(np.float64)
    assert_mask_equal(a.bufs.mask.cpu().numpy().view(np.uint32), want_mask, f"edge {fmt}")
    assert_output_close(out, want_out, f"edge {fmt}")
    assert not out[0].any()
