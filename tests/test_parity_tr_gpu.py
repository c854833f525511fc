"""Parity of the thumbnail + residual path (2-bit thumbnails, 8-bit residuals)
with the CPU oracle, through the C ABI.

Thumbnails, residuals, scales and masks must match bit for bit; outputs must
be within max-abs 1e-2 and mean-abs 1e-3 of the oracle's fp64 attention over
the reconstructed keys.
"""
import numpy as np
import pytest
import torch

import ffd_workloads as fw
import oracle
from gpu_util import assert_mask_equal, assert_output_close, bf16_to_np_f32, to_dev_bf16, u16
from sparse_long_context_ffd_b200 import ffd

pytestmark = pytest.mark.gpu
INF = float("inf")

# (seed, batch, group, kv_heads, capacity, block, split, len_lo, len_hi)
SMALL = [
    (0, 1, 4, 1, 1024, 64, 4, 1024, 1024),
    (1, 3, 4, 2, 2048, 64, 3, 1, 2048),
    (2, 2, 8, 1, 2048, 64, 16, 700, 2048),
    (3, 2, 1, 3, 1536, 64, 5, 1, 1536),
    (4, 2, 2, 2, 2048, 128, 2, 1, 2048),
    (5, 3, 8, 2, 4096, 128, 7, 100, 4096),
    (6, 1, 4, 2, 8192, 64, 64, 5000, 8192),
    (7, 2, 4, 1, 4096, 64, 33, 1, 4096),
    (10, 2, 4, 2, 4480, 64, 64, 1, 4480),
    # splits longer than 4096 tokens: the sparse steps keep the stage layout
    # with thumbnail and scale rows inside the stage
    (11, 1, 4, 2, 10240, 64, 80, 1, 10240),
]

THUMB_POISON = 0x5A
RESID_POISON = 0xA5


def _small(case):
    seed, B, G, Hkv, cap, T, S, lo, hi = case
    w = fw.random_small_workload(seed, B, G, Hkv, cap, T, S, 2.0, lo, hi, needles=2)
    return w, fw.make_inputs(w)


class TrCase:
    """Device inputs and buffers of the thumbnail + residual path."""

    def __init__(self, w, inp, lengths=None):
        self.w = w
        self.shape = ffd.make_shape(w.batch, w.num_q_heads, w.num_kv_heads, w.capacity,
                                    w.block_size, w.split_blocks)
        self.q = to_dev_bf16(inp["q"])
        self.k = to_dev_bf16(inp["k"])
        self.v = to_dev_bf16(inp["v"])
        ln = inp["lengths"] if lengths is None else lengths
        self.lengths = torch.from_numpy(np.ascontiguousarray(ln, dtype=np.int32)).cuda()
        self.bufs = ffd.ThumbResidBuffers(self.shape)
        self.bufs.k_thumb.fill_(THUMB_POISON)
        self.bufs.k_resid.fill_(RESID_POISON)
        self.bufs.k_scales.view(torch.int16).fill_(fw.SCALE_POISON_BF16)
        self.bufs.out.view(torch.int16).fill_(0x7FC1)  # NaN canary
        self.bufs.mask.fill_(-1)

    def quantize(self, block_begin=0):
        ffd.quantize_keys_tr(self.shape, self.k, self.lengths, block_begin, self.bufs.k_thumb,
                             self.bufs.k_resid, self.bufs.k_scales)

    def decode(self, delta, reference=ffd.FFD_REFERENCE_RUNNING_MAX, requant_last=False, k=None):
        ffd.decode_tr(self.shape, self.q, self.k if requant_last else k, self.v, self.bufs.k_thumb,
                      self.bufs.k_resid, self.bufs.k_scales, self.lengths, delta, self.bufs.out,
                      self.bufs.mask, self.bufs.workspace, reference=reference,
                      requant_last=requant_last)
        torch.cuda.synchronize()
        return (bf16_to_np_f32(self.bufs.out).astype(np.float64),
                self.bufs.mask.cpu().numpy().view(np.uint32))

    def copies(self):
        return (self.bufs.k_thumb.cpu().numpy(), self.bufs.k_resid.cpu().numpy(),
                u16(self.bufs.k_scales))


def _oracle_copies(w, k, lengths):
    shape = (w.batch, w.num_kv_heads, w.capacity)
    thumb = np.full(shape + (32,), THUMB_POISON, np.uint8)
    resid = np.full(shape + (128,), RESID_POISON, np.uint8)
    scales = fw.poison_scales((w.batch, w.num_kv_heads, w.capacity // w.block_size, 128))
    oracle.quantize_keys_tr(k, lengths, w.block_size, 0, thumb, resid, scales)
    return thumb, resid, scales


# ------------------------------------------------------------- quantiser --

@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"s{c[0]}")
def test_quantize_tr_bitexact(case):
    w, inp = _small(case)
    tc = TrCase(w, inp)
    tc.quantize(0)
    torch.cuda.synchronize()
    want = _oracle_copies(w, inp["k"], inp["lengths"])
    for got, exp, name in zip(tc.copies(), want, ("thumb", "resid", "scales")):
        assert np.array_equal(got, exp), name


def test_quantize_tr_append_last_block_bitexact():
    w = fw.random_small_workload(21, 3, 4, 2, 1024, 64, 4, 2.0, 200, 700)
    inp = fw.make_inputs(w)
    ln = inp["lengths"].copy()
    tc = TrCase(w, inp, lengths=ln)
    tc.quantize(0)
    for _ in range(70):
        ln = ln + 1
        tc.lengths.copy_(torch.from_numpy(ln))
        tc.quantize(ffd.FFD_LAST_BLOCK)
    torch.cuda.synchronize()
    want = oracle.quantize_keys_tr(inp["k"], ln, w.block_size)
    got = tc.copies()
    T = w.block_size
    for b in range(w.batch):
        nb = -(-int(ln[b]) // T)
        assert np.array_equal(got[0][b, :, :nb * T], want[0][b, :, :nb * T])
        assert np.array_equal(got[1][b, :, :nb * T], want[1][b, :, :nb * T])
        assert np.array_equal(got[2][b, :, :nb], want[2][b, :, :nb])


def test_quantize_tr_subnormal_and_extreme_keys():
    T, cap = 64, 192
    k = np.zeros((1, 1, cap, 128), np.float32)
    k[0, 0, :64] = np.float32(2 * 2.0**-133)   # saturating code and residual
    k[0, 0, 1:64:2] *= -1
    k[0, 0, 64:128] = np.float32(3.0e-39)      # other subnormals
    rng = np.random.default_rng(5)
    k[0, 0, 128:] = rng.standard_normal((64, 128)).astype(np.float32) * 1e30
    kb = fw.f32_to_bf16_bits(k)
    w = fw.Workload("sub", 1, 1, 1, cap, T, 2, 1.0, 0, context=cap)
    inp = dict(q=np.zeros((1, 1, 128), np.uint16), k=kb, v=kb.copy(),
               lengths=np.array([cap], np.int32))
    tc = TrCase(w, inp)
    tc.quantize(0)
    torch.cuda.synchronize()
    want = oracle.quantize_keys_tr(kb, inp["lengths"], T)
    for got, exp, name in zip(tc.copies(), want, ("thumb", "resid", "scales")):
        assert np.array_equal(got, exp), name


# ---------------------------------------------------------------- decode --

@pytest.mark.parametrize("delta", [0.0, 0.75, 2.0, INF])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"s{c[0]}")
def test_decode_tr_small(case, delta):
    w, inp = _small(case)
    thumb, resid, scales = oracle.quantize_keys_tr(inp["k"], inp["lengths"], w.block_size)
    want_out, want_mask, _ = oracle.decode_tr(inp["q"], inp["v"], thumb, resid, scales,
                                              inp["lengths"], w.block_size, w.split_blocks, delta)
    tc = TrCase(w, inp)
    tc.quantize(0)
    out, mask = tc.decode(delta)
    assert_mask_equal(mask, want_mask, f"tr case {case[0]} delta {delta}")
    assert_output_close(out, want_out, f"tr case {case[0]} delta {delta}")
    assert ffd.check_device_status(tc.bufs.workspace) == 0


@pytest.mark.parametrize("ref", [ffd.FFD_REFERENCE_SINK_LOCAL, ffd.FFD_REFERENCE_SINK_LOCAL_FIXED],
                         ids=["seeded", "fixed"])
@pytest.mark.parametrize("delta", [0.0, 1.0, 3.0])
@pytest.mark.parametrize("case", SMALL[:6], ids=lambda c: f"s{c[0]}")
def test_decode_tr_pseudo_max_small(case, delta, ref):
    # (the library's FFD_REFERENCE_* and the oracle's reference codes share
    # their numbering)
    w, inp = _small(case)
    thumb, resid, scales = oracle.quantize_keys_tr(inp["k"], inp["lengths"], w.block_size)
    want_out, want_mask, _ = oracle.decode_tr(inp["q"], inp["v"], thumb, resid, scales,
                                              inp["lengths"], w.block_size, w.split_blocks, delta,
                                              reference=ref)
    tc = TrCase(w, inp)
    tc.quantize(0)
    out, mask = tc.decode(delta, reference=ref)
    assert_mask_equal(mask, want_mask, f"tr pseudo {ref} case {case[0]} delta {delta}")
    assert_output_close(out, want_out, f"tr pseudo {ref} case {case[0]} delta {delta}")


@pytest.mark.parametrize("T", [64, 128])
def test_decode_tr_edge_lengths(T):
    cap = 16 * T
    lengths = np.array([0, 1, T - 1, T, T + 1, cap - 1, cap, 5 * T + 17], np.int32)
    w = fw.Workload("edge", len(lengths), 8, 2, cap, T, 3, 1.0, 42, context=cap, needles=1)
    inp = fw.make_inputs(w, lengths=lengths)
    thumb, resid, scales = oracle.quantize_keys_tr(inp["k"], lengths, T)
    for delta in (0.0, 1.0, INF):
        want_out, want_mask, _ = oracle.decode_tr(inp["q"], inp["v"], thumb, resid, scales,
                                                  lengths, T, 3, delta)
        tc = TrCase(w, inp)
        tc.quantize(0)
        out, mask = tc.decode(delta)
        assert_mask_equal(mask, want_mask, f"tr T{T} delta {delta}")
        assert_output_close(out, want_out, f"tr T{T} delta {delta}")
        assert not out[0].any() and not mask[0].any()


def test_decode_tr_bad_lengths_flagged_and_graph_replay():
    w, inp = _small(SMALL[5])
    tc = TrCase(w, inp)
    tc.quantize(0)
    out1, mask1 = tc.decode(0.75)
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    tc.bufs.out.zero_()
    torch.cuda.synchronize()
    with torch.cuda.graph(graph, stream=stream):
        ffd.decode_tr(tc.shape, tc.q, tc.k, tc.v, tc.bufs.k_thumb, tc.bufs.k_resid,
                      tc.bufs.k_scales, tc.lengths, 0.75, tc.bufs.out, tc.bufs.mask,
                      tc.bufs.workspace, requant_last=True)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert np.array_equal(bf16_to_np_f32(tc.bufs.out).astype(np.float64), out1)
    assert np.array_equal(tc.bufs.mask.cpu().numpy().view(np.uint32), mask1)
    assert ffd.check_device_status(tc.bufs.workspace) == 0
    bad = inp["lengths"].copy()
    bad[1] = w.capacity + 1
    tc.lengths.copy_(torch.from_numpy(bad))
    out, mask = tc.decode(2.0)
    assert ffd.check_device_status(tc.bufs.workspace) == ffd.FFD_DEVICE_FLAG_BAD_LENGTH
    assert not out[1].any() and not mask[1].any()


@pytest.mark.parametrize("T,delta,reference", [
    (64, 2.0, ffd.FFD_REFERENCE_RUNNING_MAX), (128, 0.75, ffd.FFD_REFERENCE_RUNNING_MAX),
    (64, INF, ffd.FFD_REFERENCE_RUNNING_MAX), (64, 0.5, ffd.FFD_REFERENCE_SINK_LOCAL),
    (128, 1.5, ffd.FFD_REFERENCE_SINK_LOCAL), (64, 1.0, ffd.FFD_REFERENCE_SINK_LOCAL_FIXED)])
def test_decode_tr_step_equals_quantize_then_decode(T, delta, reference):
    # several splits per sequence; decoding starts 4 tokens early and appends
    # one token per step, re-quantising the last block inside the launch
    w = fw.random_small_workload(70 + T, 3, 4, 2, 32 * T, T, 3, 2.0, 12 * T, 32 * T, needles=2)
    inp = fw.make_inputs(w)
    final = inp["lengths"].copy()
    a = TrCase(w, inp, lengths=final - 4)
    b = TrCase(w, inp, lengths=final - 4)
    a.quantize(0)
    b.quantize(0)
    for step in range(4):
        ln = torch.from_numpy(final - 3 + step).cuda()
        a.lengths.copy_(ln)
        b.lengths.copy_(ln)
        a.decode(delta, reference=reference, requant_last=True)
        b.quantize(ffd.FFD_LAST_BLOCK)
        b.decode(delta, reference=reference)
        assert torch.equal(a.bufs.out.view(torch.int16), b.bufs.out.view(torch.int16))
        assert torch.equal(a.bufs.mask, b.bufs.mask)
        assert torch.equal(a.bufs.k_thumb, b.bufs.k_thumb)
        assert torch.equal(a.bufs.k_resid, b.bufs.k_resid)
        assert torch.equal(a.bufs.k_scales.view(torch.int16), b.bufs.k_scales.view(torch.int16))
    thumb, resid, scales = oracle.quantize_keys_tr(inp["k"], final, T)
    want_out, want_mask, _ = oracle.decode_tr(inp["q"], inp["v"], thumb, resid, scales, final, T,
                                              w.split_blocks, delta, reference=reference)
    assert_mask_equal(a.bufs.mask.cpu().numpy().view(np.uint32), want_mask, "tr step")
    assert_output_close(bf16_to_np_f32(a.bufs.out).astype(np.float64), want_out, "tr step")
    assert ffd.check_device_status(a.bufs.workspace) == 0


# ------------------------------------------------------ full-size configs --

@pytest.mark.parametrize("name,deltas", [
    ("tiny", None), ("llama", None), ("long128k", None), ("ragged", None),
    ("max256k", list(fw.MAX256K_DELTAS))])
def test_decode_tr_full_config(name, deltas):
    w = fw.WORKLOADS[name]
    inp = fw.make_inputs(w)
    T = w.block_size
    thumb, resid, scales = oracle.quantize_keys_tr(inp["k"], inp["lengths"], T)
    sc = oracle.block_scores_tr(inp["q"], thumb, scales, inp["lengths"], T)
    tc = TrCase(w, inp)
    tc.quantize(0)
    torch.cuda.synchronize()
    got = tc.copies()
    for b in range(w.batch):
        nb = -(-int(inp["lengths"][b]) // T)
        assert np.array_equal(got[0][b, :, :nb * T], thumb[b, :, :nb * T])
        assert np.array_equal(got[1][b, :, :nb * T], resid[b, :, :nb * T])
        assert np.array_equal(got[2][b, :, :nb], scales[b, :, :nb])
    nblk = w.capacity // T
    for delta in deltas or [w.delta]:
        _, want_mask = oracle.select(sc, inp["lengths"], w.num_kv_heads, w.capacity, T,
                                     w.split_blocks, delta)
        want_out, _ = oracle.attend_tr(inp["q"], thumb, resid, scales, inp["v"], inp["lengths"],
                                       want_mask, T)
        out, mask = tc.decode(delta)
        assert_mask_equal(mask, want_mask, f"tr {name} delta {delta}")
        mx, mean = assert_output_close(out, want_out, f"tr {name} delta {delta}")
        kept = sum(int(oracle.mask_to_blocks(mask[b, g], nblk).sum())
                   for b in range(w.batch) for g in range(w.num_kv_heads))
        print("tr", name, delta, "kept", kept, "max-abs", mx, "mean-abs", mean)


@pytest.mark.parametrize("delta", [3.0, INF])
def test_decode_tr_short_context_shares_splits_between_ctas(delta):
    # one 16K sequence of the long-context shape: 8 CTAs share each split
    w = fw.scaled_workload(fw.WORKLOADS["long128k"], capacity=16384, context=16384)
    inp = fw.make_inputs(w)
    thumb, resid, scales = oracle.quantize_keys_tr(inp["k"], inp["lengths"], w.block_size)
    want_out, want_mask, _ = oracle.decode_tr(inp["q"], inp["v"], thumb, resid, scales, inp["lengths"],
                                              w.block_size, w.split_blocks, delta)
    tc = TrCase(w, inp)
    tc.quantize(0)
    out, mask = tc.decode(delta, requant_last=True)
    assert_mask_equal(mask, want_mask, f"tr 16K {delta}")
    assert_output_close(out, want_out, f"tr 16K {delta}")
    assert ffd.check_device_status(tc.bufs.workspace) == 0


@pytest.mark.parametrize("batch", [4, 1])
def test_decode_tr_kept_fraction_and_call_history_do_not_change_results(batch):
    # The controlled-sparsity workloads at a 32K context on one workspace,
    # calls alternating between 1/64 and all blocks kept: the sparse variant's
    # per-call helper switch (from the previous call's selection bits; the
    # thumbnail format helps below 1/8 kept) runs both ways, with one CTA per
    # split (B4) and two (B1).  Every call must match the oracle.
    cases = []
    for name in ("rho1of64", "rho1"):
        w = fw.scaled_workload(fw.WORKLOADS[name], batch=batch, capacity=32768, context=32768)
        inp = fw.make_inputs(w)
        thumb, resid, scales = oracle.quantize_keys_tr(inp["k"], inp["lengths"], w.block_size)
        want_out, want_mask, _ = oracle.decode_tr(inp["q"], inp["v"], thumb, resid, scales,
                                                  inp["lengths"], w.block_size, w.split_blocks, w.delta)
        cases.append((name, w, inp, want_out, want_mask))
    ws = None
    for name, w, inp, want_out, want_mask in cases + cases + cases[:1]:
        tc = TrCase(w, inp)
        if ws is None:
            ws = tc.bufs.workspace
        tc.quantize(0)
        ffd.decode_tr(tc.shape, tc.q, tc.k, tc.v, tc.bufs.k_thumb, tc.bufs.k_resid, tc.bufs.k_scales,
                      tc.lengths, w.delta, tc.bufs.out, tc.bufs.mask, ws, requant_last=True)
        torch.cuda.synchronize()
        out = bf16_to_np_f32(tc.bufs.out).astype(np.float64)
        mask = tc.bufs.mask.cpu().numpy().view(np.uint32)
        assert_mask_equal(mask, want_mask, f"tr {name} B{batch}")
        assert_output_close(out, want_out, f"tr {name} B{batch}")
        assert ffd.check_device_status(ws) == 0


@pytest.mark.parametrize("name", ["rho1of64", "rho0p25"])
def test_decode_tr_controlled_sparsity_at_full_size(name):
    # The kept-fraction sweep's thumbnail rows at full size (128K, same
    # seeds): the fused step against the oracle, mask bit-exact.
    w = fw.WORKLOADS[name]
    inp = fw.make_inputs(w)
    thumb, resid, scales = oracle.quantize_keys_tr(inp["k"], inp["lengths"], w.block_size)
    want_out, want_mask, _ = oracle.decode_tr(inp["q"], inp["v"], thumb, resid, scales, inp["lengths"],
                                              w.block_size, w.split_blocks, w.delta)
    tc = TrCase(w, inp)
    tc.quantize(0)
    out, mask = tc.decode(w.delta, requant_last=True)
    assert_mask_equal(mask, want_mask, f"tr {name}")
    assert_output_close(out, want_out, f"tr {name}")
    assert ffd.check_device_status(tc.bufs.workspace) == 0
