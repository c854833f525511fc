"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Masks and the int4 key copy must match bit for bit; outputs must be within
max-abs 1e-2 and mean-abs 1e-3 of the oracle's fp64 attention (bf16 output,
fp32 accumulation).  Small cases span several tiles, splits and ragged
tails; the full-size cases run the same launch configuration as the bench.
"""
import math

import numpy as np
import pytest
import torch

import ffd_workloads as fw
import oracle
from gpu_util import GpuCase, assert_mask_equal, assert_output_close, to_dev_bf16
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
    (8, 1, 4, 1, 2048, 64, 1, 2048, 2048),
    (9, 2, 2, 1, 8192, 128, 40, 3000, 8192),
    # splits of a multiple of 32 blocks whose last split overhangs the capacity
    (10, 2, 4, 2, 4480, 64, 64, 1, 4480),
    (11, 3, 2, 1, 12800, 128, 32, 1, 12800),
]


def _small(case):
    seed, B, G, Hkv, cap, T, S, lo, hi = case
    w = fw.random_small_workload(seed, B, G, Hkv, cap, T, S, 2.0, lo, hi, needles=2)
    return w, fw.make_inputs(w)


def _oracle(w, inp, delta, lengths=None):
    ln = inp["lengths"] if lengths is None else lengths
    packed, scales = oracle.quantize_keys(inp["k"], ln, w.block_size)
    out, mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], packed, scales, ln,
                                 w.block_size, w.split_blocks, delta)
    return out, mask, packed, scales


# ------------------------------------------------------------- quantiser --

@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"s{c[0]}")
def test_quantize_bitexact(case):
    w, inp = _small(case)
    gc = GpuCase(w, inp)
    gc.quantize(0)
    torch.cuda.synchronize()
    packed = fw.poison_packed((w.batch, w.num_kv_heads, w.capacity, 64))
    scales = fw.poison_scales((w.batch, w.num_kv_heads, w.capacity // w.block_size, 128))
    oracle.quantize_keys(inp["k"], inp["lengths"], w.block_size, 0, packed, scales)
    assert np.array_equal(gc.packed(), packed)
    assert np.array_equal(gc.scales(), scales)


def test_quantize_append_last_block_bitexact():
    w = fw.random_small_workload(20, 3, 4, 2, 1024, 64, 4, 2.0, 200, 700)
    inp = fw.make_inputs(w)
    start = inp["lengths"].copy()
    gc = GpuCase(w, inp, lengths=start)
    gc.quantize(0)
    ln = start.copy()
    for step in range(70):  # append one token per sequence, requantise its last block
        ln = ln + 1
        gc.lengths.copy_(torch.from_numpy(ln))
        gc.quantize(ffd.FFD_LAST_BLOCK)
    torch.cuda.synchronize()
    want_p, want_s = oracle.quantize_keys(inp["k"], ln, w.block_size)
    got_p, got_s = gc.packed(), gc.scales()
    for b in range(w.batch):
        nb = -(-int(ln[b]) // w.block_size)
        assert np.array_equal(got_p[b, :, :nb * w.block_size], want_p[b, :, :nb * w.block_size])
        assert np.array_equal(got_s[b, :, :nb], want_s[b, :, :nb])


def test_quantize_subnormal_keys_saturate():
    T, cap = 64, 128
    tiny = np.float32(10 * 2.0**-133)
    k = np.full((1, 1, cap, 128), tiny, np.float32)
    k[0, 0, 1::2] = -tiny
    k[0, 0, 64:] = np.float32(3.0e-39)  # second block: other subnormal values
    kb = fw.f32_to_bf16_bits(k)
    w = fw.Workload("sub", 1, 1, 1, cap, T, 2, 1.0, 0, context=cap)
    inp = dict(q=np.zeros((1, 1, 128), np.uint16), k=kb, v=kb.copy(),
               lengths=np.array([cap], np.int32))
    gc = GpuCase(w, inp)
    gc.quantize(0)
    torch.cuda.synchronize()
    want_p, want_s = oracle.quantize_keys(kb, inp["lengths"], T)
    assert np.array_equal(gc.packed(), want_p)
    assert np.array_equal(gc.scales(), want_s)


# ---------------------------------------------------------------- decode --

@pytest.mark.parametrize("delta", [0.0, 0.75, 2.0, INF])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"s{c[0]}")
def test_decode_small(case, delta):
    w, inp = _small(case)
    want_out, want_mask, want_p, want_s = _oracle(w, inp, delta)
    gc = GpuCase(w, inp)
    gc.quantize(0)
    out, mask = gc.decode(delta)
    assert_mask_equal(mask, want_mask, f"case {case[0]} delta {delta}")
    assert_output_close(out, want_out, f"case {case[0]} delta {delta}")


@pytest.mark.parametrize("T", [64, 128])
def test_decode_edge_lengths(T):
    cap = 16 * T
    lengths = np.array([0, 1, T - 1, T, T + 1, cap - 1, cap, 5 * T + 17], np.int32)
    w = fw.Workload("edge", len(lengths), 8, 2, cap, T, 3, 1.0, 42, context=cap, needles=1)
    inp = fw.make_inputs(w, lengths=lengths)
    for delta in (0.0, 1.0, INF):
        want_out, want_mask, _, _ = _oracle(w, inp, delta)
        gc = GpuCase(w, inp)
        gc.quantize(0)
        out, mask = gc.decode(delta)
        assert_mask_equal(mask, want_mask, f"T{T} delta {delta}")
        assert_output_close(out, want_out, f"T{T} delta {delta}")
        assert not out[0].any() and not mask[0].any()  # empty sequence


def test_bad_lengths_are_flagged_on_device():
    w = fw.random_small_workload(30, 4, 4, 2, 1024, 64, 4, 2.0, 100, 1024)
    inp = fw.make_inputs(w)
    bad = inp["lengths"].copy()
    bad[1] = w.capacity + 1
    bad[3] = -5
    gc = GpuCase(w, inp)
    gc.quantize(0)
    gc.lengths.copy_(torch.from_numpy(bad))
    out, mask = gc.decode(2.0)
    flags = ffd.check_device_status(gc.bufs.workspace)
    assert flags == ffd.FFD_DEVICE_FLAG_BAD_LENGTH
    assert ffd.check_device_status(gc.bufs.workspace) == 0  # read clears it
    for b in (1, 3):
        assert not out[b].any() and not mask[b].any()
    good = [0, 2]
    want_out, want_mask, _, _ = _oracle(w, inp, 2.0)
    assert_mask_equal(mask[good], want_mask[good])
    assert_output_close(out[good], want_out[good])


def test_repeated_calls_and_graph_replay_match():
    w, inp = _small(SMALL[5])
    gc = GpuCase(w, inp)
    gc.quantize(0)
    out1, mask1 = gc.decode(0.75)
    out2, mask2 = gc.decode(0.75)  # counters were reset by the previous call
    assert np.array_equal(out1, out2) and np.array_equal(mask1, mask2)
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    gc.bufs.out.zero_()
    torch.cuda.synchronize()
    with torch.cuda.graph(graph, stream=stream):
        ffd.quantize_keys(gc.shape, gc.k, gc.lengths, ffd.FFD_LAST_BLOCK, gc.bufs.k_packed,
                          gc.bufs.k_scales)
        ffd.decode(gc.shape, gc.q, gc.k, gc.v, gc.bufs.k_packed, gc.bufs.k_scales, gc.lengths,
                   0.75, gc.bufs.out, gc.bufs.mask, gc.bufs.workspace)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    from gpu_util import bf16_to_np_f32
    assert np.array_equal(bf16_to_np_f32(gc.bufs.out).astype(np.float64), out1)
    assert np.array_equal(gc.bufs.mask.cpu().numpy().view(np.uint32), mask1)
    assert ffd.check_device_status(gc.bufs.workspace) == 0


def test_output_and_mask_buffers_not_overrun():
    w, inp = _small(SMALL[1])
    gc = GpuCase(w, inp)
    gc.quantize(0)
    n_out = gc.bufs.out.numel()
    n_mask = gc.bufs.mask.numel()
    out_big = torch.full((n_out + 64,), 1.5, dtype=torch.bfloat16, device="cuda")
    mask_big = torch.full((n_mask + 64,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    ffd.decode(gc.shape, gc.q, gc.k, gc.v, gc.bufs.k_packed, gc.bufs.k_scales, gc.lengths, 2.0,
               out_big, mask_big, gc.bufs.workspace)
    torch.cuda.synchronize()
    assert (out_big[n_out:] == 1.5).all()
    assert (mask_big[n_mask:] == 0x5A5A5A5A).all()


# ------------------------------------------------------ full-size configs --

def _full_config(name, deltas=None):
    w = fw.WORKLOADS[name]
    inp = fw.make_inputs(w)
    packed, scales = oracle.quantize_keys(inp["k"], inp["lengths"], w.block_size)
    sc = oracle.block_scores(inp["q"], packed, scales, inp["lengths"], w.block_size)
    gc = GpuCase(w, inp)
    gc.quantize(0)
    torch.cuda.synchronize()
    assert _packed_valid_equal(gc.packed(), packed, inp["lengths"], w.block_size)
    got_s = gc.scales()
    for b in range(w.batch):
        nb = -(-int(inp["lengths"][b]) // w.block_size)
        assert np.array_equal(got_s[b, :, :nb], scales[b, :, :nb])
    report = []
    for delta in deltas or [w.delta]:
        _, want_mask = oracle.select(sc, inp["lengths"], w.num_kv_heads, w.capacity,
                                     w.block_size, w.split_blocks, delta)
        want_out, _ = oracle.attend(inp["q"], inp["k"], inp["v"], inp["lengths"], want_mask,
                                    w.block_size)
        out, mask = gc.decode(delta)
        assert_mask_equal(mask, want_mask, f"{name} delta {delta}")
        mx, mean = assert_output_close(out, want_out, f"{name} delta {delta}")
        nblk = w.capacity // w.block_size
        kept = sum(int(oracle.mask_to_blocks(mask[b, g], nblk).sum())
                   for b in range(w.batch) for g in range(w.num_kv_heads))
        report.append((delta, kept, mx, mean))
    return report


def _packed_valid_equal(got, want, lengths, T):
    for b in range(len(lengths)):
        nb = -(-int(lengths[b]) // T)
        if not np.array_equal(got[b, :, :nb * T], want[b, :, :nb * T]):
            return False
    return True


@pytest.mark.parametrize("name", ["tiny", "llama", "long128k", "ragged"])
def test_full_config(name):
    rep = _full_config(name)
    print(name, rep)


def test_max256k_delta_sweep():
    rep = _full_config("max256k", list(fw.MAX256K_DELTAS))
    print("max256k", rep)


# ------------------------------------------------- fused step (append path) --

@pytest.mark.parametrize("T,delta", [(64, 2.0), (128, 0.75), (64, INF)])
def test_decode_step_equals_quantize_then_decode(T, delta):
    # inputs drawn for the final lengths; decoding starts 5 tokens earlier and
    # appends one token per step (the data past the current length is real)
    w = fw.random_small_workload(50 + T, 3, 4, 2, 32 * T, T, 5, 2.0, 6 * T, 32 * T, needles=2)
    inp = fw.make_inputs(w)
    final = inp["lengths"].copy()
    a = GpuCase(w, inp, lengths=final - 5)
    b = GpuCase(w, inp, lengths=final - 5)
    a.quantize(0)
    b.quantize(0)
    for step in range(5):
        ln = torch.from_numpy(final - 4 + step).cuda()
        a.lengths.copy_(ln)
        b.lengths.copy_(ln)
        ffd.decode_step(a.shape, a.q, a.k, a.v, a.bufs.k_packed, a.bufs.k_scales, a.lengths, delta,
                        a.bufs.out, a.bufs.mask, a.bufs.workspace)
        b.quantize(ffd.FFD_LAST_BLOCK)
        ffd.decode(b.shape, b.q, b.k, b.v, b.bufs.k_packed, b.bufs.k_scales, b.lengths, delta,
                   b.bufs.out, b.bufs.mask, b.bufs.workspace)
        torch.cuda.synchronize()
        assert torch.equal(a.bufs.out.view(torch.int16), b.bufs.out.view(torch.int16))
        assert torch.equal(a.bufs.mask, b.bufs.mask)
        assert torch.equal(a.bufs.k_packed, b.bufs.k_packed)
        assert torch.equal(a.bufs.k_scales.view(torch.int16), b.bufs.k_scales.view(torch.int16))
    want_out, want_mask, _, _ = _oracle(w, inp, delta, lengths=final)
    from gpu_util import bf16_to_np_f32
    assert_mask_equal(a.bufs.mask.cpu().numpy().view(np.uint32), want_mask, f"step T{T} {delta}")
    assert_output_close(bf16_to_np_f32(a.bufs.out).astype(np.float64), want_out, f"step T{T} {delta}")
    assert ffd.check_device_status(a.bufs.workspace) == 0


# ------------------------------------- pseudo-max reference (sink + local) --
# both pseudo-max modes: the running maximum seeded with the pseudo-max, and
# the pages' fixed threshold (the library's FFD_REFERENCE_* and the oracle's
# reference codes share their numbering)
PSEUDO_REFS = [ffd.FFD_REFERENCE_SINK_LOCAL, ffd.FFD_REFERENCE_SINK_LOCAL_FIXED]


def _ref_id(r):
    return "fixed" if r == ffd.FFD_REFERENCE_SINK_LOCAL_FIXED else "seeded"


@pytest.mark.parametrize("ref", PSEUDO_REFS, ids=_ref_id)
@pytest.mark.parametrize("delta", [0.0, 0.75, 2.0, INF])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"s{c[0]}")
def test_decode_pseudo_max_small(case, delta, ref):
    w, inp = _small(case)
    packed, scales = oracle.quantize_keys(inp["k"], inp["lengths"], w.block_size)
    want_out, want_mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], packed, scales,
                                           inp["lengths"], w.block_size, w.split_blocks, delta,
                                           reference=ref)
    gc = GpuCase(w, inp)
    gc.quantize(0)
    ffd.decode_ex(gc.shape, gc.q, gc.k, gc.v, gc.bufs.k_packed, gc.bufs.k_scales, gc.lengths,
                  delta, gc.bufs.out, gc.bufs.mask, gc.bufs.workspace, reference=ref)
    torch.cuda.synchronize()
    from gpu_util import bf16_to_np_f32
    mask = gc.bufs.mask.cpu().numpy().view(np.uint32)
    tag = f"pseudo {_ref_id(ref)} case {case[0]} delta {delta}"
    assert_mask_equal(mask, want_mask, tag)
    assert_output_close(bf16_to_np_f32(gc.bufs.out).astype(np.float64), want_out, tag)
    assert ffd.check_device_status(gc.bufs.workspace) == 0


@pytest.mark.parametrize("ref", PSEUDO_REFS, ids=_ref_id)
@pytest.mark.parametrize("T,delta", [(64, 0.5), (128, 1.5)])
def test_decode_step_pseudo_max_equals_quantize_then_decode(T, delta, ref):
    # several splits per sequence, so CTAs that do not own the last block
    # build its int4 tile themselves while the owner rewrites it
    w = fw.random_small_workload(60 + T, 3, 4, 2, 32 * T, T, 3, 2.0, 12 * T, 32 * T, needles=2)
    inp = fw.make_inputs(w)
    final = inp["lengths"].copy()
    a = GpuCase(w, inp, lengths=final - 4)
    b = GpuCase(w, inp, lengths=final - 4)
    a.quantize(0)
    b.quantize(0)
    for step in range(4):
        ln = torch.from_numpy(final - 3 + step).cuda()
        a.lengths.copy_(ln)
        b.lengths.copy_(ln)
        ffd.decode_ex(a.shape, a.q, a.k, a.v, a.bufs.k_packed, a.bufs.k_scales, a.lengths, delta,
                      a.bufs.out, a.bufs.mask, a.bufs.workspace, reference=ref, requant_last=True)
        b.quantize(ffd.FFD_LAST_BLOCK)
        ffd.decode_ex(b.shape, b.q, b.k, b.v, b.bufs.k_packed, b.bufs.k_scales, b.lengths, delta,
                      b.bufs.out, b.bufs.mask, b.bufs.workspace, reference=ref)
        torch.cuda.synchronize()
        assert torch.equal(a.bufs.out.view(torch.int16), b.bufs.out.view(torch.int16))
        assert torch.equal(a.bufs.mask, b.bufs.mask)
        assert torch.equal(a.bufs.k_packed, b.bufs.k_packed)
        assert torch.equal(a.bufs.k_scales.view(torch.int16), b.bufs.k_scales.view(torch.int16))
    packed, scales = oracle.quantize_keys(inp["k"], final, w.block_size)
    want_out, want_mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], packed, scales, final,
                                           w.block_size, w.split_blocks, delta, reference=ref)
    from gpu_util import bf16_to_np_f32
    assert_mask_equal(a.bufs.mask.cpu().numpy().view(np.uint32), want_mask, "pseudo step")
    assert_output_close(bf16_to_np_f32(a.bufs.out).astype(np.float64), want_out, "pseudo step")


@pytest.mark.parametrize("ref", PSEUDO_REFS, ids=_ref_id)
@pytest.mark.parametrize("name,delta", [("long128k", 3.0), ("max256k", 1.0), ("ragged", 3.0)])
def test_full_config_pseudo_max(name, delta, ref):
    w = fw.WORKLOADS[name]
    inp = fw.make_inputs(w)
    packed, scales = oracle.quantize_keys(inp["k"], inp["lengths"], w.block_size)
    sc = oracle.block_scores(inp["q"], packed, scales, inp["lengths"], w.block_size)
    _, want_mask = oracle.select(sc, inp["lengths"], w.num_kv_heads, w.capacity, w.block_size,
                                 w.split_blocks, delta, reference=ref)
    want_out, _ = oracle.attend(inp["q"], inp["k"], inp["v"], inp["lengths"], want_mask,
                                w.block_size)
    gc = GpuCase(w, inp)
    gc.quantize(0)
    ffd.decode_ex(gc.shape, gc.q, gc.k, gc.v, gc.bufs.k_packed, gc.bufs.k_scales, gc.lengths,
                  delta, gc.bufs.out, gc.bufs.mask, gc.bufs.workspace, reference=ref)
    torch.cuda.synchronize()
    from gpu_util import bf16_to_np_f32
    mask = gc.bufs.mask.cpu().numpy().view(np.uint32)
    tag = f"{name} pseudo {_ref_id(ref)}"
    assert_mask_equal(mask, want_mask, tag)
    mx, mean = assert_output_close(bf16_to_np_f32(gc.bufs.out).astype(np.float64), want_out, tag)
    nblk = w.capacity // w.block_size
    kept = sum(int(oracle.mask_to_blocks(mask[b, g], nblk).sum())
               for b in range(w.batch) for g in range(w.num_kv_heads))
    print(tag, "kept", kept, "max-abs", mx, "mean-abs", mean)


# ---------------------------- concentrated attention, small kept fractions --

@pytest.mark.parametrize("batch", [4, 1], ids=["one_cta_per_split", "several_ctas_per_split"])
def test_kept_fraction_and_call_history_do_not_change_results(batch):
    # The controlled-sparsity workloads (n of every 64 blocks raised above the
    # rest) at a 32K context: B4 x 8 kv-heads gives one CTA per split, B1 eight.
    # Calls alternate between 1/64 and all blocks kept on the same workspace,
    # so the cooperative selector's per-call switch (from the previous call's
    # selection bits) is exercised both ways; every call must match the oracle.
    from gpu_util import bf16_to_np_f32
    cases = []
    for name in ("rho1of64", "rho1"):
        w = fw.scaled_workload(fw.WORKLOADS[name], batch=batch, capacity=32768, context=32768)
        inp = fw.make_inputs(w)
        packed, scales = oracle.quantize_keys(inp["k"], inp["lengths"], w.block_size)
        want_out, want_mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], packed, scales,
                                               inp["lengths"], w.block_size, w.split_blocks, w.delta)
        cases.append((name, w, inp, want_out, want_mask))
    ws = None
    for name, w, inp, want_out, want_mask in cases + cases + cases[:1]:
        gc = GpuCase(w, inp)
        if ws is None:
            ws = gc.bufs.workspace
        gc.quantize(0)
        ffd.decode_ex(gc.shape, gc.q, gc.k, gc.v, gc.bufs.k_packed, gc.bufs.k_scales, gc.lengths,
                      w.delta, gc.bufs.out, gc.bufs.mask, ws, requant_last=True)
        torch.cuda.synchronize()
        mask = gc.bufs.mask.cpu().numpy().view(np.uint32)
        assert_mask_equal(mask, want_mask, f"{name} B{batch}")
        assert_output_close(bf16_to_np_f32(gc.bufs.out).astype(np.float64), want_out, f"{name} B{batch}")
        assert ffd.check_device_status(ws) == 0


@pytest.mark.parametrize("context", [16384, 32768])
@pytest.mark.parametrize("delta", [3.0, 0.5, INF])
def test_short_context_shares_splits_between_ctas(context, delta):
    # One sequence of the long-context shape at 16K / 32K: 32 / 64 (split,
    # kv-head) units, so 8 / 4 CTAs share each split (each scans all of it and
    # attends over every 8th / 4th kept block); the fused step against the
    # oracle, mask bit-exact.
    from gpu_util import bf16_to_np_f32
    w = fw.scaled_workload(fw.WORKLOADS["long128k"], capacity=context, context=context)
    inp = fw.make_inputs(w)
    packed, scales = oracle.quantize_keys(inp["k"], inp["lengths"], w.block_size)
    want_out, want_mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], packed, scales,
                                           inp["lengths"], w.block_size, w.split_blocks, delta)
    gc = GpuCase(w, inp)
    gc.quantize(0)
    for _ in range(2):  # (the second call sees the first one's selection bits)
        ffd.decode_ex(gc.shape, gc.q, gc.k, gc.v, gc.bufs.k_packed, gc.bufs.k_scales, gc.lengths,
                      delta, gc.bufs.out, gc.bufs.mask, gc.bufs.workspace, requant_last=True)
        torch.cuda.synchronize()
        assert_mask_equal(gc.bufs.mask.cpu().numpy().view(np.uint32), want_mask, f"{context} {delta}")
        assert_output_close(bf16_to_np_f32(gc.bufs.out).astype(np.float64), want_out, f"{context} {delta}")
    assert ffd.check_device_status(gc.bufs.workspace) == 0


@pytest.mark.parametrize("name", ["rho1of64", "rho0p25"])
def test_controlled_sparsity_at_full_size(name):
    # The 128K long-context shape with n of every 64 blocks raised above the
    # rest (the kept-fraction sweep's inputs, same seeds), in the launch the
    # sweep times: the fused step against the oracle, mask bit-exact.
    from gpu_util import bf16_to_np_f32
    w = fw.WORKLOADS[name]
    inp = fw.make_inputs(w)
    packed, scales = oracle.quantize_keys(inp["k"], inp["lengths"], w.block_size)
    want_out, want_mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], packed, scales, inp["lengths"],
                                           w.block_size, w.split_blocks, w.delta)
    gc = GpuCase(w, inp)
    gc.quantize(0)
    ffd.decode_ex(gc.shape, gc.q, gc.k, gc.v, gc.bufs.k_packed, gc.bufs.k_scales, gc.lengths, w.delta,
                  gc.bufs.out, gc.bufs.mask, gc.bufs.workspace, requant_last=True)
    torch.cuda.synchronize()
    assert_mask_equal(gc.bufs.mask.cpu().numpy().view(np.uint32), want_mask, name)
    assert_output_close(bf16_to_np_f32(gc.bufs.out).astype(np.float64), want_out, name)
    assert ffd.check_device_status(gc.bufs.workspace) == 0
