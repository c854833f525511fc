"""Edge cases of the method on the GPU against the oracle: the largest split
the library accepts, scores that all tie (the inclusive Top-delta test at
delta = 0), a zero query, and single-token sequences with the largest group."""
import numpy as np
import pytest
import torch

import ffd_workloads as fw
import oracle
from gpu_util import GpuCase, assert_mask_equal, assert_output_close, bf16_to_np_f32
from sparse_long_context_ffd_b200 import ffd

pytestmark = pytest.mark.gpu


def _both_formats(w, inp, delta):
    """(int4 out, mask), (thumbnail out, mask), each checked against the oracle."""
    T, S = w.block_size, w.split_blocks
    gc = GpuCase(w, inp)
    gc.quantize(0)
    out, mask = gc.decode(delta)
    p, sc = oracle.quantize_keys(inp["k"], inp["lengths"], T)
    want_out, want_mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], p, sc, inp["lengths"], T,
                                           S, delta)
    assert_mask_equal(mask, want_mask, "int4")
    assert_output_close(out, want_out, "int4")
    bufs = ffd.ThumbResidBuffers(gc.shape)
    ffd.quantize_keys_tr(gc.shape, gc.k, gc.lengths, 0, bufs.k_thumb, bufs.k_resid, bufs.k_scales)
    ffd.decode_tr(gc.shape, gc.q, None, gc.v, bufs.k_thumb, bufs.k_resid, bufs.k_scales, gc.lengths,
                  delta, bufs.out, bufs.mask, bufs.workspace)
    torch.cuda.synchronize()
    th, re, sc2 = oracle.quantize_keys_tr(inp["k"], inp["lengths"], T)
    want_out2, want_mask2, _ = oracle.decode_tr(inp["q"], inp["v"], th, re, sc2, inp["lengths"], T,
                                                S, delta)
    mask2 = bufs.mask.cpu().numpy().view(np.uint32)
    out2 = bf16_to_np_f32(bufs.out).astype(np.float64)
    assert_mask_equal(mask2, want_mask2, "thumbnail")
    assert_output_close(out2, want_out2, "thumbnail")
    assert ffd.check_device_status(gc.bufs.workspace) == 0
    assert ffd.check_device_status(bufs.workspace) == 0
    return (out, mask), (out2, mask2)


@pytest.mark.parametrize("T", [64, 128])
def test_largest_split(T):
    # FFD_MAX_SPLIT_BLOCKS blocks per split: the selection queue and keep bits
    # at their largest; two sequences, one filling a split and a bit more
    S = ffd.FFD_MAX_SPLIT_BLOCKS
    cap = (S + 8) * T
    lengths = np.array([cap, S * T - 5], np.int32)
    w = fw.Workload("maxsplit", 2, 8, 2, cap, T, S, 1.0, 44, context=cap, needles=3)
    inp = fw.make_inputs(w, lengths=lengths)
    for delta in (0.5, 2.0):
        _both_formats(w, inp, delta)


def test_tied_scores_are_all_kept_at_delta_zero():
    # every key row equal: every block scores the same, and score >= max - 0
    # keeps them all (the inclusive test); attention is then uniform
    T, S, cap = 64, 5, 64 * 23
    lengths = np.array([cap, 700], np.int32)
    w = fw.Workload("ties", 2, 4, 1, cap, T, S, 0.0, 45, context=cap, needles=0)
    inp = fw.make_inputs(w, lengths=lengths, with_needles=False)
    row = inp["k"][0, 0, 0].copy()
    inp["k"][:] = row
    (out, mask), (out2, mask2) = _both_formats(w, inp, 0.0)
    nblk = cap // T
    for b, n in enumerate(lengths):
        nb = -(-int(n) // T)
        for m in (mask, mask2):
            bits = oracle.mask_to_blocks(m[b, 0], nblk)
            assert bits[:nb].all() and not bits[nb:].any()
        mean_v = fw.bf16_bits_to_f32(inp["v"][b, 0, :n]).astype(np.float64).mean(axis=0)
        assert np.abs(out[b] - mean_v).max() < 1e-2


def test_zero_query_keeps_every_block():
    # q = 0: every score is 0 (the fold's a == 0 case), every block is kept at
    # any delta, and attention is uniform
    T, S, cap = 64, 4, 64 * 20
    lengths = np.array([cap - 3], np.int32)
    w = fw.Workload("zeroq", 1, 4, 2, cap, T, S, 1.0, 46, context=cap, needles=0)
    inp = fw.make_inputs(w, lengths=lengths, with_needles=False)
    inp["q"][:] = 0
    (out, mask), (out2, _) = _both_formats(w, inp, 0.0)
    nb = -(-int(lengths[0]) // T)
    assert all(oracle.mask_to_blocks(mask[0, g], cap // T)[:nb].all() for g in range(2))
    G = w.group
    for g in range(2):
        mean_v = fw.bf16_bits_to_f32(inp["v"][0, g, :lengths[0]]).astype(np.float64).mean(axis=0)
        for h in range(G):
            assert np.abs(out[0, g * G + h] - mean_v).max() < 1e-2
            assert np.abs(out2[0, g * G + h] - mean_v).max() < 1e-2


def test_single_token_sequences_largest_group():
    T, S, cap = 128, 3, 128 * 6
    lengths = np.array([1, 1, 2, 129], np.int32)
    w = fw.Workload("tiny_seq", 4, 16, 2, cap, T, S, 1.0, 47, context=cap, needles=0)
    inp = fw.make_inputs(w, lengths=lengths, with_needles=False)
    (out, _), _ = _both_formats(w, inp, 1.0)
    # one token: the output is that token's value row, for every head of the group
    G = w.group
    for b in (0, 1):
        for g in range(2):
            v0 = fw.bf16_bits_to_f32(inp["v"][b, g, 0]).astype(np.float64)
            for h in range(G):
                assert np.abs(out[b, g * G + h] - v0).max() < 1e-2
