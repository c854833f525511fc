"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test compares the oracle with one of: a library routine (torch's
scaled-dot-product attention in fp64), a closed form, a brute-force enumeration
of the selection, an error bound, an invariant of the method, or the
hand-worked example in tests/golden/.  No expected value here comes from the
CUDA path.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import ffd_workloads as fw
import oracle
from ffd_workloads import bf16_bits_to_f32 as from_bf16
from ffd_workloads import f32_to_bf16_bits as to_bf16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
D = 128


def _rand_case(seed, B=3, G=4, Hkv=2, cap=1024, T=64, S=3, lo=1, hi=None, needles=1):
    w = fw.random_small_workload(seed, batch=B, group=G, num_kv_heads=Hkv, capacity=cap,
                                 block_size=T, split_blocks=S, delta=2.0, lengths_lo=lo,
                                 lengths_hi=cap if hi is None else hi, needles=needles)
    return w, fw.make_inputs(w)


def _library_attention(q, k, v, lengths, token_keep=None):
    """Reference attention through torch's scaled_dot_product_attention (fp64)."""
    B, Hq, _ = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    for b in range(B):
        n = int(lengths[b])
        if n == 0:
            continue
        qq = torch.from_numpy(from_bf16(q[b]).astype(np.float64))[:, None, :]
        kk = torch.from_numpy(from_bf16(k[b, :, :n]).astype(np.float64)).repeat_interleave(G, 0)
        vv = torch.from_numpy(from_bf16(v[b, :, :n]).astype(np.float64)).repeat_interleave(G, 0)
        mask = None
        if token_keep is not None:
            m = torch.from_numpy(token_keep[b][:, :n]).repeat_interleave(G, 0)[:, None, :]
            if not bool(m.any()):
                continue
            mask = m
        o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask)
        out[b] = o[:, 0, :].numpy()
    return out


def _token_keep(mask, T, cap):
    """[B,Hkv,words] block mask -> [B][Hkv, cap] bool token mask."""
    B, Hkv, _ = mask.shape
    nblk = cap // T
    res = []
    for b in range(B):
        rows = [np.repeat(oracle.mask_to_blocks(mask[b, g], nblk), T) for g in range(Hkv)]
        res.append(np.stack(rows))
    return res


# ---------------------------------------------------------------- attention --

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_dense_mode_equals_library_attention(seed):
    w, inp = _rand_case(seed)
    out, mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], None, None, inp["lengths"],
                                 w.block_size, w.split_blocks, float("inf"))
    ref = _library_attention(inp["q"], inp["k"], inp["v"], inp["lengths"])
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-10)
    nblk = w.capacity // w.block_size
    for b in range(w.batch):
        nb = -(-int(inp["lengths"][b]) // w.block_size)
        for g in range(w.num_kv_heads):
            bits = oracle.mask_to_blocks(mask[b, g], nblk)
            assert bits[:nb].all() and not bits[nb:].any()


@pytest.mark.parametrize("seed", [3, 4])
def test_masked_attention_equals_library_attention(seed):
    w, inp = _rand_case(seed)
    rng = np.random.default_rng(seed)
    words = oracle.mask_words(w.capacity, w.block_size)
    mask = rng.integers(0, 2**32, size=(w.batch, w.num_kv_heads, words), dtype=np.uint64).astype(np.uint32)
    out, lse = oracle.attend(inp["q"], inp["k"], inp["v"], inp["lengths"], mask, w.block_size)
    keep = _token_keep(mask, w.block_size, w.capacity)
    ref = _library_attention(inp["q"], inp["k"], inp["v"], inp["lengths"], keep)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-10)
    # log-sum-exp against torch.logsumexp over the selected logits
    G = w.group
    for b in range(w.batch):
        n = int(inp["lengths"][b])
        for h in range(w.num_q_heads):
            sel = keep[b][h // G][:n]
            if not sel.any():
                assert lse[b, h] == -math.inf
                continue
            qh = from_bf16(inp["q"][b, h]).astype(np.float64)
            kk = from_bf16(inp["k"][b, h // G, :n]).astype(np.float64)[sel]
            ref_lse = torch.logsumexp(torch.from_numpy(kk @ qh / math.sqrt(D)), 0).item()
            assert abs(lse[b, h] - ref_lse) < 1e-10


def test_attention_closed_forms():
    T, cap = 64, 256
    rng = np.random.default_rng(7)
    v = to_bf16(rng.standard_normal((1, 1, cap, D)).astype(np.float32))
    vf = from_bf16(v).astype(np.float64)
    lengths = np.array([200], np.int32)
    full = np.full((1, 1, 1), 0xF, np.uint32)  # 4 blocks
    # identical keys: every weight equal -> plain mean of the V rows
    k_same = np.tile(to_bf16(rng.standard_normal(D).astype(np.float32)), (1, 1, cap, 1))
    q = to_bf16(rng.standard_normal((1, 2, D)).astype(np.float32))
    out, _ = oracle.attend(q, k_same, v[:, :1].repeat(1, 1), lengths, full, T)
    mean = vf[0, 0, :200].mean(axis=0)
    np.testing.assert_allclose(out[0, 0], mean, atol=1e-12)
    np.testing.assert_allclose(out[0, 1], mean, atol=1e-12)
    # zero query: uniform weights whatever the keys are
    k_rand = to_bf16(rng.standard_normal((1, 1, cap, D)).astype(np.float32))
    out, lse = oracle.attend(np.zeros((1, 1, D), np.uint16), k_rand, v, lengths, full, T)
    np.testing.assert_allclose(out[0, 0], mean, atol=1e-12)
    assert abs(lse[0, 0] - math.log(200)) < 1e-12
    # one key far above the rest: output is that key's V row
    qv = np.zeros(D, np.float32)
    qv[0] = 1.0
    k_dom = np.zeros((1, 1, cap, D), np.float32)
    k_dom[0, 0, 77, 0] = 512.0  # logit 512/sqrt(128) ~ 45 above every other (0)
    out, _ = oracle.attend(to_bf16(qv)[None, None], to_bf16(k_dom), v, lengths, full, T)
    np.testing.assert_allclose(out[0, 0], vf[0, 0, 77], atol=1e-15 * 200 + 1e-12)
    # an empty selection and an empty sequence give zero rows
    out, lse = oracle.attend(q[:, :1], k_rand, v, lengths, np.zeros((1, 1, 1), np.uint32), T)
    assert not out.any() and lse[0, 0] == -math.inf
    out, lse = oracle.attend(q[:, :1], k_rand, v, np.array([0], np.int32), full, T)
    assert not out.any()


@pytest.mark.parametrize("seed", [5, 6])
def test_output_is_convex_combination_of_selected_rows(seed):
    w, inp = _rand_case(seed)
    out, mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], *oracle.quantize_keys(
        inp["k"], inp["lengths"], w.block_size), inp["lengths"], w.block_size, w.split_blocks, 1.0)
    keep = _token_keep(mask, w.block_size, w.capacity)
    for b in range(w.batch):
        n = int(inp["lengths"][b])
        for h in range(w.num_q_heads):
            sel = keep[b][h // w.group][:n]
            rows = from_bf16(inp["v"][b, h // w.group, :n][sel]).astype(np.float64)
            assert (out[b, h] >= rows.min(axis=0) - 1e-12).all()
            assert (out[b, h] <= rows.max(axis=0) + 1e-12).all()


# ---------------------------------------------------------------- quantiser --

def _unpack_codes(packed):
    """Independent nibble decoder: byte i holds channel 2i (low) and 2i+1 (high)."""
    lo = (packed & 0x0F).astype(np.int32) - 8
    hi = (packed >> 4).astype(np.int32) - 8
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), np.int32)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def test_quantizer_exact_on_power_of_two_grid():
    # K = m * 2^e with integer m in [-7, 7] and |m| = 7 present in every
    # (block, channel): the scale is exactly 2^e and the codes are exactly m.
    T, cap = 64, 256
    rng = np.random.default_rng(11)
    m = rng.integers(-7, 8, size=(1, 2, cap, D))
    for j in range(cap // T):
        row = j * T + rng.integers(0, T)
        m[:, :, row, :] = 7 * rng.choice([-1, 1], size=(1, 2, D))
    e = rng.integers(-6, 4, size=(1, 2, cap // T, D))
    k = (m * np.exp2(np.repeat(e, T, axis=2))).astype(np.float32)
    kb = to_bf16(k)
    assert np.array_equal(from_bf16(kb), k)  # exactly representable
    packed, scales = oracle.quantize_keys(kb, np.array([cap], np.int32), T)
    assert np.array_equal(from_bf16(scales), np.exp2(e).astype(np.float32))
    assert np.array_equal(_unpack_codes(packed), m)


def test_quantizer_reconstruction_bound_and_tail():
    w, inp = _rand_case(8, B=2, G=1, Hkv=2, cap=512, T=64, lo=130, hi=300)
    packed = fw.poison_packed((w.batch, w.num_kv_heads, w.capacity, D // 2))
    scales = fw.poison_scales((w.batch, w.num_kv_heads, w.capacity // w.block_size, D))
    oracle.quantize_keys(inp["k"], inp["lengths"], w.block_size, 0, packed, scales)
    codes = _unpack_codes(packed)
    T = w.block_size
    for b in range(w.batch):
        n = int(inp["lengths"][b])
        nb = -(-n // T)
        for g in range(w.num_kv_heads):
            kf = from_bf16(inp["k"][b, g, :n]).astype(np.float64)
            sf = np.repeat(from_bf16(scales[b, g, :nb]).astype(np.float64), T, axis=0)[:n]
            kc = codes[b, g, :n]
            assert np.abs(kc).max() <= 7
            # round-to-nearest: reconstruction error at most half a step
            assert (np.abs(kf - sf * kc) <= sf / 2 * (1 + 1e-6) + 1e-30).all()
            # bf16 scale within half an ulp (2^-9 relative) of amax / 7
            for j in range(nb):
                amax = np.abs(kf[j * T:(j + 1) * T]).max(axis=0)
                s = from_bf16(scales[b, g, j]).astype(np.float64)
                assert (np.abs(s - amax / 7) <= amax / 7 * 2.0**-8).all()
            # tokens past the length: code 0 (nibble 8); blocks past nb untouched
            t_end = nb * T
            assert (codes[b, g, n:t_end] == 0).all()
            assert (packed[b, g, t_end:] == fw.PACKED_POISON_BYTE).all()
            assert (scales[b, g, nb:] == fw.SCALE_POISON_BF16).all()
    # the poisoned tail (|K| = 8 >> N(0,1) amax) must not reach the scales
    k2 = inp["k"].copy()
    for b in range(w.batch):
        k2[b, :, int(inp["lengths"][b]):] = 0
    _, scales2 = oracle.quantize_keys(k2, inp["lengths"], w.block_size)
    for b in range(w.batch):
        nb = -(-int(inp["lengths"][b]) // T)
        assert np.array_equal(scales2[b, :, :nb], scales[b, :, :nb])


def test_quantizer_append_equals_from_scratch():
    T, cap = 64, 512
    rng = np.random.default_rng(12)
    k = to_bf16(rng.standard_normal((1, 2, cap, D)).astype(np.float32))
    L = 400
    ref_p, ref_s = oracle.quantize_keys(k, np.array([L], np.int32), T)
    p, s = oracle.quantize_keys(k, np.array([100], np.int32), T)
    for n in range(101, L + 1):  # append one token, requantise the last block
        oracle.quantize_keys(k, np.array([n], np.int32), T, -1, p, s)
    nb = -(-L // T)
    assert np.array_equal(p[:, :, :nb * T], ref_p[:, :, :nb * T])
    assert np.array_equal(s[:, :, :nb], ref_s[:, :, :nb])


# -------------------------------------------------------------- query fold --

def test_fold_closed_forms():
    rng = np.random.default_rng(13)
    # unit scales and integer queries with max |q| = 127: the fold is the identity
    qi_true = rng.integers(-127, 128, size=D)
    qi_true[17] = -127
    q = to_bf16(qi_true.astype(np.float32))
    ones = to_bf16(np.ones(D, np.float32))
    qi, c = oracle.fold_query(q, ones)
    assert np.array_equal(qi, qi_true)
    assert c == np.float32(1.0 / math.sqrt(D))
    # power-of-two channel scales cancel against the same powers in q
    e = rng.integers(-5, 5, size=D)
    q2 = to_bf16((qi_true * np.exp2(-e)).astype(np.float32))
    qi2, c2 = oracle.fold_query(q2, to_bf16(np.exp2(e).astype(np.float32)))
    assert np.array_equal(qi2, qi_true) and c2 == c
    # zero query
    qi3, c3 = oracle.fold_query(np.zeros(D, np.uint16), ones)
    assert not qi3.any() and c3 == 0.0


def test_fold_error_bound():
    rng = np.random.default_rng(14)
    for _ in range(50):
        q = to_bf16(rng.standard_normal(D).astype(np.float32))
        s = to_bf16(np.abs(rng.standard_normal(D)).astype(np.float32) / 7)
        qi, c = oracle.fold_query(q, s)
        p = from_bf16(q).astype(np.float64) * from_bf16(s)
        a = np.abs(p).max()
        assert np.abs(qi).max() == 127
        assert (np.abs(qi * a / 127 - p) <= a / 254 * (1 + 1e-6)).all()
        assert abs(c - a / 127 / math.sqrt(D)) <= 1e-6 * c


# ------------------------------------------------------------ block scores --

def test_block_scores_integer_case():
    # unit scales (amax = 7 in every channel of every block) and integer query
    # with max |q| = 127: the score is max_t (q . k_t) / sqrt(D) exactly.
    T, cap = 64, 256
    rng = np.random.default_rng(15)
    m = rng.integers(-7, 8, size=(1, 1, cap, D))
    m[:, :, ::T, :] = 7
    k = to_bf16(m.astype(np.float32))
    qint = rng.integers(-127, 128, size=(1, 2, D))
    qint[:, :, 0] = 127
    q = to_bf16(qint.astype(np.float32))
    lengths = np.array([cap - 5], np.int32)
    packed, scales = oracle.quantize_keys(k, lengths, T)
    # garbage in the packed rows past the length must not reach the scores
    packed[:, :, cap - 5:] = 0xFF
    sc = oracle.block_scores(q, packed, scales, lengths, T)
    dots = np.einsum("hc,tc->ht", qint[0], m[0, 0])
    for j in range(cap // T):
        t1 = min((j + 1) * T, int(lengths[0]))
        want = dots[:, j * T:t1].max(axis=1).astype(np.float32) * np.float32(1 / math.sqrt(D))
        assert np.array_equal(sc[0, :, j], want)


def test_block_score_ignores_tokens_past_length():
    # the last block holds one valid token with a negative dot product; the
    # remaining rows of the block (code 0, or garbage) must not lift the max
    T, cap = 64, 128
    k = np.zeros((1, 1, cap, D), np.float32)
    k[0, 0, :T] = 1.0
    k[0, 0, T] = -1.0
    q = to_bf16(np.ones((1, 1, D), np.float32))
    lengths = np.array([T + 1], np.int32)
    packed, scales = oracle.quantize_keys(to_bf16(k), lengths, T)
    sc = oracle.block_scores(q, packed, scales, lengths, T)
    # one token of -1 in every channel: scale bf16(1/7) = 0.142578125, code -7,
    # query folds to qi = 127 -> score = -7 * 0.142578125 * D / sqrt(D)
    assert sc[0, 0, 1] < 0
    assert abs(sc[0, 0, 1] - (-7 * 0.142578125 * D / math.sqrt(D))) < 1e-4
    packed[0, 0, T + 1:] = 0xFF
    assert oracle.block_scores(q, packed, scales, lengths, T)[0, 0, 1] == sc[0, 0, 1]


def test_quantizer_saturates_on_subnormal_scales():
    # keys of 10 * 2^-133 (bf16 subnormals): amax / 7 rounds to the smallest
    # bf16 subnormal 2^-133, so K / s = 10 and the code saturates at +-7
    T, cap = 64, 64
    tiny = np.float32(10 * 2.0**-133)
    k = np.full((1, 1, cap, D), tiny, np.float32)
    k[0, 0, 1::2] = -tiny
    kb = to_bf16(k)
    assert np.array_equal(from_bf16(kb), k)
    packed, scales = oracle.quantize_keys(kb, np.array([cap], np.int32), T)
    assert (from_bf16(scales) == np.float32(2.0**-133)).all()
    codes = _unpack_codes(packed)
    assert (codes[0, 0, 0::2] == 7).all() and (codes[0, 0, 1::2] == -7).all()


def test_block_scores_within_quantisation_bound():
    w, inp = _rand_case(16, B=2, G=4, Hkv=2, cap=512, lo=100, hi=512)
    T = w.block_size
    packed, scales = oracle.quantize_keys(inp["k"], inp["lengths"], T)
    sc = oracle.block_scores(inp["q"], packed, scales, inp["lengths"], T)
    codes = _unpack_codes(packed)
    for b in range(w.batch):
        n = int(inp["lengths"][b])
        for h in range(w.num_q_heads):
            g = h // w.group
            qh = from_bf16(inp["q"][b, h]).astype(np.float64)
            for j in range(-(-n // T)):
                s = from_bf16(scales[b, g, j]).astype(np.float64)
                kc = codes[b, g, j * T:min((j + 1) * T, n)]
                exact = (kc * s) @ qh / math.sqrt(D)  # dequantised keys, fp64
                a = np.abs(qh * s).max()
                bound = a / 254 * np.abs(kc).sum(axis=1).max() / math.sqrt(D)
                assert abs(sc[b, h, j] - exact.max()) <= bound * (1 + 1e-5) + 1e-6
            assert (sc[b, h, -(-n // T):] == -np.inf).all()


def _permute_tokens_in_blocks(x, lengths, T, rng):
    """Shuffle the valid tokens of every block (axis 2) among themselves."""
    y = x.copy()
    for b in range(x.shape[0]):
        n = int(lengths[b])
        for j0 in range(0, n, T):
            idx = np.arange(j0, min(j0 + T, n))
            y[b, :, idx] = x[b, :, rng.permutation(idx)]
    return y


def test_scores_equivariant_under_channel_and_token_permutations():
    # The fold is elementwise over channels with a permutation-invariant max,
    # the integer dot products are exact and the block score is a max over the
    # block's tokens: permuting q's and K's channels together, or the tokens
    # inside a block, must leave every score bit-identical and permute the
    # int4 copy and its scales with them.  (A channel paired with another
    # channel's scale, or a token counted in the wrong block, breaks it.)
    w, inp = _rand_case(19, B=2, G=4, Hkv=2, cap=512, lo=70, hi=512)
    T = w.block_size
    q, k, lengths = inp["q"], inp["k"], inp["lengths"]
    packed, scales = oracle.quantize_keys(k, lengths, T)
    sc = oracle.block_scores(q, packed, scales, lengths, T)
    rng = np.random.default_rng(190)
    perm = rng.permutation(D)
    packed_c, scales_c = oracle.quantize_keys(np.ascontiguousarray(k[..., perm]), lengths, T)
    assert np.array_equal(scales_c, scales[..., perm])
    assert np.array_equal(_unpack_codes(packed_c), _unpack_codes(packed)[..., perm])
    sc_c = oracle.block_scores(np.ascontiguousarray(q[..., perm]), packed_c, scales_c, lengths, T)
    assert np.array_equal(sc_c, sc)
    k_t = _permute_tokens_in_blocks(k, lengths, T, rng)
    packed_t, scales_t = oracle.quantize_keys(k_t, lengths, T)
    assert np.array_equal(scales_t, scales)
    assert np.array_equal(oracle.block_scores(q, packed_t, scales_t, lengths, T), sc)


def test_power_of_two_scaling_carries_through_copy_scores_and_selection():
    # Scaling K (or q) by 2^e is exact in bf16 and commutes with every
    # rounding of the quantiser and the fold: the int4 codes and the int8
    # query stay the same, the scales (or the fold's a) gain 2^e, so every
    # block score is multiplied by exactly 2^e, and the Top-delta selection
    # with delta 2^e equals the original one.  (A fold that ignored the scales
    # or a score factor without a, for example, breaks it.)
    w, inp = _rand_case(31, B=2, G=4, Hkv=2, cap=512, lo=70, hi=512)
    T, S = w.block_size, 3
    q, k, lengths = inp["q"], inp["k"], inp["lengths"]
    packed, scales = oracle.quantize_keys(k, lengths, T)
    sc = oracle.block_scores(q, packed, scales, lengths, T)
    _, mask = oracle.select(sc, lengths, w.num_kv_heads, w.capacity, T, S, 1.5)
    for ek, eq in [(3, 0), (-4, 0), (0, 5), (2, -3)]:
        k2 = to_bf16((from_bf16(k) * np.float32(2.0**ek)).astype(np.float32))
        q2 = to_bf16((from_bf16(q) * np.float32(2.0**eq)).astype(np.float32))
        packed2, scales2 = oracle.quantize_keys(k2, lengths, T)
        assert np.array_equal(packed2, packed)
        assert np.array_equal(from_bf16(scales2), from_bf16(scales) * np.float32(2.0**ek))
        sc2 = oracle.block_scores(q2, packed2, scales2, lengths, T)
        assert np.array_equal(sc2, sc * np.float32(2.0**(ek + eq)))
        _, mask2 = oracle.select(sc2, lengths, w.num_kv_heads, w.capacity, T, S,
                                 1.5 * 2.0**(ek + eq))
        assert np.array_equal(mask2, mask)


@pytest.mark.parametrize("G,T", [(1, 128), (2, 64), (8, 128)])
def test_other_group_and_block_sizes(G, T):
    # The pins above mostly run G = 4, T = 64; the GPU path also serves
    # G in {1, 2, 8} and T = 128 (the 256K workload).  Re-check the defining
    # facts there: dense and masked attention against torch SDPA, the int4
    # copy's half-step bound and scale rule, and the block-score bound.
    w, inp = _rand_case(40 + G, B=2, G=G, Hkv=2, cap=1024, T=T, S=3, lo=150, hi=1024)
    q, k, v, lengths = inp["q"], inp["k"], inp["v"], inp["lengths"]
    out, mask, _ = oracle.decode(q, k, v, None, None, lengths, T, w.split_blocks, float("inf"))
    np.testing.assert_allclose(out, _library_attention(q, k, v, lengths), rtol=0, atol=1e-10)
    packed, scales = oracle.quantize_keys(k, lengths, T)
    codes = _unpack_codes(packed)
    sc = oracle.block_scores(q, packed, scales, lengths, T)
    for b in range(w.batch):
        n = int(lengths[b])
        nb = -(-n // T)
        for g in range(w.num_kv_heads):
            kf = from_bf16(k[b, g, :n]).astype(np.float64)
            sf = np.repeat(from_bf16(scales[b, g, :nb]).astype(np.float64), T, axis=0)[:n]
            kc = codes[b, g, :n]
            assert np.abs(kc).max() <= 7
            assert (np.abs(kf - sf * kc) <= sf / 2 * (1 + 1e-6) + 1e-30).all()
            assert (codes[b, g, n:nb * T] == 0).all()
            for j in range(nb):
                amax = np.abs(kf[j * T:(j + 1) * T]).max(axis=0)
                sj = from_bf16(scales[b, g, j]).astype(np.float64)
                assert (np.abs(sj - amax / 7) <= amax / 7 * 2.0**-8).all()
        for h in range(w.num_q_heads):
            g = h // G
            qh = from_bf16(q[b, h]).astype(np.float64)
            for j in range(nb):
                sj = from_bf16(scales[b, g, j]).astype(np.float64)
                kc = codes[b, g, j * T:min((j + 1) * T, n)]
                exact = (kc * sj) @ qh / math.sqrt(D)
                bound = np.abs(qh * sj).max() / 254 * np.abs(kc).sum(axis=1).max() / math.sqrt(D)
                assert abs(sc[b, h, j] - exact.max()) <= bound * (1 + 1e-5) + 1e-6
    out_s, mask_s, _ = oracle.decode(q, k, v, packed, scales, lengths, T, w.split_blocks, 1.0)
    keep = _token_keep(mask_s, T, w.capacity)
    np.testing.assert_allclose(out_s, _library_attention(q, k, v, lengths, keep), rtol=0, atol=1e-10)


# ---------------------------------------------------------------- selection --

def _read_golden():
    cases, meta = [], {}
    with open(os.path.join(GOLDEN, "topdelta_worked_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            if key == "case":
                kv = dict(item.split("=") for item in rest)
                cases.append(kv)
            else:
                meta[key] = rest
    return meta, cases


def test_select_hand_worked_example():
    meta, cases = _read_golden()
    T, S, nb = int(meta["block_size"][0]), int(meta["split_blocks"][0]), int(meta["num_blocks"][0])
    scores = np.array([[list(map(float, meta["scores_head0"])),
                        list(map(float, meta["scores_head1"]))]], np.float32)
    lengths = np.array([nb * T], np.int32)
    assert len(cases) == 3
    for case in cases:
        keep, mask = oracle.select(scores, lengths, 1, nb * T, T, S, float(case["delta"]))
        assert "".join(map(str, keep[0, 0])) == case["keep_head0"]
        assert "".join(map(str, keep[0, 1])) == case["keep_head1"]
        assert int(mask[0, 0, 0]) == int(case["mask"], 16)


def _declarative_keep(s, nb, S, delta):
    """keep_j <=> s_j >= max(s over blocks of j's split up to j) - delta."""
    out = np.zeros(nb, bool)
    for j in range(nb):
        start = (j // S) * S
        ref = max(s[start:j + 1])
        out[j] = s[j] >= np.float32(np.float32(ref) - np.float32(delta))
    return out


@pytest.mark.parametrize("seed", range(6))
def test_select_matches_bruteforce_enumeration(seed):
    rng = np.random.default_rng(100 + seed)
    for _ in range(8):
        nb = int(rng.integers(1, 13))
        S = int(rng.choice([1, 3, 4, nb]))
        G = int(rng.choice([1, 4]))
        T = 64
        # scores on a coarse grid, so ties and equality with m - delta occur
        scores = (rng.integers(-8, 9, size=(1, G, nb)) * 0.5).astype(np.float32)
        delta = float(rng.choice([0.0, 0.5, 1.0, 2.5, np.inf]))
        _, mask = oracle.select(scores, np.array([nb * T], np.int32), 1, nb * T, T, S, delta)
        got = oracle.mask_to_blocks(mask[0, 0], nb)
        per_head = [_declarative_keep(scores[0, h], nb, S, delta) for h in range(G)]
        satisfying = []
        for bits in itertools.product([False, True], repeat=nb):
            X = np.array(bits)
            if all(X[j] == any(ph[j] for ph in per_head) for j in range(nb)):
                satisfying.append(X)
        assert len(satisfying) == 1
        assert np.array_equal(satisfying[0], got)


def test_select_invariants():
    rng = np.random.default_rng(21)
    B, G, Hkv, T, S, nblk = 2, 4, 2, 64, 5, 23
    lengths = np.array([nblk * T, 9 * T + 3], np.int32)
    scores = rng.standard_normal((B, G * Hkv, nblk)).astype(np.float32)
    for b in range(B):
        nb = -(-int(lengths[b]) // T)
        scores[b, :, nb:] = -np.inf
    cap = nblk * T

    def blocks(mask):
        return np.array([[oracle.mask_to_blocks(mask[b, g], nblk) for g in range(Hkv)]
                         for b in range(B)])

    # critical deltas: the gaps (running max - score), each just below and at
    crit = set()
    for b in range(B):
        nb = -(-int(lengths[b]) // T)
        for h in range(G * Hkv):
            for j in range(nb):
                st = (j // S) * S
                gap = float(np.float32(scores[b, h, st:j + 1].max()) - scores[b, h, j])
                crit.update([gap, float(np.nextafter(np.float32(gap), np.float32(0)))])
    deltas = sorted(d for d in crit if d >= 0) + [np.inf]
    prev = None
    for d in deltas:
        keep, mask = oracle.select(scores, lengths, Hkv, cap, T, S, d)
        cur = blocks(mask)
        if prev is not None:
            assert (cur | ~prev).all() or (prev <= cur).all()  # monotone in delta
            assert (prev <= cur).all()
        prev = cur
        for b in range(B):
            nb = -(-int(lengths[b]) // T)
            assert not cur[b, :, nb:].any()  # nothing past the sequence
            assert cur[b, :, 0:nb:S].all()  # first block of every split
            for g in range(Hkv):  # union over the group == OR of per-head keeps
                union = keep[b, g * G:(g + 1) * G, :].any(axis=0).astype(bool)
                assert np.array_equal(union, cur[b, g])
                for h in range(g * G, (g + 1) * G):  # same as a G = 1 run of that head
                    _, m1 = oracle.select(scores[b:b + 1, h:h + 1], lengths[b:b + 1], 1,
                                          cap, T, S, d)
                    assert not (oracle.mask_to_blocks(m1[0, 0], nblk) & ~cur[b, g]).any()
    # delta = 0 keeps exactly the running-maximum records
    keep, _ = oracle.select(scores, lengths, Hkv, cap, T, S, 0.0)
    for b in range(B):
        nb = -(-int(lengths[b]) // T)
        for h in range(G * Hkv):
            for j in range(nb):
                st = (j // S) * S
                assert keep[b, h, j] == (scores[b, h, j] >= scores[b, h, st:j + 1].max())


def test_select_rejects_bad_arguments():
    s = np.zeros((1, 1, 4), np.float32)
    ln = np.array([256], np.int32)
    for bad in (-1.0, float("nan")):
        with pytest.raises(oracle.OracleError):
            oracle.select(s, ln, 1, 256, 64, 2, bad)
    with pytest.raises(oracle.OracleError):
        oracle.select(s, np.array([257], np.int32), 1, 256, 64, 2, 1.0)
    with pytest.raises(oracle.OracleError):
        oracle.select(s, np.array([-1], np.int32), 1, 256, 64, 2, 1.0)


# ------------------------------------------------------------ whole decode --

def test_decode_batch_independence_and_shard_invariance():
    w, inp = _rand_case(30, B=4, G=2, Hkv=2, cap=1024, T=64, S=3, lo=1, hi=1024)
    T, S = w.block_size, w.split_blocks
    packed, scales = oracle.quantize_keys(inp["k"], inp["lengths"], T)
    out, mask, sc = oracle.decode(inp["q"], inp["k"], inp["v"], packed, scales, inp["lengths"],
                                  T, S, 1.5)
    for b in range(w.batch):
        o1, m1, _ = oracle.decode(inp["q"][b:b + 1], inp["k"][b:b + 1], inp["v"][b:b + 1],
                                  packed[b:b + 1], scales[b:b + 1], inp["lengths"][b:b + 1],
                                  T, S, 1.5)
        assert np.array_equal(o1[0], out[b]) and np.array_equal(m1[0], mask[b])
        # truncating the sequence at a split boundary leaves earlier splits' selection alone
        n = int(inp["lengths"][b])
        cut = ((-(-n // T) - 1) // S) * S * T
        if cut == 0:
            continue
        _, m2, _ = oracle.decode(inp["q"][b:b + 1], inp["k"][b:b + 1], inp["v"][b:b + 1],
                                 packed[b:b + 1], scales[b:b + 1], np.array([cut], np.int32),
                                 T, S, 1.5)
        nblk = w.capacity // T
        for g in range(w.num_kv_heads):
            full_bits = oracle.mask_to_blocks(mask[b, g], nblk)
            cut_bits = oracle.mask_to_blocks(m2[0, g], nblk)
            assert np.array_equal(full_bits[:cut // T], cut_bits[:cut // T])
            assert not cut_bits[cut // T:].any()


def test_decode_edge_lengths():
    T, cap = 64, 512
    rng = np.random.default_rng(31)
    q = to_bf16(rng.standard_normal((6, 4, D)).astype(np.float32))
    k = to_bf16(rng.standard_normal((6, 1, cap, D)).astype(np.float32))
    v = to_bf16(rng.standard_normal((6, 1, cap, D)).astype(np.float32))
    lengths = np.array([0, 1, T - 1, T + 1, cap - 1, cap], np.int32)
    packed, scales = oracle.quantize_keys(k, lengths, T)
    out, mask, _ = oracle.decode(q, k, v, packed, scales, lengths, T, 3, 2.0)
    assert not out[0].any() and not mask[0].any()
    dense, _, _ = oracle.decode(q, k, v, None, None, lengths, T, 3, float("inf"))
    ref = _library_attention(q, k, v, lengths)
    np.testing.assert_allclose(dense, ref, atol=1e-10)
    # a single token: the output is that token's V row
    np.testing.assert_allclose(out[1], np.tile(from_bf16(v[1, 0, 0]), (4, 1)), atol=1e-12)
    with pytest.raises(oracle.OracleError):
        oracle.decode(q, k, v, packed, scales, np.array([0, 1, 2, 3, 4, cap + 1], np.int32),
                      T, 3, 2.0)


@pytest.mark.parametrize("name,overrides", [
    ("tiny", {}),
    ("llama", dict(batch=1, num_q_heads=8, num_kv_heads=2, capacity=8192, context=8192)),
    ("max256k", dict(num_q_heads=8, num_kv_heads=2, capacity=16384, context=16384, needles=6)),
    ("ragged", dict(batch=3, num_q_heads=8, num_kv_heads=2, capacity=16384, ragged=(4096, 16384))),
])
def test_planted_needles_are_selected(name, overrides):
    w = fw.scaled_workload(fw.WORKLOADS[name], **overrides)
    inp = fw.make_inputs(w)
    packed, scales = oracle.quantize_keys(inp["k"], inp["lengths"], w.block_size)
    sc = oracle.block_scores(inp["q"], packed, scales, inp["lengths"], w.block_size)
    nblk = w.capacity // w.block_size
    for delta in (1.0, 2.0, 3.0, 4.0):
        keep, mask = oracle.select(sc, inp["lengths"], w.num_kv_heads, w.capacity,
                                   w.block_size, w.split_blocks, delta)
        for b in range(w.batch):
            for g in range(w.num_kv_heads):
                bits = oracle.mask_to_blocks(mask[b, g], nblk)
                for i, j in enumerate(inp["needles"][b]):
                    assert bits[j], (name, delta, b, g, j)
                    # the targeted head keeps it on its own
                    assert keep[b, g * w.group + i % w.group, j]


# ------------------------------------------- pseudo-max reference (sink/local) --

def test_select_pseudo_max_hand_worked_example():
    meta, cases = {}, []
    with open(os.path.join(GOLDEN, "topdelta_pseudo_max_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            if key == "case":
                cases.append(dict(item.split("=") for item in rest))
            else:
                meta[key] = rest
    T, S, nb = int(meta["block_size"][0]), int(meta["split_blocks"][0]), int(meta["num_blocks"][0])
    scores = np.array([[list(map(float, meta["scores_head0"]))]], np.float32)
    lengths = np.array([nb * T], np.int32)
    assert len(cases) == 4
    for case in cases:
        _, mask = oracle.select(scores, lengths, 1, nb * T, T, S, float(case["delta"]),
                                pseudo_max=case["reference"] == "pseudo")
        assert int(mask[0, 0, 0]) == int(case["mask"], 16), case


def _declarative_keep_pseudo(s, nb, S, delta):
    """keep_j <=> s_j >= max(pseudo, s over j's split up to j) - delta, with
    pseudo = max(s_0, s_{nb-1})."""
    pseudo = max(s[0], s[nb - 1])
    out = np.zeros(nb, bool)
    for j in range(nb):
        start = (j // S) * S
        ref = max(pseudo, max(s[start:j + 1]))
        out[j] = s[j] >= np.float32(np.float32(ref) - np.float32(delta))
    return out


@pytest.mark.parametrize("seed", range(6))
def test_select_pseudo_max_matches_bruteforce_enumeration(seed):
    rng = np.random.default_rng(300 + seed)
    for _ in range(8):
        nb = int(rng.integers(1, 13))
        S = int(rng.choice([1, 3, 4, nb]))
        G = int(rng.choice([1, 4]))
        T = 64
        scores = (rng.integers(-8, 9, size=(1, G, nb)) * 0.5).astype(np.float32)
        delta = float(rng.choice([0.0, 0.5, 1.0, 2.5, np.inf]))
        _, mask = oracle.select(scores, np.array([nb * T], np.int32), 1, nb * T, T, S, delta,
                                pseudo_max=True)
        got = oracle.mask_to_blocks(mask[0, 0], nb)
        per_head = [_declarative_keep_pseudo(scores[0, h], nb, S, delta) for h in range(G)]
        satisfying = [np.array(bits) for bits in itertools.product([False, True], repeat=nb)
                      if all(bits[j] == any(ph[j] for ph in per_head) for j in range(nb))]
        assert len(satisfying) == 1 and np.array_equal(satisfying[0], got)


def test_select_pseudo_max_invariants():
    rng = np.random.default_rng(31)
    B, G, Hkv, T, S, nblk = 2, 4, 2, 64, 5, 23
    lengths = np.array([nblk * T, 9 * T + 3], np.int32)
    scores = rng.standard_normal((B, G * Hkv, nblk)).astype(np.float32)
    for b in range(B):
        scores[b, :, -(-int(lengths[b]) // T):] = -np.inf
    cap = nblk * T
    prev = None
    for d in [0.0, 0.25, 0.5, 1.0, 2.0, 4.0, np.inf]:
        keep_p, mask_p = oracle.select(scores, lengths, Hkv, cap, T, S, d, pseudo_max=True)
        _, mask_r = oracle.select(scores, lengths, Hkv, cap, T, S, d)
        cur = np.array([[oracle.mask_to_blocks(mask_p[b, g], nblk) for g in range(Hkv)]
                        for b in range(B)])
        run = np.array([[oracle.mask_to_blocks(mask_r[b, g], nblk) for g in range(Hkv)]
                        for b in range(B)])
        assert (cur <= run).all()  # a higher reference keeps a subset
        if prev is not None:
            assert (prev <= cur).all()  # monotone in delta
        prev = cur
        for b in range(B):
            nb = -(-int(lengths[b]) // T)
            for h in range(G * Hkv):
                # the head's highest-scoring block is always kept (no head keeps nothing)
                assert keep_p[b, h, int(np.argmax(scores[b, h, :nb]))]
                # block 0 opens its split, so it is kept whenever it sets the pseudo-max
                if scores[b, h, 0] >= scores[b, h, nb - 1]:
                    assert keep_p[b, h, 0]
            if d == np.inf:
                assert cur[b, :, :nb].all()


def test_decode_pseudo_max_attends_over_its_mask():
    w, inp = _rand_case(77, B=3, G=4, Hkv=2, cap=2048, T=64, S=4, lo=300, hi=2048)
    packed, scales = oracle.quantize_keys(inp["k"], inp["lengths"], w.block_size)
    for delta in (0.0, 1.0):
        out, mask, _ = oracle.decode(inp["q"], inp["k"], inp["v"], packed, scales, inp["lengths"],
                                     w.block_size, w.split_blocks, delta, pseudo_max=True)
        ref = _library_attention(inp["q"], inp["k"], inp["v"], inp["lengths"],
                                 _token_keep(mask, w.block_size, w.capacity))
        np.testing.assert_allclose(out, ref, atol=1e-10)


# ------------------------- the pages' rule: pseudo-max as a fixed threshold --

def _golden_examples(name):
    """Parse a golden file of 'example' sections: meta lines and case lines."""
    examples = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            if key == "example":
                examples.append({"meta": {}, "cases": []})
            elif key == "case":
                examples[-1]["cases"].append(dict(item.split("=") for item in rest))
            else:
                examples[-1]["meta"][key] = rest
    return examples


_REFS = {"running": oracle.RUNNING_MAX, "seeded": oracle.PSEUDO_MAX_SEEDED,
         "fixed": oracle.PSEUDO_MAX_FIXED}


def test_select_pseudo_max_fixed_hand_worked_examples():
    examples = _golden_examples("topdelta_pseudo_max_fixed_example.txt")
    assert len(examples) == 2 and sum(len(e["cases"]) for e in examples) == 13
    for ex in examples:
        meta = ex["meta"]
        T, nb = int(meta["block_size"][0]), int(meta["num_blocks"][0])
        scores = np.array([[list(map(float, meta["scores_head0"]))]], np.float32)
        lengths = np.array([nb * T], np.int32)
        for case in ex["cases"]:
            _, mask = oracle.select(scores, lengths, 1, nb * T, T, int(case["split"]),
                                    float(case["delta"]), reference=_REFS[case["reference"]])
            assert int(mask[0, 0, 0]) == int(case["mask"], 16), case


def _declarative_keep_fixed(s, nb, delta):
    """keep_j <=> s_j >= max(s_0, s_{nb-1}) - delta (fp32 subtraction)."""
    thr = np.float32(np.float32(max(s[0], s[nb - 1])) - np.float32(delta))
    return np.array([s[j] >= thr for j in range(nb)], bool)


@pytest.mark.parametrize("seed", range(6))
def test_select_pseudo_max_fixed_matches_bruteforce_enumeration(seed):
    rng = np.random.default_rng(500 + seed)
    for _ in range(8):
        nb = int(rng.integers(1, 13))
        S = int(rng.choice([1, 3, 4, nb]))
        G = int(rng.choice([1, 4]))
        T = 64
        scores = (rng.integers(-8, 9, size=(1, G, nb)) * 0.5).astype(np.float32)
        delta = float(rng.choice([0.0, 0.5, 1.0, 2.5, np.inf]))
        keep, mask = oracle.select(scores, np.array([nb * T], np.int32), 1, nb * T, T, S, delta,
                                   reference=oracle.PSEUDO_MAX_FIXED)
        got = oracle.mask_to_blocks(mask[0, 0], nb)
        per_head = [_declarative_keep_fixed(scores[0, h], nb, delta) for h in range(G)]
        satisfying = [np.array(bits) for bits in itertools.product([False, True], repeat=nb)
                      if all(bits[j] == any(ph[j] for ph in per_head) for j in range(nb))]
        assert len(satisfying) == 1 and np.array_equal(satisfying[0], got)
        for h in range(G):
            assert np.array_equal(keep[0, h, :nb].astype(bool), per_head[h])


def test_select_pseudo_max_fixed_invariants():
    rng = np.random.default_rng(41)
    B, G, Hkv, T, nblk = 2, 4, 2, 64, 23
    lengths = np.array([nblk * T, 9 * T + 3], np.int32)
    scores = rng.standard_normal((B, G * Hkv, nblk)).astype(np.float32)
    cap = nblk * T
    prev = None
    for d in [0.0, 0.25, 0.5, 1.0, 2.0, 4.0, np.inf]:
        keep_f, mask_f = oracle.select(scores, lengths, Hkv, cap, T, 5, d,
                                       reference=oracle.PSEUDO_MAX_FIXED)
        _, mask_s = oracle.select(scores, lengths, Hkv, cap, T, 5, d,
                                  reference=oracle.PSEUDO_MAX_SEEDED)

        def blocks(m):
            return np.array([[oracle.mask_to_blocks(m[b, g], nblk) for g in range(Hkv)]
                             for b in range(B)])
        fixed, seeded = blocks(mask_f), blocks(mask_s)
        assert (seeded <= fixed).all()  # the seeded maximum never drops below the pseudo-max
        for S in (1, 2, 7, nblk):  # no split enters the fixed rule
            _, m2 = oracle.select(scores, lengths, Hkv, cap, T, S, d,
                                  reference=oracle.PSEUDO_MAX_FIXED)
            assert np.array_equal(m2, mask_f)
        if prev is not None:
            assert (prev <= fixed).all()  # monotone in delta
        prev = fixed
        for b in range(B):
            nb = -(-int(lengths[b]) // T)
            for h in range(G * Hkv):
                mt = max(scores[b, h, 0], scores[b, h, nb - 1])
                # every block at or above the pseudo-max is kept: the sink or
                # local block that sets it in particular
                assert keep_f[b, h, :nb][scores[b, h, :nb] >= mt].all()
                assert not keep_f[b, h, nb:].any()
            if d == np.inf:
                assert fixed[b, :, :nb].all()
        # the group union is the OR of the heads' own selections
        for b in range(B):
            for g in range(Hkv):
                heads = keep_f[b, g * G:(g + 1) * G].astype(bool).any(axis=0)
                assert np.array_equal(heads, fixed[b, g])


def test_decode_pseudo_max_fixed_attends_over_its_mask():
    w, inp = _rand_case(78, B=3, G=4, Hkv=2, cap=2048, T=64, S=4, lo=300, hi=2048)
    packed, scales = oracle.quantize_keys(inp["k"], inp["lengths"], w.block_size)
    sc = oracle.block_scores(inp["q"], packed, scales, inp["lengths"], w.block_size)
    for delta in (0.0, 1.0):
        out, mask, sc2 = oracle.decode(inp["q"], inp["k"], inp["v"], packed, scales,
                                       inp["lengths"], w.block_size, w.split_blocks, delta,
                                       reference=oracle.PSEUDO_MAX_FIXED)
        assert np.array_equal(sc2, sc)
        _, want = oracle.select(sc, inp["lengths"], w.num_kv_heads, w.capacity, w.block_size,
                                w.split_blocks, delta, reference=oracle.PSEUDO_MAX_FIXED)
        assert np.array_equal(mask, want)
        ref = _library_attention(inp["q"], inp["k"], inp["v"], inp["lengths"],
                                 _token_keep(mask, w.block_size, w.capacity))
        np.testing.assert_allclose(out, ref, atol=1e-10)


def test_sparsity_adapts_to_attention_sharpness():
    # Methodology 2, Adaptivity (gist.science explainer): when attention is
    # concentrated, fewer blocks fall within delta of the peak.  Same queries,
    # same delta: flat keys keep (nearly) every block; keys whose first block
    # of every split dominates keep little more than those blocks.
    T, S, G, nblk = 64, 8, 4, 64
    cap = T * nblk
    rng = np.random.default_rng(7)
    q0 = rng.standard_normal(128).astype(np.float32)
    q = np.tile(q0, (1, G, 1))                       # [1, G, 128]: one direction for the group
    flat = (0.1 * rng.standard_normal((1, 1, cap, 128))).astype(np.float32)
    sharp = flat.copy()
    bump = 5.0 * np.sqrt(128.0) * q0 / np.dot(q0, q0)  # raises q.k / sqrt(D) by 5 (delta is 1)
    for j in range(0, nblk, S):                      # the first block of every split
        sharp[0, 0, j * T:(j + 1) * T] += bump
    v = rng.standard_normal((1, 1, cap, 128)).astype(np.float32)
    lengths = np.array([cap], np.int32)
    qb, vb = fw.f32_to_bf16_bits(q), fw.f32_to_bf16_bits(v)
    kept = {}
    for name, k in (("flat", flat), ("sharp", sharp)):
        kb = fw.f32_to_bf16_bits(k)
        p, s = oracle.quantize_keys(kb, lengths, T)
        _, mask, _ = oracle.decode(qb, kb, vb, p, s, lengths, T, S, 1.0)
        kept[name] = oracle.mask_to_blocks(mask[0, 0], nblk)
        th, re, sc = oracle.quantize_keys_tr(kb, lengths, T)
        _, mask_tr, _ = oracle.decode_tr(qb, vb, th, re, sc, lengths, T, S, 1.0)
        kept[name + "_tr"] = oracle.mask_to_blocks(mask_tr[0, 0], nblk)
    for fmt in ("", "_tr"):
        assert kept["flat" + fmt].sum() >= 0.9 * nblk
        assert kept["sharp" + fmt].sum() <= nblk // S + 2
        assert all(kept["sharp" + fmt][j] for j in range(0, nblk, S))  # the dominant blocks stay
