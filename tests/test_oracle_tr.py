"""Pins of the oracle's thumbnail + residual key format (2-bit thumbnails,
8-bit residuals) against facts that do not come from the oracle itself: the
hand-worked example in tests/golden/, nearest-level and error-bound properties
of the quantiser, keys on which the reconstruction is exact, torch's fp64
attention on such keys, and closed-form integer scores.  No expected value
here comes from the CUDA path.
"""
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


def _thumb_codes(thumb):
    """Independent decoder of the packing: channel 16w + i sits in the
    little-endian 32-bit word w at bit 2 (i // 2) + 16 (i % 2)."""
    words = np.ascontiguousarray(thumb).view("<u4").astype(np.int64)
    out = np.empty(thumb.shape[:-1] + (thumb.shape[-1] * 4,), np.int32)
    for i in range(16):
        shift = 2 * (i // 2) + 16 * (i % 2)
        out[..., i::16] = (words >> shift) & 3
    return out


def _read_golden():
    vals = {}
    with open(os.path.join(GOLDEN, "thumb_residual_worked_example.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, *rest = line.split()
                vals[key] = rest
    return vals


def _rand_keys(seed, B=2, Hkv=2, cap=512, scale=1.0):
    rng = np.random.default_rng(seed)
    return to_bf16((scale * rng.standard_normal((B, Hkv, cap, D))).astype(np.float32))


def test_thumb_residual_hand_worked_example():
    g = _read_golden()
    T, L = int(g["block_size"][0]), int(g["length"][0])
    k = np.zeros((1, 1, T, D), np.float32)
    k[0, 0, 0, :3] = [float(x) for x in g["k_t0"]]
    k[0, 0, 1, :3] = [float(x) for x in g["k_t1"]]
    lengths = np.array([L], np.int32)
    thumb, resid, scales = oracle.quantize_keys_tr(to_bf16(k), lengths, T)
    want_s = np.zeros(D, np.uint16)
    want_s[:3] = [int(x, 16) for x in g["scales"]]
    assert np.array_equal(scales[0, 0, 0], want_s)
    words = thumb[0, 0].view("<u4")
    assert words[0, 0] == int(g["thumb_word0_t0"][0], 16)
    assert words[1, 0] == int(g["thumb_word0_t1"][0], 16)
    assert (words[:, 1:] == int(g["thumb_other_words"][0], 16)).all()
    for t in range(2):
        assert list(resid[0, 0, t, :3]) == [int(x) for x in g[f"resid_t{t}"]]
        assert (resid[0, 0, t, 3:] == int(g["resid_other"][0])).all()
    q = np.zeros((1, 1, D), np.float32)
    q[0, 0, :3] = [float(x) for x in g["q"]]
    qb = to_bf16(q)
    qi, _ = oracle.fold_query_tr(qb[0, 0], scales[0, 0, 0])
    assert list(qi[:3]) == [int(x) for x in g["qi"]] and not qi[3:].any()
    sc = oracle.block_scores_tr(qb, thumb, scales, lengths, T)
    assert abs(sc[0, 0, 0] - float(g["score"][0])) < 1e-6
    khat = oracle.reconstruct_keys_tr(thumb, resid, scales, lengths, T)
    sf = from_bf16(scales[0, 0, 0]).astype(np.float64)
    for t in range(2):
        z = np.array([int(x) for x in g[f"z_t{t}"]], np.float64)
        assert np.array_equal(khat[0, 0, t, :3], sf[:3] * z / 254)
    assert not khat[0, 0, :, 3:].any()


def test_thumbnail_is_a_nearest_level_and_scale_bound():
    T = 64
    k = _rand_keys(21, cap=256)
    lengths = np.array([256, 200], np.int32)
    thumb, resid, scales = oracle.quantize_keys_tr(k, lengths, T)
    u = _thumb_codes(thumb)
    assert u.min() >= 0 and u.max() <= 3
    for b in range(2):
        n = int(lengths[b])
        for g in range(2):
            kf = from_bf16(k[b, g, :n]).astype(np.float64)
            s_blk = from_bf16(scales[b, g, :-(-n // T)]).astype(np.float64)
            sf = np.repeat(s_blk, T, axis=0)[:n]
            lvl = (u[b, g, :n] - 1.5) * sf
            # distance to the chosen level = distance to the nearest of the four
            all_lvls = (np.arange(4)[:, None, None] - 1.5) * sf[None]
            best = np.abs(kf[None] - all_lvls).min(axis=0)
            assert (np.abs(kf - lvl) <= best + 1e-12 * sf).all()
            # the scale is amax / 1.5 within half a bf16 ulp
            for j in range(s_blk.shape[0]):
                amax = np.abs(kf[j * T:(j + 1) * T]).max(axis=0)
                assert (np.abs(s_blk[j] - amax / 1.5) <= amax / 1.5 * 2.0**-8).all()


def test_reconstruction_error_bound_tail_and_untouched_blocks():
    T, cap = 64, 512
    k = _rand_keys(22, cap=cap)
    lengths = np.array([300, 130], np.int32)
    thumb = np.full((2, 2, cap, D // 4), 0x5A, np.uint8)
    resid = np.full((2, 2, cap, D), 0x5A, np.uint8)
    scales = fw.poison_scales((2, 2, cap // T, D))
    oracle.quantize_keys_tr(k, lengths, T, 0, thumb, resid, scales)
    khat = oracle.reconstruct_keys_tr(thumb, resid, scales, lengths, T)
    for b in range(2):
        n = int(lengths[b])
        nb = -(-n // T)
        for g in range(2):
            kf = from_bf16(k[b, g, :n]).astype(np.float64)
            sf = np.repeat(from_bf16(scales[b, g, :nb]).astype(np.float64), T, axis=0)[:n]
            # 10-bit reconstruction: within half a residual step s / 254
            assert (np.abs(kf - khat[b, g, :n]) <= sf / 508 * (1 + 1e-5) + 1e-30).all()
            # tokens past the length in the last block are zero bytes
            assert not thumb[b, g, n:nb * T].any() and not resid[b, g, n:nb * T].any()
            # blocks past the length are not written
            assert (thumb[b, g, nb * T:] == 0x5A).all() and (resid[b, g, nb * T:] == 0x5A).all()
            assert (scales[b, g, nb:] == fw.SCALE_POISON_BF16).all()


def test_reconstruction_exact_on_half_scale_grid():
    # k = m s / 2 with m in [-3, 3], s = 2^e and |m| = 3 present in every
    # (block, channel): the scale is exactly s and k_hat == k exactly
    T, cap = 64, 256
    rng = np.random.default_rng(23)
    m = rng.integers(-3, 4, size=(1, 2, cap, D))
    for j in range(cap // T):
        m[:, :, j * T + rng.integers(0, T), :] = 3 * rng.choice([-1, 1], size=(1, 2, D))
    e = rng.integers(-8, 6, size=(1, 2, cap // T, D))
    k = (m * np.exp2(np.repeat(e, T, axis=2)) / 2).astype(np.float32)
    kb = to_bf16(k)
    assert np.array_equal(from_bf16(kb), k)
    lengths = np.array([cap], np.int32)
    thumb, resid, scales = oracle.quantize_keys_tr(kb, lengths, T)
    assert np.array_equal(from_bf16(scales), np.exp2(e).astype(np.float32))
    khat = oracle.reconstruct_keys_tr(thumb, resid, scales, lengths, T)
    assert np.array_equal(khat, k.astype(np.float64))
    # odd m sit on a thumbnail level: residual 0 (byte 128)
    odd = (m % 2) != 0
    assert (resid[odd] == 128).all()


def test_subnormal_keys_saturate_the_code():
    # k = +-2 * 2^-133 (bf16 subnormals): 2/1.5 * 2^-133 rounds to the bf16
    # subnormal 2^-133, so k / s = +-2: the code saturates at 3 (0) and the
    # residual at +127 (-127), which still reconstructs k exactly
    T, cap = 64, 64
    tiny = np.float32(2 * 2.0**-133)
    k = np.full((1, 1, cap, D), tiny, np.float32)
    k[0, 0, 1::2] = -tiny
    kb = to_bf16(k)
    assert np.array_equal(from_bf16(kb), k)
    lengths = np.array([cap], np.int32)
    thumb, resid, scales = oracle.quantize_keys_tr(kb, lengths, T)
    assert (from_bf16(scales) == np.float32(2.0**-133)).all()
    u = _thumb_codes(thumb)
    assert (u[0, 0, 0::2] == 3).all() and (u[0, 0, 1::2] == 0).all()
    assert (resid[0, 0, 0::2] == 255).all() and (resid[0, 0, 1::2] == 1).all()
    khat = oracle.reconstruct_keys_tr(thumb, resid, scales, lengths, T)
    assert np.array_equal(khat, k.astype(np.float64))


def test_append_equals_from_scratch():
    T, cap = 64, 512
    k = _rand_keys(24, B=1, cap=cap)
    L = 333
    ref = oracle.quantize_keys_tr(k, np.array([L], np.int32), T)
    th, re, sc = oracle.quantize_keys_tr(k, np.array([90], np.int32), T)
    for n in range(91, L + 1):
        oracle.quantize_keys_tr(k, np.array([n], np.int32), T, -1, th, re, sc)
    nb = -(-L // T)
    assert np.array_equal(th[:, :, :nb * T], ref[0][:, :, :nb * T])
    assert np.array_equal(re[:, :, :nb * T], ref[1][:, :, :nb * T])
    assert np.array_equal(sc[:, :, :nb], ref[2][:, :, :nb])


def test_thumbnail_scores_integer_case():
    # keys on the thumbnail levels with power-of-two scales and a query whose
    # folded values are exact (entries 0 or +-qmax 2^-e_c): the score is
    # max_t (q . k_t) / sqrt(D) up to two fp32 roundings
    T, cap = 64, 256
    rng = np.random.default_rng(25)
    lvl = rng.choice([-3, -1, 1, 3], size=(1, 1, cap, D))
    for j in range(cap // T):
        lvl[:, :, j * T, :] = 3
    e = rng.integers(-4, 4, size=(1, 1, cap // T, D))
    k = (lvl * np.exp2(np.repeat(e, T, axis=2)) / 2).astype(np.float32)
    lengths = np.array([cap - 7], np.int32)
    thumb, resid, scales = oracle.quantize_keys_tr(to_bf16(k), lengths, T)
    assert np.array_equal(from_bf16(scales), np.exp2(e).astype(np.float32))
    for j in range(cap // T):
        sign = rng.choice([-1, 0, 1], size=(2, D))
        sign[:, 0] = 1
        q = (sign * np.exp2(-e[0, 0, j])).astype(np.float32)[None]
        sc = oracle.block_scores_tr(to_bf16(q), thumb, scales, lengths, T)
        t1 = min((j + 1) * T, int(lengths[0]))
        dots = q[0].astype(np.float64) @ k[0, 0, j * T:t1].astype(np.float64).T
        want = dots.max(axis=1) / math.sqrt(D)
        assert np.allclose(sc[0, :, j], want, rtol=3e-7, atol=0)


def test_thumbnail_scores_within_quantisation_bound():
    T, cap = 64, 512
    k = _rand_keys(26, cap=cap)
    rng = np.random.default_rng(27)
    q = to_bf16(rng.standard_normal((2, 8, D)).astype(np.float32))
    lengths = np.array([512, 301], np.int32)
    thumb, resid, scales = oracle.quantize_keys_tr(k, lengths, T)
    sc = oracle.block_scores_tr(q, thumb, scales, lengths, T)
    u = _thumb_codes(thumb)
    G = 4
    for b in range(2):
        n = int(lengths[b])
        for h in range(8):
            g = h // G
            qh = from_bf16(q[b, h]).astype(np.float64)
            for j in range(-(-n // T)):
                s = from_bf16(scales[b, g, j]).astype(np.float64)
                lv = 2 * u[b, g, j * T:min((j + 1) * T, n)] - 3  # level (2u-3) s/2
                exact = (lv * s / 2) @ qh / math.sqrt(D)
                a = np.abs(qh * s).max()
                bound = a / 508 * np.abs(lv).sum(axis=1).max() / math.sqrt(D)
                assert abs(sc[b, h, j] - exact.max()) <= bound * (1 + 1e-5) + 1e-6
            assert (sc[b, h, -(-n // T):] == -np.inf).all()


def _sdpa(q, k64, v, lengths, G, token_keep=None):
    B, Hq, _ = q.shape
    out = np.zeros((B, Hq, D))
    for b in range(B):
        n = int(lengths[b])
        if n == 0:
            continue
        qq = torch.from_numpy(from_bf16(q[b]).astype(np.float64))[:, None, :]
        kk = torch.from_numpy(k64[b, :, :n]).repeat_interleave(G, 0)
        vv = torch.from_numpy(from_bf16(v[b, :, :n]).astype(np.float64)).repeat_interleave(G, 0)
        mask = None
        if token_keep is not None:
            mask = torch.from_numpy(token_keep[b][:, :n]).repeat_interleave(G, 0)[:, None, :]
            if not bool(mask.any()):
                continue
        out[b] = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask)[:, 0].numpy()
    return out


def test_power_of_two_scaling_carries_through_thumbnails_and_scores():
    # bf16(amax / 1.5) and k / s commute with a 2^e scaling of K, so the
    # thumbnails and residuals stay the same, the scales and the reconstructed
    # keys gain 2^e, and every thumbnail block score (with q scaled as well)
    # is multiplied by exactly 2^(e_k + e_q).
    T, cap = 64, 512
    k = _rand_keys(30, cap=cap)
    rng = np.random.default_rng(31)
    q = to_bf16(rng.standard_normal((2, 8, D)).astype(np.float32))
    lengths = np.array([512, 190], np.int32)
    thumb, resid, scales = oracle.quantize_keys_tr(k, lengths, T)
    sc = oracle.block_scores_tr(q, thumb, scales, lengths, T)
    khat = oracle.reconstruct_keys_tr(thumb, resid, scales, lengths, T)
    for ek, eq in [(4, 0), (-3, 2)]:
        k2 = to_bf16((from_bf16(k) * np.float32(2.0**ek)).astype(np.float32))
        q2 = to_bf16((from_bf16(q) * np.float32(2.0**eq)).astype(np.float32))
        thumb2, resid2, scales2 = oracle.quantize_keys_tr(k2, lengths, T)
        assert np.array_equal(thumb2, thumb) and np.array_equal(resid2, resid)
        assert np.array_equal(from_bf16(scales2), from_bf16(scales) * np.float32(2.0**ek))
        khat2 = oracle.reconstruct_keys_tr(thumb2, resid2, scales2, lengths, T)
        assert np.array_equal(khat2, khat * 2.0**ek)
        sc2 = oracle.block_scores_tr(q2, thumb2, scales2, lengths, T)
        assert np.array_equal(sc2, sc * np.float32(2.0**(ek + eq)))


def test_thumbnail_copy_and_scores_equivariant_under_permutations():
    # Per-channel quantisation, an elementwise fold with a permutation-
    # invariant max, exact integer sums and a max over tokens: permuting q's
    # and K's channels together permutes thumbnails, residuals, scales and
    # reconstructed keys with them and leaves every block score bit-identical;
    # shuffling the valid tokens inside each block leaves scales and scores
    # unchanged.
    T, cap = 64, 512
    k = _rand_keys(28, cap=cap)
    rng = np.random.default_rng(29)
    q = to_bf16(rng.standard_normal((2, 8, D)).astype(np.float32))
    lengths = np.array([512, 237], np.int32)
    thumb, resid, scales = oracle.quantize_keys_tr(k, lengths, T)
    sc = oracle.block_scores_tr(q, thumb, scales, lengths, T)
    khat = oracle.reconstruct_keys_tr(thumb, resid, scales, lengths, T)
    perm = rng.permutation(D)
    thumb_c, resid_c, scales_c = oracle.quantize_keys_tr(np.ascontiguousarray(k[..., perm]), lengths, T)
    assert np.array_equal(scales_c, scales[..., perm])
    assert np.array_equal(_thumb_codes(thumb_c), _thumb_codes(thumb)[..., perm])
    assert np.array_equal(resid_c, resid[..., perm])
    assert np.array_equal(oracle.reconstruct_keys_tr(thumb_c, resid_c, scales_c, lengths, T),
                          khat[..., perm])
    sc_c = oracle.block_scores_tr(np.ascontiguousarray(q[..., perm]), thumb_c, scales_c, lengths, T)
    assert np.array_equal(sc_c, sc)
    k_t = k.copy()
    for b in range(k.shape[0]):
        n = int(lengths[b])
        for j0 in range(0, n, T):
            idx = np.arange(j0, min(j0 + T, n))
            k_t[b, :, idx] = k[b, :, rng.permutation(idx)]
    thumb_t, _, scales_t = oracle.quantize_keys_tr(k_t, lengths, T)
    assert np.array_equal(scales_t, scales)
    assert np.array_equal(oracle.block_scores_tr(q, thumb_t, scales_t, lengths, T), sc)


@pytest.mark.parametrize("delta", [math.inf, 1.0])
def test_decode_tr_on_exact_keys_equals_library_attention(delta):
    # keys on the half-scale grid are reconstructed exactly, so the computer
    # must equal torch's fp64 attention over the original keys (restricted to
    # the selected blocks)
    T, cap, G, S = 64, 512, 4, 3
    rng = np.random.default_rng(28)
    m = rng.integers(-3, 4, size=(2, 2, cap, D))
    m[:, :, ::T, :] = 3
    e = rng.integers(-3, 2, size=(2, 2, cap // T, D))
    k = (m * np.exp2(np.repeat(e, T, axis=2)) / 2).astype(np.float32)
    v = to_bf16(rng.standard_normal((2, 2, cap, D)).astype(np.float32))
    q = to_bf16(rng.standard_normal((2, 8, D)).astype(np.float32))
    lengths = np.array([cap, 333], np.int32)
    thumb, resid, scales = oracle.quantize_keys_tr(to_bf16(k), lengths, T)
    out, mask, _ = oracle.decode_tr(q, v, thumb, resid, scales, lengths, T, S, delta)
    keep = []
    for b in range(2):
        keep.append(np.stack([np.repeat(oracle.mask_to_blocks(mask[b, g], cap // T), T)
                              for g in range(2)]))
    want = _sdpa(q, k.astype(np.float64), v, lengths, G, keep)
    assert np.abs(out - want).max() < 1e-9
    if math.isinf(delta):
        for b in range(2):
            assert oracle.mask_to_blocks(mask[b, 0], cap // T).sum() == -(-int(lengths[b]) // T)


def test_attend_tr_is_attention_over_reconstructed_keys():
    T, cap, G = 64, 256, 2
    k = _rand_keys(29, cap=cap)
    rng = np.random.default_rng(30)
    v = to_bf16(rng.standard_normal((2, 2, cap, D)).astype(np.float32))
    q = to_bf16(rng.standard_normal((2, 4, D)).astype(np.float32))
    lengths = np.array([256, 77], np.int32)
    thumb, resid, scales = oracle.quantize_keys_tr(k, lengths, T)
    mask = np.full((2, 2, 1), 0b1011, np.uint32)
    out, _ = oracle.attend_tr(q, thumb, resid, scales, v, lengths, mask, T)
    khat = oracle.reconstruct_keys_tr(thumb, resid, scales, lengths, T)
    keep = [np.stack([np.repeat(oracle.mask_to_blocks(mask[b, g], cap // T), T) for g in range(2)])
            for b in range(2)]
    assert np.abs(out - _sdpa(q, khat, v, lengths, G, keep)).max() < 1e-9
    # and close to attention over the original keys (10-bit reconstruction)
    dense = np.full((2, 2, 1), 0xF, np.uint32)
    out_d, _ = oracle.attend_tr(q, thumb, resid, scales, v, lengths, dense, T)
    ref = _sdpa(q, from_bf16(k).astype(np.float64), v, lengths, G)
    assert np.abs(out_d - ref).max() < 2e-2


@pytest.mark.parametrize("G,T", [(1, 128), (8, 128)])
def test_block_size_128_and_other_group_sizes(G, T):
    # the pins above run T = 64; the GPU path also serves T = 128 and every G
    cap = 1024
    k = _rand_keys(40 + G, cap=cap)
    rng = np.random.default_rng(41 + G)
    v = to_bf16(rng.standard_normal((2, 2, cap, D)).astype(np.float32))
    q = to_bf16(rng.standard_normal((2, 2 * G, D)).astype(np.float32))
    lengths = np.array([1024, 333], np.int32)
    thumb, resid, scales = oracle.quantize_keys_tr(k, lengths, T)
    khat = oracle.reconstruct_keys_tr(thumb, resid, scales, lengths, T)
    u = _thumb_codes(thumb)
    sc = oracle.block_scores_tr(q, thumb, scales, lengths, T)
    for b in range(2):
        n = int(lengths[b])
        nb = -(-n // T)
        for g in range(2):
            kf = from_bf16(k[b, g, :n]).astype(np.float64)
            sf = np.repeat(from_bf16(scales[b, g, :nb]).astype(np.float64), T, axis=0)[:n]
            assert (np.abs(kf - khat[b, g, :n]) <= sf / 508 * (1 + 1e-5) + 1e-30).all()
            assert not thumb[b, g, n:nb * T].any() and not resid[b, g, n:nb * T].any()
        for h in range(2 * G):
            g = h // G
            qh = from_bf16(q[b, h]).astype(np.float64)
            for j in range(nb):
                sj = from_bf16(scales[b, g, j]).astype(np.float64)
                lv = 2 * u[b, g, j * T:min((j + 1) * T, n)] - 3
                exact = (lv * sj / 2) @ qh / math.sqrt(D)
                bound = np.abs(qh * sj).max() / 508 * np.abs(lv).sum(axis=1).max() / math.sqrt(D)
                assert abs(sc[b, h, j] - exact.max()) <= bound * (1 + 1e-5) + 1e-6
    words = oracle.mask_words(cap, T)
    mask = rng.integers(0, 2**32, size=(2, 2, words), dtype=np.uint64).astype(np.uint32)
    out, _ = oracle.attend_tr(q, thumb, resid, scales, v, lengths, mask, T)
    keep = [np.stack([np.repeat(oracle.mask_to_blocks(mask[b, g], cap // T), T) for g in range(2)])
            for b in range(2)]
    assert np.abs(out - _sdpa(q, khat, v, lengths, G, keep)).max() < 1e-9


def test_decode_tr_mask_follows_thumbnail_scores():
    # the step's mask is the Top-delta selection (pinned by enumeration in the
    # int4 tests) applied to the thumbnail scores, for every reference
    w = fw.random_small_workload(31, batch=3, group=4, num_kv_heads=2, capacity=1024,
                                 block_size=64, split_blocks=3, delta=2.0, lengths_lo=1,
                                 lengths_hi=1024, needles=1)
    inp = fw.make_inputs(w)
    T = w.block_size
    thumb, resid, scales = oracle.quantize_keys_tr(inp["k"], inp["lengths"], T)
    sc = oracle.block_scores_tr(inp["q"], thumb, scales, inp["lengths"], T)
    for ref in (oracle.RUNNING_MAX, oracle.PSEUDO_MAX_SEEDED, oracle.PSEUDO_MAX_FIXED):
        for delta in (0.0, 1.5, 4.0):
            _, mask, sc2 = oracle.decode_tr(inp["q"], inp["v"], thumb, resid, scales, inp["lengths"],
                                            T, w.split_blocks, delta, reference=ref)
            assert np.array_equal(sc2, sc)
            _, want = oracle.select(sc, inp["lengths"], w.num_kv_heads, w.capacity, T,
                                    w.split_blocks, delta, reference=ref)
            assert np.array_equal(mask, want)


@pytest.mark.parametrize("name,overrides", [
    ("tiny", {}),
    ("llama", dict(batch=1, num_q_heads=8, num_kv_heads=2, capacity=8192, context=8192)),
    ("max256k", dict(num_q_heads=8, num_kv_heads=2, capacity=16384, context=16384, needles=6)),
    ("ragged", dict(batch=3, num_q_heads=8, num_kv_heads=2, capacity=16384, ragged=(4096, 16384))),
])
def test_planted_needles_selected_by_thumbnails(name, overrides):
    # the 2-bit thumbnails must still find the planted blocks (the pages use
    # them as the importance proxy)
    w = fw.scaled_workload(fw.WORKLOADS[name], **overrides)
    inp = fw.make_inputs(w)
    T = w.block_size
    thumb, _, scales = oracle.quantize_keys_tr(inp["k"], inp["lengths"], T)
    sc = oracle.block_scores_tr(inp["q"], thumb, scales, inp["lengths"], T)
    nblk = w.capacity // T
    for delta in (1.0, 2.0, 3.0, 4.0):
        keep, mask = oracle.select(sc, inp["lengths"], w.num_kv_heads, w.capacity, T,
                                   w.split_blocks, delta)
        for b in range(w.batch):
            for g in range(w.num_kv_heads):
                bits = oracle.mask_to_blocks(mask[b, g], nblk)
                for i, j in enumerate(inp["needles"][b]):
                    assert bits[j], (name, delta, b, g, j)
                    assert keep[b, g * w.group + i % w.group, j]


def test_tr_rejects_bad_arguments():
    k = np.zeros((1, 1, 128, D), np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.quantize_keys_tr(k, np.array([129], np.int32), 64)
    th, re, sc = oracle.quantize_keys_tr(k, np.array([100], np.int32), 64)
    q = np.zeros((1, 1, D), np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.decode_tr(q, k, th, re, sc, np.array([100], np.int32), 64, 2, -1.0)
    with pytest.raises(oracle.OracleError):
        oracle.decode_tr(q, k, th, re, sc, np.array([100], np.int32), 64, 0, 1.0)
