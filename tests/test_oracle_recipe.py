"""Pins of the oracle's two recipe options for the cache (reading note, "The inference
infrastructure": K-smoothing of K and adaptive scale selection of V within each chunk; reading
note, "Engineering details of NVFP4 training": candidate scale magnitudes {4, 6}).

The pages name both options and define neither.  The readings pinned here:
  K-smoothing  mu = the exact channel mean rounded once to fp32 (nearest, ties to even); x - mu
               is quantised; the key the cache stands for is x_hat' + mu.
  adaptive     per 16-element block, scale targets 6 and 4 are both tried and the one with the
               smaller fp64 squared error kept (ties keep 6); g is unchanged.
Each expected value below follows from the format constants by hand, from a closed form, or from
an invariant that a dropped term, a wrong sign or a swapped candidate would break.
"""
import numpy as np

import oracle
from tests._bf16 import bf16_bits_to_f32, f32_to_bf16_bits


def _bits(x, exact=True):
    """bf16 bit patterns of x; with ``exact`` the values must already be bf16 numbers."""
    x = np.asarray(x, np.float64)
    b = f32_to_bf16_bits(x.astype(np.float32))
    if exact:
        assert np.array_equal(bf16_bits_to_f32(b).astype(np.float64), x), "inputs must be exact bf16"
    return b


def _val(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


def _codes(codes, d):
    """E2M1 code of every element: [..., d/2] bytes -> [..., d] nibbles."""
    lo, hi = codes & 0xF, codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[:-1] + (d,))


def _deq(codes, scales, g, d):
    """x_hat = E2M1 * E4M3 * g (fp64) of one quantised chunk [B, H, L, ...]."""
    e2 = np.vectorize(oracle.e2m1_decode)(_codes(codes, d)).astype(np.float64)
    e4 = np.vectorize(oracle.e4m3_decode)(scales).astype(np.float64)
    return e2 * np.repeat(e4, 16, axis=-1) * g[:, :, None, None].astype(np.float64)


# ---------------------------------------------------------------- K-smoothing: the channel mean

def test_key_mean_of_constant_and_arithmetic_channels():
    L, d = 200, 16
    x = np.zeros((1, L, 1, d))
    consts = [0.0, 1.0, -3.5, 2.0 ** -30, 448.0, -0.009765625]
    for i, c in enumerate(consts):
        x[0, :, 0, i] = c                               # a constant channel: mean = the constant
    x[0, :, 0, 8] = np.arange(1, L + 1)                 # 1..200: mean (L + 1) / 2 = 100.5
    x[0, :, 0, 9] = np.where(np.arange(L) % 2 == 0, 7.0, -7.0)  # +-7 in turn: mean 0
    mu = oracle.key_mean(_bits(x))
    assert mu.shape == (1, 1, d) and mu.dtype == np.float32
    for i, c in enumerate(consts):
        assert mu[0, 0, i] == np.float32(c)
    assert mu[0, 0, 8] == np.float32(100.5)
    assert mu[0, 0, 9] == 0.0


def test_key_mean_is_exact_whatever_the_order():
    # [2^60, 1, -2^60, 1]: an fp64 running sum would lose the first 1 (2^60 + 1 rounds back to
    # 2^60) and give 0.25, a pairwise one 0; the exact mean is 0.5
    x = np.zeros((1, 4, 1, 16))
    x[0, :, 0, 0] = [2.0 ** 60, 1.0, -(2.0 ** 60), 1.0]
    x[0, :, 0, 1] = [1.0, 2.0 ** 60, 1.0, -(2.0 ** 60)]
    mu = oracle.key_mean(_bits(x))
    assert mu[0, 0, 0] == np.float32(0.5) and mu[0, 0, 1] == np.float32(0.5)


def test_key_mean_rounds_once_to_nearest_even():
    # (2^24 + 1) / 2 = 2^23 + 0.5 and (2^24 + 3) / 2 = 2^23 + 1.5 are exact fp32 midpoints: ties go
    # to the even significand; (2^24 + 2^17 + 1 + 2^-7) / 2 lies just above a midpoint and rounds up
    x = np.zeros((1, 2, 1, 16))
    x[0, :, 0, 0] = [2.0 ** 24, 1.0]
    x[0, :, 0, 1] = [2.0 ** 24, 3.0]
    x[0, :, 0, 2] = [2.0 ** 24 + 2.0 ** 17, 1.0 + 2.0 ** -7]  # mean 2^23 + 2^16 + 0.5 + 2^-8
    x[0, :, 0, 3] = [-(2.0 ** 24), -1.0]
    mu = oracle.key_mean(_bits(x))
    assert mu[0, 0, 0] == np.float32(2.0 ** 23)
    assert mu[0, 0, 1] == np.float32(2.0 ** 23 + 2.0)
    assert mu[0, 0, 2] == np.float32(2.0 ** 23 + 2.0 ** 16 + 1.0)
    assert mu[0, 0, 3] == np.float32(-(2.0 ** 23))


def _fp32_nearest(q):
    """Nearest fp32 to the rational q, ties to even, by bisection over positive bit patterns."""
    from fractions import Fraction
    import struct
    if q == 0:
        return 0.0
    neg, a = q < 0, abs(q)
    val = lambda u: Fraction(struct.unpack("<f", struct.pack("<I", u))[0])
    lo, hi = 0, 0x7F7FFFFF  # largest pattern with value <= a
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if val(mid) <= a:
            lo = mid
        else:
            hi = mid - 1
    below, above = val(lo), val(lo + 1)
    pick = lo if (a - below < above - a or (a - below == above - a and lo % 2 == 0)) else lo + 1
    f = struct.unpack("<f", struct.pack("<I", pick))[0]
    return -f if neg else f


def test_key_mean_against_exact_rationals():
    from fractions import Fraction
    rng = np.random.default_rng(21)
    for L, scale in ((3, 1.0), (7, 2.0 ** -130), (64, 2.0 ** 100), (200, 1.0), (5, 2.0 ** -140)):
        v = rng.standard_normal((1, L, 1, 16)) * scale * np.exp2(rng.integers(-20, 21, size=(1, L, 1, 16)))
        bits = _bits(v, exact=False)
        mu = oracle.key_mean(bits)
        vals = _val(bits)
        for i in range(16):
            want = _fp32_nearest(sum(Fraction(float(t)) for t in vals[0, :, 0, i]) / L)
            assert mu[0, 0, i] == np.float32(want), (L, scale, i)
    # a lone smallest subnormal among zeros: 2^-133 / 3 lies between fp32 subnormals
    x = np.zeros((1, 3, 1, 16))
    x[0, 0, 0, 0] = 2.0 ** -133
    mu = oracle.key_mean(_bits(x))
    assert mu[0, 0, 0] == np.float32(_fp32_nearest(Fraction(2) ** -133 / 3))
    assert mu[0, 0, 0] == np.float32(21845 * 2.0 ** -149)  # 2^16 / 3 = 21845.33 steps of 2^-149


def test_key_mean_per_head_and_batch_with_token_stride():
    rng = np.random.default_rng(3)
    B, L, H, d = 2, 9, 3, 32
    x = _bits(rng.standard_normal((B, L, H, d)), exact=False)
    mu = oracle.key_mean(x)
    # each (b, h) on its own, and a strided view of a wider token row gives the same means
    for b in range(B):
        for h in range(H):
            one = oracle.key_mean(np.ascontiguousarray(x[b:b + 1, :, h:h + 1]))
            assert np.array_equal(one[0, 0], mu[b, h])
    wide = np.zeros((B, L, H + 2, d), np.uint16)
    wide[:, :, :H] = x
    w = oracle.lib()
    out = np.zeros((B, H, d), np.float32)
    assert w.oracle_key_mean(oracle._ptr(wide), B, L, H, d, (H + 2) * d, oracle._ptr(out)) == 0
    assert np.array_equal(out, mu)


# ------------------------------------------------------- K-smoothing: the quantised chunk

def test_zero_mean_chunk_quantises_as_without_smoothing():
    # every channel holds +v, -v pairs in consecutive tokens: its token-order sum is exactly 0
    rng = np.random.default_rng(5)
    L, H, d = 24, 2, 128
    half = _val(_bits(rng.standard_normal((1, L // 2, H, d)), exact=False))
    half[..., 7] *= 16
    x = np.empty((1, L, H, d))
    x[:, 0::2], x[:, 1::2] = half, -half
    bits = _bits(x)
    mu = oracle.key_mean(bits)
    assert np.all(mu == 0.0)
    plain = oracle.quantize_chunk(bits)
    smooth = oracle.quantize_chunk(bits, mean=mu)
    for a, b in zip(plain, smooth):
        assert np.array_equal(a, b)


def test_a_chunk_of_one_repeated_key_reconstructs_exactly():
    rng = np.random.default_rng(6)
    L, H, d = 40, 2, 128
    v = _val(_bits(rng.standard_normal((1, 1, H, d)) * 4, exact=False))
    x = np.repeat(v, L, axis=1)
    bits = _bits(x)
    cache = oracle.Cache(1, H, d, L, 2, smooth_k=True)
    cache.append(1, bits, bits)
    assert np.array_equal(cache.k_mean[0, :, 1], v[0, 0].astype(np.float32))
    assert np.all(cache.k_g[:, :, 1] == 0.0) and np.all(cache.k_codes[:, :, L:] == 0)
    kh = cache.dequantize("k")[0, :, L:]                          # [H, L, d]
    assert np.array_equal(kh, np.broadcast_to(v[0, 0][:, None, :], (H, L, d)))
    # without smoothing the same chunk is only within the NVFP4 error bound
    plain = oracle.Cache(1, H, d, L, 2)
    plain.append(1, bits, bits)
    assert not np.array_equal(plain.dequantize("k")[0, :, L:], kh)


def test_smoothed_error_bound_and_offset_channels():
    rng = np.random.default_rng(8)
    B, L, H, d = 1, 64, 2, 128
    x = rng.standard_normal((B, L, H, d))
    x[..., 11] += 40.0                                # channels with a large offset
    x[..., 90] -= 25.0
    bits = _bits(x, exact=False)
    xf = _val(bits)
    mu = oracle.key_mean(bits)
    codes, scales, g = oracle.quantize_chunk(bits, mean=mu)
    xp = (bf16_bits_to_f32(bits) - mu[:, None, :, :]).astype(np.float64)  # the fp32 difference
    xh = _deq(codes, scales, g, d).transpose(0, 2, 1, 3)              # [B, L, H, d]
    e4 = np.vectorize(oracle.e4m3_decode)(scales).astype(np.float64)
    sg = (np.repeat(e4, 16, axis=-1) * g[:, :, None, None]).transpose(0, 2, 1, 3)
    # the same bound as unsmoothed NVFP4, on x - mu: |err| <= s * g
    assert np.all(np.abs(xp - xh) <= sg * 1.0001)
    rec = xh + mu[:, None, :, :].astype(np.float64)
    # the offset channels cost nothing: the smoothed error is far below the plain one there
    pc, ps, pg = oracle.quantize_chunk(bits)
    plain = _deq(pc, ps, pg, d).transpose(0, 2, 1, 3)
    e_s = np.sqrt(np.mean((rec - xf) ** 2))
    e_p = np.sqrt(np.mean((plain - xf) ** 2))
    assert e_s < 0.5 * e_p


# ------------------------------------------------------------- adaptive {4, 6} block scale

def _anchored(block, d=16):
    """Token 0 holds the chunk maximum 1344 (so g = 1344 / 2688 = 0.5 exactly), token 1 the block."""
    x = np.zeros((1, 2, 1, d))
    x[0, 0, 0, 0] = 1344.0
    x[0, 1, 0, :len(block)] = block
    return _bits(x)


def test_target_four_is_chosen_where_it_is_exact():
    # with g = 0.5 the block 2 * {0, .5, 1, 1.5, 2, 3, 4} has maximum 8: target 4 gives s = 4,
    # s g = 2 and every element an exact E2M1 code; target 6 gives s = E4M3(8 / 3) = 2.75, which
    # cannot represent the block
    vals = 2.0 * np.array([0, .5, 1, 1.5, 2, 3, 4, -.5, -1, -1.5, -2, -3, -4, 4, 3, 1])
    bits = _anchored(vals)
    c6, s6, g6 = oracle.quantize_chunk(bits)
    c4, s4, g4 = oracle.quantize_chunk(bits, adaptive=True)
    assert g6[0, 0] == g4[0, 0] == np.float32(0.5)
    assert oracle.e4m3_decode(int(s6[0, 0, 1, 0])) == 2.75
    assert oracle.e4m3_decode(int(s4[0, 0, 1, 0])) == 4.0
    x = vals.astype(np.float64)
    assert np.array_equal(_deq(c4, s4, g4, 16)[0, 0, 1], x)
    assert not np.array_equal(_deq(c6, s6, g6, 16)[0, 0, 1], x)
    # the anchor block would need a target-4 scale of 672 > 448; saturated it is no better, so
    # it keeps target 6 (s = 448)
    assert s4[0, 0, 0, 0] == s6[0, 0, 0, 0] and oracle.e4m3_decode(int(s4[0, 0, 0, 0])) == 448.0


def test_equal_errors_keep_target_six():
    # {6, 3, 1.5, 0} is exact under both targets (s = 2 for 6, s = 3 for 4): the tie keeps 6
    bits = _anchored(np.array([6.0, 3.0, 1.5, 0.0, -6.0, -3.0, -1.5]))
    c4, s4, g4 = oracle.quantize_chunk(bits, adaptive=True)
    assert oracle.e4m3_decode(int(s4[0, 0, 1, 0])) == 2.0
    c6, s6, _ = oracle.quantize_chunk(bits)
    assert np.array_equal(c4, c6) and np.array_equal(s4, s6)


def test_adaptive_blocks_are_never_worse_and_lower_the_total_error():
    rng = np.random.default_rng(9)
    B, L, H, d = 1, 48, 3, 128
    x = rng.standard_normal((B, L, H, d))
    x[..., 5] *= 20.0
    bits = _bits(x, exact=False)
    xf = _val(bits).transpose(0, 2, 1, 3)
    plain = _deq(*oracle.quantize_chunk(bits), d)
    adapt = _deq(*oracle.quantize_chunk(bits, adaptive=True), d)
    err_p = ((plain - xf) ** 2).reshape(B, H, L, d // 16, 16).sum(-1)
    err_a = ((adapt - xf) ** 2).reshape(B, H, L, d // 16, 16).sum(-1)
    assert np.all(err_a <= err_p * (1 + 1e-12))
    changed = np.mean(err_a < err_p)
    assert 0.05 < changed < 0.95                    # both targets occur
    assert err_a.sum() < err_p.sum()
    assert np.mean(err_a / err_p) < 0.9             # the typical block gains about a fifth


def test_adaptive_zero_and_underflow_blocks_match_target_six():
    x = np.zeros((1, 2, 1, 32))
    x[0, 0, 0, 0] = 2.0 ** 100                      # g = 2^100 / 2688: the other blocks' scales underflow
    x[0, 1, 0, 16:20] = [1.0, -2.0, 0.5, 3.0]
    bits = _bits(x)
    for a, b in zip(oracle.quantize_chunk(bits), oracle.quantize_chunk(bits, adaptive=True)):
        assert np.array_equal(a, b)


def test_cache_options_touch_only_their_tensor():
    rng = np.random.default_rng(10)
    B, Lc, H, d = 1, 32, 2, 128
    k = _bits(rng.standard_normal((B, Lc, H, d)) + 3.0, exact=False)
    v = _bits(rng.standard_normal((B, Lc, H, d)), exact=False)
    plain = oracle.Cache(B, H, d, Lc, 1)
    plain.append(0, k, v)
    ad = oracle.Cache(B, H, d, Lc, 1, adaptive_v=True)
    ad.append(0, k, v)
    sm = oracle.Cache(B, H, d, Lc, 1, smooth_k=True)
    sm.append(0, k, v)
    assert np.array_equal(ad.k_codes, plain.k_codes) and np.array_equal(ad.k_scales, plain.k_scales)
    assert not np.array_equal(ad.v_scales, plain.v_scales)
    assert np.array_equal(sm.v_codes, plain.v_codes) and np.array_equal(sm.v_scales, plain.v_scales)
    assert not np.array_equal(sm.k_codes, plain.k_codes)


# ------------------------------------------------------------ attention over smoothed keys

def test_attention_over_chunks_of_repeated_keys_closed_form():
    # every key of chunk c is u_c: smoothing stores u_c exactly (mu = u_c, x - mu = 0), so the
    # logits are sigma q . u_c and the output is sum_c n e^{s_c} Vbar_c / sum_c n e^{s_c}
    rng = np.random.default_rng(12)
    B, H, d, Lc, C = 1, 2, 128, 24, 4
    cache = oracle.Cache(B, H, d, Lc, C, smooth_k=True)
    us = []
    for slot in range(C):
        u = _val(_bits(rng.standard_normal((1, 1, H, d)) / 4, exact=False))
        us.append(u[0, 0])
        v = _bits(rng.standard_normal((B, Lc, H, d)), exact=False)
        cache.append(slot, _bits(np.repeat(u, Lc, axis=1)), v)
    q = _bits(rng.standard_normal((B, 5, H, d)), exact=False)
    rows = np.array([(0, h, i) for h in range(H) for i in range(5)], np.int32)
    got = oracle.attention_rows(q, cache, 3, 1, 2, rows)           # visible chunks 0, 2, 3
    vh = cache.dequantize("v")
    qf = bf16_bits_to_f32(q).astype(np.float64)
    sigma = 1.0 / np.sqrt(d)
    for r, (b, h, i) in enumerate(rows):
        s = np.array([sigma * qf[b, i, h] @ us[c][h] for c in (0, 2, 3)])
        w = np.exp(s - s.max())
        vbar = np.stack([vh[b, h, c * Lc:(c + 1) * Lc].mean(axis=0) for c in (0, 2, 3)])
        want = (w[:, None] * vbar).sum(0) / w.sum()
        assert np.allclose(got[r], want, rtol=0, atol=1e-12)


def test_attention_over_smoothed_keys_brute_force():
    rng = np.random.default_rng(13)
    B, H, d, Lc, C = 1, 2, 128, 20, 3
    cache = oracle.Cache(B, H, d, Lc, C, smooth_k=True, adaptive_v=True)
    for slot in range(C):
        k = rng.standard_normal((B, Lc, H, d)) + rng.standard_normal((1, 1, H, d)) * 4
        v = rng.standard_normal((B, Lc, H, d))
        cache.append(slot, f32_to_bf16_bits(k.astype(np.float32)), f32_to_bf16_bits(v.astype(np.float32)))
    q = f32_to_bf16_bits(rng.standard_normal((B, 7, H, d)).astype(np.float32))
    rows = np.array([(0, h, i) for h in range(H) for i in range(7)], np.int32)
    slots = [2, 0]
    got = oracle.attention_rows_slots(q, cache, slots, rows)
    kh, vh = cache.dequantize("k"), cache.dequantize("v")       # keys include mu
    keys = np.concatenate([np.arange(c * Lc, (c + 1) * Lc) for c in sorted(slots)])
    qf = bf16_bits_to_f32(q).astype(np.longdouble)
    for r, (b, h, i) in enumerate(rows):
        s = (kh[b, h, keys].astype(np.longdouble) @ qf[b, i, h]) / np.sqrt(np.longdouble(d))
        p = np.exp(s - s.max())
        want = (p[:, None] * vh[b, h, keys].astype(np.longdouble)).sum(0) / p.sum()
        assert np.allclose(got[r], want.astype(np.float64), rtol=0, atol=1e-12)
    # and smoothing matters: the same codes without mu give different outputs
    bare = oracle.Cache(B, H, d, Lc, C)
    for name in ("k_codes", "k_scales", "k_g", "v_codes", "v_scales", "v_g"):
        setattr(bare, name, getattr(cache, name))
    assert not np.allclose(oracle.attention_rows_slots(q, bare, slots, rows), got, atol=1e-3)
