"""Pins of the oracle's NVFP4 quantiser: exact round trips at the format's fixed points,
round-half-even ties, the zero / underflow special cases, invariances and the storage
closed form.  None of these re-derives the oracle's formula: each expected value follows
from the format constants (16-element blocks, M_FP8 = 448, M_FP4 = 6) by hand."""
import numpy as np
import pytest

import oracle
from tests._bf16 import bf16_bits_to_f32, f32_to_bf16_bits
from tests.conftest import read_golden

E2M1 = {int(c): float(v) for c, v in read_golden("e2m1_values.txt")}
POS_E4M3 = [c for c in range(1, 127)]  # every positive finite E4M3 code


def _e4m3_value(code):
    return oracle.e4m3_decode(code)


def _fixed_point_chunk(k, d=128):
    """Blocks [6*s, c_1*s, ..., c_15*s] * 2^k for every positive finite E4M3 scale s and
    every E2M1 code c; a block with s = 448 carries the chunk maximum 2688 * 2^k, so the
    FP32 scale is exactly 2^k and every value must survive the round trip bit for bit."""
    others = [c for c in range(16) if c != 7]  # 15 codes; 6.0 (code 7) leads each block
    scales = POS_E4M3 + [0x7E] * ((-len(POS_E4M3)) % (d // 16))
    nblk = len(scales)
    x = np.zeros(nblk * 16, np.float64)
    for b, s_code in enumerate(scales):
        s = _e4m3_value(s_code)
        x[b * 16] = 6.0 * s
        for j, c in enumerate(others):
            x[b * 16 + 1 + j] = E2M1[c] * s
    x = x * 2.0 ** k
    L = x.size // d
    return x.reshape(1, L, 1, d)


@pytest.mark.parametrize("k", [0, -20, 17, -100])
def test_fixed_points_roundtrip_exactly(k):
    x = _fixed_point_chunk(k)
    bits = f32_to_bf16_bits(x.astype(np.float32))
    assert np.array_equal(bf16_bits_to_f32(bits).astype(np.float64), x)  # inputs are exact bf16
    codes, scales, g = oracle.quantize_chunk(bits)
    assert g[0, 0] == np.float32(2.0 ** k)
    cache = oracle.Cache(1, 1, 128, x.shape[1], 1)
    cache.k_codes[:] = codes
    cache.k_scales[:] = scales
    cache.k_g[:, :, 0] = g
    back = cache.dequantize("k").reshape(-1)
    assert np.array_equal(back, x.reshape(-1))


def test_ties_round_half_to_even():
    ties = [(float(v), int(c)) for v, c in read_golden("e2m1_ties.txt")]
    mids = [(v, c) for v, c in ties if abs(v) < 6.0 and v not in (0.2499, 0.2501, 4.9999, 5.0001)]
    d = 16
    row = [6.0] + [v for v, _ in mids]
    row = row + [0.0] * (d - len(row))
    for k in (0, -9, 12):
        x = np.array(row, np.float64).reshape(1, 1, 1, d) * 2.0 ** k
        # a second block-row holding the chunk maximum 2688 * 2^k pins g = 2^k
        anchor = np.zeros((1, 1, 1, d))
        anchor[..., 0] = 2688.0 * 2.0 ** k
        chunk = np.concatenate([x, anchor], axis=1)
        codes, scales, g = oracle.quantize_chunk(f32_to_bf16_bits(chunk.astype(np.float32)))
        assert g[0, 0] == np.float32(2.0 ** k)
        assert _e4m3_value(int(scales[0, 0, 0, 0])) == 1.0
        nib = [(codes[0, 0, 0, i // 2] >> (4 * (i % 2))) & 0xF for i in range(d)]
        assert nib[0] == 7
        for i, (_, want) in enumerate(mids):
            assert nib[1 + i] == want, (i, mids[i])


def test_zero_block_zero_chunk_and_negative_zero():
    d = 32
    x = np.zeros((1, 2, 1, d), np.float32)
    x[0, 0, 0, 16:] = np.linspace(-3, 3, 16)
    x[0, 1, 0, :16] = -0.0
    codes, scales, g = oracle.quantize_chunk(f32_to_bf16_bits(x))
    assert scales[0, 0, 0, 0] == 0 and np.all(codes[0, 0, 0, :8] == 0)
    assert scales[0, 0, 1, 0] == 0 and np.all(codes[0, 0, 1, :8] == 0)  # -0.0 block -> code 0
    zero = np.zeros((2, 3, 2, d), np.float32)
    codes, scales, g = oracle.quantize_chunk(f32_to_bf16_bits(zero))
    assert np.all(g == 0) and np.all(codes == 0) and np.all(scales == 0)


def test_block_scale_underflow_and_smallest_subnormal():
    d = 16
    k = 0
    g = 2.0 ** k
    chunk = np.zeros((1, 3, 1, d), np.float64)
    chunk[0, 0, 0, 0] = 2688.0 * g          # anchor: g = 2^k
    chunk[0, 1, 0, 0] = 6.0 * g * 2.0 ** -11  # a_b/(6g) = 2^-11 < 2^-10: rounds to scale 0
    chunk[0, 2, 0, 0] = 6.0 * g * 1.5 * 2.0 ** -10  # 0.75 * 2^-9: nearest scale is 2^-9
    codes, scales, gs = oracle.quantize_chunk(f32_to_bf16_bits(chunk.astype(np.float32)))
    assert gs[0, 0] == 1.0
    assert scales[0, 0, 1, 0] == 0 and np.all(codes[0, 0, 1] == 0)
    assert scales[0, 0, 2, 0] == 0x01
    # x * r = 1.5 * 2^-10 * 6 / 2^-9 = 4.5 -> nearest E2M1 is 4 (code 6)
    assert codes[0, 0, 2, 0] & 0xF == 6


def test_scale_product_underflow_gives_zero_codes():
    # chunk maximum 2^-113 gives g = 2^-113 / 2688 (about 2^-124.4); a block whose maximum is
    # the bf16 subnormal 2^-131 gets the smallest block scale 2^-9, and 2^-9 * g is so small
    # that 1 / (s * g) overflows fp32: that block's codes are all zero by rule.
    d = 16
    chunk = np.zeros((1, 2, 1, d), np.float64)
    chunk[0, 0, 0, 0] = 2.0 ** -113
    chunk[0, 1, 0, 0] = 2.0 ** -131
    chunk[0, 1, 0, 1] = -(2.0 ** -131)
    bits = f32_to_bf16_bits(chunk.astype(np.float32))
    assert bf16_bits_to_f32(bits)[0, 1, 0, 0] == np.float32(2.0 ** -131)
    codes, scales, gs = oracle.quantize_chunk(bits)
    assert gs[0, 0] == np.float32(2.0 ** -113) / np.float32(2688.0)
    assert scales[0, 0, 1, 0] == 0x01
    assert np.all(codes[0, 0, 1] == 0)
    assert scales[0, 0, 0, 0] == 0x7E  # the anchor block itself maps to 448


def _random_chunk(rng, B, L, H, d, gain=16.0):
    x = rng.standard_normal((B, L, H, d))
    ch = rng.integers(0, d, size=(B, H))
    for b in range(B):
        for h in range(H):
            x[b, :, h, ch[b, h]] *= gain
    return f32_to_bf16_bits(x.astype(np.float32))


def test_error_bound_and_head_independence():
    rng = np.random.default_rng(11)
    B, L, H, d = 2, 24, 3, 128
    bits = _random_chunk(rng, B, L, H, d)
    codes, scales, g = oracle.quantize_chunk(bits)
    cache = oracle.Cache(B, H, d, L, 1)
    cache.k_codes[:] = codes
    cache.k_scales[:] = scales
    cache.k_g[:, :, 0] = g
    xh = cache.dequantize("k")  # [B, H, L, d]
    x = bf16_bits_to_f32(bits).astype(np.float64).transpose(0, 2, 1, 3)
    s = np.vectorize(_e4m3_value)(scales).astype(np.float64)  # [B, H, L, d/16]
    sg = np.repeat(s, 16, axis=-1) * g[:, :, None, None].astype(np.float64)
    # E2M1 spacing is at most 2 (between 4 and 6) and clamping at 6 costs < 0.5: |err| <= s*g
    # (the 1e-4 slack covers the rounding of the fp32 reciprocal)
    assert np.all(np.abs(x - xh) <= sg * 1.0001)
    assert np.all(g > 0)
    # each (b, h) is quantised on its own: slicing one head out gives the same bytes
    c1, s1, g1 = oracle.quantize_chunk(np.ascontiguousarray(bits[1:2, :, 2:3, :]))
    assert np.array_equal(c1[0, 0], codes[1, 2]) and np.array_equal(s1[0, 0], scales[1, 2])
    assert g1[0, 0] == g[1, 2]


def test_power_of_two_scaling_moves_only_the_fp32_scale():
    rng = np.random.default_rng(5)
    bits = _random_chunk(rng, 1, 16, 2, 128)
    x = bf16_bits_to_f32(bits)
    c0, s0, g0 = oracle.quantize_chunk(bits)
    for k in (-30, -3, 9, 40):
        ck, sk, gk = oracle.quantize_chunk(f32_to_bf16_bits(x * np.float32(2.0 ** k)))
        assert np.array_equal(ck, c0) and np.array_equal(sk, s0)
        assert np.array_equal(gk, g0 * np.float32(2.0 ** k))


def test_token_stride_is_honoured():
    rng = np.random.default_rng(9)
    bits = _random_chunk(rng, 1, 8, 2, 128)
    padded = np.zeros((1, 8, 3, 128), np.uint16)  # token stride 3*128 > H*d
    padded[:, :, :2, :] = bits
    a = oracle.quantize_chunk(bits)
    flat = padded.reshape(1, 8, 3 * 128)
    x = oracle.lib()
    codes = np.zeros((1, 2, 8, 64), np.uint8)
    scales = np.zeros((1, 2, 8, 8), np.uint8)
    g = np.zeros((1, 2), np.float32)
    import ctypes
    rc = x.oracle_quantize_chunk(ctypes.c_void_p(flat.ctypes.data), 1, 8, 2, 128, 3 * 128,
                                 ctypes.c_void_p(codes.ctypes.data),
                                 ctypes.c_void_p(scales.ctypes.data), ctypes.c_void_p(g.ctypes.data))
    assert rc == 0
    assert np.array_equal(codes, a[0]) and np.array_equal(scales, a[1]) and np.array_equal(g, a[2])


def test_storage_closed_form_nine_eighths():
    # reading note, "The inference infrastructure": K+V storage falls from 4*Tc*H*d bytes
    # (bf16) to 9/8*Tc*H*d bytes (NVFP4), about 3.6x
    Tc, H, d = 4680, 12, 128
    codes, scales, _ = oracle.quantize_chunk(np.zeros((1, 4, 2, d), np.uint16))
    per_token_head = codes.shape[-1] + scales.shape[-1]  # bytes of one tensor, one token, one head
    nvfp4 = 2 * per_token_head * Tc * H
    assert nvfp4 * 8 == 9 * Tc * H * d
    assert round(4 * Tc * H * d / nvfp4, 2) == 3.56


def test_bad_arguments_are_rejected():
    with pytest.raises(ValueError):
        oracle.quantize_chunk(np.zeros((1, 2, 1, 24), np.uint16))  # d not a multiple of 16


def test_multi_chunk_dequantisation_uses_each_chunks_scale():
    # three chunks whose magnitudes differ by 10^3: dequantising with the wrong chunk's FP32
    # scale would be off by that factor, far outside the NVFP4 error bound checked above
    rng = np.random.default_rng(21)
    B, H, d, Lc, C = 1, 2, 128, 10, 3
    cache = oracle.Cache(B, H, d, Lc, C)
    xs = []
    for slot, mag in enumerate((1.0, 1e3, 1e-3)):
        k = (rng.standard_normal((B, Lc, H, d)) * mag).astype(np.float32)
        kb = f32_to_bf16_bits(k)
        cache.append(slot, kb, kb)
        xs.append(bf16_bits_to_f32(kb).astype(np.float64).transpose(0, 2, 1, 3))
    for which in ("k", "v"):
        xh = cache.dequantize(which)
        for slot in range(C):
            x = xs[slot]
            got = xh[:, :, slot * Lc:(slot + 1) * Lc]
            rel = np.linalg.norm(got - x) / np.linalg.norm(x)
            assert rel < 0.2, (which, slot, rel)
