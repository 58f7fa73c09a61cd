"""Pins of the oracle's sink+window attention: the visible-chunk rule against the workloads'
stated key totals, closed forms (one visible key, all keys equal), masked-key invariance,
and brute force against an explicit mask matrix in extended precision."""
import numpy as np
import pytest

import oracle
from tests._bf16 import bf16_bits_to_f32, f32_to_bf16_bits
from tests.conftest import read_golden


@pytest.mark.parametrize("row", read_golden("visible_key_totals.txt"), ids=lambda r: r[0])
def test_visible_key_totals_match_workloads(row):
    _, Lc, C, t, n_sink, window, total = row
    vis = oracle.visible_chunks(int(t), int(n_sink), int(window), int(C))
    assert len(vis) * int(Lc) == int(total)
    assert vis == sorted(set(vis))


def test_sink_inside_window_is_counted_once():
    assert oracle.visible_chunks(1, 1, 3, 8) == [0, 1]
    assert oracle.visible_chunks(0, 1, 1, 4) == [0]
    assert oracle.visible_chunks(5, 2, 2, 8) == [0, 1, 4, 5]
    assert oracle.visible_chunks(3, 0, 1, 4) == [3]


def _filled_cache(rng, B, H, d, Lc, C, gain=8.0):
    cache = oracle.Cache(B, H, d, Lc, C)
    raw = []
    for slot in range(C):
        k = rng.standard_normal((B, Lc, H, d))
        v = rng.standard_normal((B, Lc, H, d))
        k[..., 3] *= gain
        v[..., 5] *= gain
        kb, vb = f32_to_bf16_bits(k.astype(np.float32)), f32_to_bf16_bits(v.astype(np.float32))
        cache.append(slot, kb, vb)
        raw.append((kb, vb))
    return cache, raw


def _all_rows(B, H, Lq):
    return np.array([(b, h, i) for b in range(B) for h in range(H) for i in range(Lq)], np.int32)


def test_single_visible_key_returns_its_value_row():
    rng = np.random.default_rng(1)
    B, H, d, Lc, C = 1, 2, 32, 1, 3
    cache, _ = _filled_cache(rng, B, H, d, Lc, C)
    q = f32_to_bf16_bits(rng.standard_normal((B, 4, H, d)).astype(np.float32))
    out = oracle.attention_rows(q, cache, q_chunk=2, n_sink=0, window=1, rows=_all_rows(B, H, 4))
    vhat = cache.dequantize("v")
    for r, (b, h, i) in enumerate(_all_rows(B, H, 4)):
        assert np.array_equal(out[r], vhat[b, h, 2])


def test_equal_keys_give_the_mean_of_visible_values():
    rng = np.random.default_rng(2)
    B, H, d, Lc, C = 1, 2, 64, 8, 5
    cache = oracle.Cache(B, H, d, Lc, C)
    krow = rng.standard_normal((1, 1, H, d)).astype(np.float32)
    for slot in range(C):
        k = np.broadcast_to(krow, (B, Lc, H, d))
        v = rng.standard_normal((B, Lc, H, d)).astype(np.float32)
        cache.append(slot, f32_to_bf16_bits(k), f32_to_bf16_bits(v))
    q = f32_to_bf16_bits(rng.standard_normal((B, 3, H, d)).astype(np.float32))
    vis = oracle.visible_chunks(4, 1, 2, C)  # [0, 3, 4]
    out = oracle.attention_rows(q, cache, 4, 1, 2, _all_rows(B, H, 3))
    vhat = cache.dequantize("v")
    for r, (b, h, i) in enumerate(_all_rows(B, H, 3)):
        toks = np.concatenate([np.arange(c * Lc, (c + 1) * Lc) for c in vis])
        want = vhat[b, h, toks].mean(axis=0)
        assert np.max(np.abs(out[r] - want)) < 1e-12


def test_masked_chunks_have_no_effect():
    rng = np.random.default_rng(3)
    B, H, d, Lc, C = 2, 2, 32, 6, 6
    cache, _ = _filled_cache(rng, B, H, d, Lc, C)
    q = f32_to_bf16_bits(rng.standard_normal((B, 5, H, d)).astype(np.float32))
    rows = _all_rows(B, H, 5)
    base = oracle.attention_rows(q, cache, 4, 1, 2, rows)  # visible [0, 3, 4]
    for c in (1, 2, 5):
        t0, t1 = c * Lc, (c + 1) * Lc
        for arr in (cache.k_codes, cache.v_codes):
            arr[:, :, t0:t1] = rng.integers(0, 256, arr[:, :, t0:t1].shape, dtype=np.uint8)
        for arr in (cache.k_scales, cache.v_scales):
            arr[:, :, t0:t1] = rng.integers(0, 0x7F, arr[:, :, t0:t1].shape, dtype=np.uint8)
        cache.k_g[:, :, c] = 1e3
        cache.v_g[:, :, c] = -7.0
    again = oracle.attention_rows(q, cache, 4, 1, 2, rows)
    assert np.array_equal(base, again)


@pytest.mark.parametrize("case", [(1, 2, 16, 8, 5, 3, 1, 2, 4), (2, 1, 16, 3, 4, 1, 0, 1, 2),
                                  (1, 3, 32, 5, 6, 5, 2, 6, 3)])
def test_brute_force_with_explicit_mask(case):
    B, H, d, Lc, C, t, n_sink, window, Lq = case
    rng = np.random.default_rng(sum(case))
    cache, _ = _filled_cache(rng, B, H, d, Lc, C, gain=4.0)
    q = f32_to_bf16_bits((rng.standard_normal((B, Lq, H, d)) * 2).astype(np.float32))
    rows = _all_rows(B, H, Lq)
    out = oracle.attention_rows(q, cache, t, n_sink, window, rows, softmax_scale=0.0)
    khat = cache.dequantize("k").astype(np.longdouble)
    vhat = cache.dequantize("v").astype(np.longdouble)
    qf = bf16_bits_to_f32(q).astype(np.longdouble)
    T = Lc * C
    chunk_of = np.arange(T) // Lc
    mask = np.zeros(T, bool)
    for j in range(T):  # key j is visible iff its chunk is a sink chunk or within the window
        c = chunk_of[j]
        mask[j] = (c < n_sink) or (t - window < c <= t)
    sigma = np.longdouble(1.0) / np.sqrt(np.longdouble(d))
    for r, (b, h, i) in enumerate(rows):
        logits = (khat[b, h] @ qf[b, i, h]) * sigma
        logits = np.where(mask, logits, -np.inf)
        w = np.exp(logits - logits[mask].max())
        want = (w[:, None] * vhat[b, h]).sum(axis=0) / w.sum()
        assert np.max(np.abs(out[r] - want.astype(np.float64))) < 1e-12


def test_softmax_scale_default_is_inverse_sqrt_d():
    rng = np.random.default_rng(4)
    B, H, d, Lc, C = 1, 1, 64, 4, 2
    cache, _ = _filled_cache(rng, B, H, d, Lc, C)
    q = f32_to_bf16_bits(rng.standard_normal((B, 2, H, d)).astype(np.float32))
    rows = _all_rows(B, H, 2)
    a = oracle.attention_rows(q, cache, 1, 1, 1, rows, softmax_scale=0.0)
    b = oracle.attention_rows(q, cache, 1, 1, 1, rows, softmax_scale=1.0 / 8.0)
    c = oracle.attention_rows(q, cache, 1, 1, 1, rows, softmax_scale=0.5)
    assert np.array_equal(a, b)
    assert not np.allclose(a, c)
