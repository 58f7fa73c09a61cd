"""Pins of the oracle's multi-shot attention sink (paper page, section 4.2 "Inference with
Multi-Shot Attention Sink"; reading note, "Multi-shot attention sinks"): the effective chunk set
global sink U shot sink (start, len) U window with overlaps counted once, worked by hand; the
reduction to the sink + window rule; brute force over an explicit mask in extended precision;
invariance of the slot-list attention to order and repeats."""
import numpy as np
import pytest

import oracle
from tests._bf16 import bf16_bits_to_f32, f32_to_bf16_bits
from tests.test_oracle_attention import _all_rows, _filled_cache


@pytest.mark.parametrize("args,want", [
    # chunk 9, global sink {0}, shot started at chunk 4 with a 2-chunk sink, window {8, 9}
    ((9, 1, 2, 4, 2, 12), [0, 4, 5, 8, 9]),
    # the shot sink {4, 5} overlaps the window {3, 4, 5}: each chunk once
    ((5, 1, 3, 4, 2, 12), [0, 3, 4, 5]),
    # the shot starts at the video start: shot sink inside the global sink
    ((7, 2, 1, 0, 1, 8), [0, 1, 7]),
    # no global sink, a shot sink and a one-chunk window
    ((10, 0, 1, 6, 3, 11), [6, 7, 8, 10]),
])
def test_multishot_sets_by_hand(args, want):
    assert oracle.multishot_chunks(*args) == want


@pytest.mark.parametrize("q,n_sink,window,cap", [(5, 2, 2, 8), (3, 1, 3, 4), (0, 0, 1, 2), (39, 1, 7, 40)])
def test_empty_shot_sink_reduces_to_sink_plus_window(q, n_sink, window, cap):
    assert oracle.multishot_chunks(q, n_sink, window, 0, 0, cap) == oracle.visible_chunks(q, n_sink, window, cap)


def test_shot_sink_in_the_future_is_rejected():
    with pytest.raises(ValueError):
        oracle.multishot_chunks(5, 1, 2, 5, 2, 12)


@pytest.mark.parametrize("case", [(1, 2, 16, 4, 12, 9, 1, 2, 4, 2, 3), (2, 1, 32, 3, 10, 9, 2, 1, 5, 1, 2),
                                  (1, 1, 16, 5, 16, 15, 1, 2, 6, 3, 2)])
def test_brute_force_with_explicit_multishot_mask(case):
    B, H, d, Lc, C, t, n_sink, window, s0, slen, Lq = case
    rng = np.random.default_rng(sum(case))
    cache, _ = _filled_cache(rng, B, H, d, Lc, C, gain=4.0)
    q = f32_to_bf16_bits((rng.standard_normal((B, Lq, H, d)) * 2).astype(np.float32))
    rows = _all_rows(B, H, Lq)
    slots = oracle.multishot_chunks(t, n_sink, window, s0, slen, C)
    out = oracle.attention_rows_slots(q, cache, slots, rows)
    khat = cache.dequantize("k").astype(np.longdouble)
    vhat = cache.dequantize("v").astype(np.longdouble)
    qf = bf16_bits_to_f32(q).astype(np.longdouble)
    chunk_of = np.arange(Lc * C) // Lc
    # key j is visible iff its chunk is in the global sink, the shot sink or the window
    mask = (chunk_of < n_sink) | ((chunk_of >= s0) & (chunk_of < s0 + slen)) | \
           ((chunk_of > t - window) & (chunk_of <= t))
    sigma = np.longdouble(1.0) / np.sqrt(np.longdouble(d))
    for r, (b, h, i) in enumerate(rows):
        logits = np.where(mask, (khat[b, h] @ qf[b, i, h]) * sigma, -np.inf)
        w = np.exp(logits - logits[mask].max())
        want = (w[:, None] * vhat[b, h]).sum(axis=0) / w.sum()
        assert np.max(np.abs(out[r] - want.astype(np.float64))) < 1e-12


def test_slot_list_order_and_repeats_do_not_matter():
    rng = np.random.default_rng(7)
    B, H, d, Lc, C = 1, 2, 32, 4, 9
    cache, _ = _filled_cache(rng, B, H, d, Lc, C)
    q = f32_to_bf16_bits(rng.standard_normal((B, 3, H, d)).astype(np.float32))
    rows = _all_rows(B, H, 3)
    a = oracle.attention_rows_slots(q, cache, [0, 3, 4, 7, 8], rows)
    b = oracle.attention_rows_slots(q, cache, [8, 4, 0, 7, 3, 4, 8, 0], rows)
    assert np.array_equal(a, b)


def test_window_slot_list_equals_the_window_rule():
    rng = np.random.default_rng(8)
    B, H, d, Lc, C = 2, 1, 32, 3, 6
    cache, _ = _filled_cache(rng, B, H, d, Lc, C)
    q = f32_to_bf16_bits(rng.standard_normal((B, 4, H, d)).astype(np.float32))
    rows = _all_rows(B, H, 4)
    a = oracle.attention_rows(q, cache, 4, 1, 2, rows)
    b = oracle.attention_rows_slots(q, cache, oracle.visible_chunks(4, 1, 2, C), rows)
    assert np.array_equal(a, b)


def test_slot_list_arguments_are_checked():
    rng = np.random.default_rng(9)
    cache, _ = _filled_cache(rng, 1, 1, 16, 2, 3)
    q = f32_to_bf16_bits(rng.standard_normal((1, 1, 1, 16)).astype(np.float32))
    for bad in ([], [3], [-1, 0]):
        with pytest.raises(ValueError):
            oracle.attention_rows_slots(q, cache, bad, _all_rows(1, 1, 1))
