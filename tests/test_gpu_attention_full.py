"""GPU parity of whole heads at full size, of repeated denoising calls on one cache, and of
queries whose magnitudes span many binades.

Sampled rows (test_gpu_attention.py) can miss a mistake that only shows at some tile position of
some kind of CTA.  Here every query row of two heads per full-size workload is compared with the
fp64 oracle: head (0, 0), and the head that the persistent launch splits between two CTAs in the
middle of the grid, so that a partial result and the combine kernel are always on the checked path.
"""
import ctypes
import dataclasses

import numpy as np
import pytest

import nvfp4_quantised_kv_b200 as nk
from nvfp4_quantised_kv_b200 import synthetic
from tests.gpu_util import (assert_attention_close, attention_rows_threaded, dev_bf16, gather_rows,
                            head_rows, kv_tiles, make_caches, sample_rows)

pytestmark = pytest.mark.gpu

W = synthetic.WORKLOADS


def _split_head(cache, w):
    """(b, h) of the first CTA in the second half of the grid whose first segment is part of a
    split item (so its result goes through a partial slot and the combine kernel)."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    nt = kv_tiles(w.chunk_tokens, w.visible_chunks)
    out = (ctypes.c_int32 * 8)()
    L = nk.lib()
    d = ctypes.byref(cache.desc)
    assert L.nvfp4kv_attention_plan(d, w.q_tokens, nt, sms, -1, -1, out) == nk.OK
    n_ctas = out[0]
    for cta in range(n_ctas // 2, n_ctas):
        assert L.nvfp4kv_attention_plan(d, w.q_tokens, nt, sms, cta, 0, out) == nk.OK
        if out[7] >= 0:
            return out[2] // w.heads, out[2] % w.heads
    raise AssertionError("no split item in the second half of the grid")


@pytest.mark.parametrize("key,layer", [("1.3b", 0), ("5b", 0), ("rollout", 17), ("fewstep", 0)])
def test_full_size_two_whole_heads_all_rows(key, layer):
    w = W[key]
    cache, ocache = make_caches(w, w.visible_chunks, layer)
    split = _split_head(cache, w)
    heads = sorted({(0, 0), split})
    qb = synthetic.queries(w, layer)
    out = cache.attention(dev_bf16(qb), w.q_chunk, w.n_sink, w.window)
    assert cache.read_status() == 0
    rows = head_rows(w, heads)
    want = attention_rows_threaded(qb, ocache, w.q_chunk, w.n_sink, w.window, rows)
    assert_attention_close(gather_rows(out.cpu().numpy(), rows), want, f"{key} heads {heads}")


def test_fewstep_four_then_two_denoising_calls_on_one_cache():
    """The few-step schedule attends to one quantised cache repeatedly: four denoising calls, then
    two more, each with the queries of its own step.  Every call matches the oracle, the calls
    leave the cache bytes as they were, and a repeated call gives the same bits."""
    import torch
    w = W["fewstep"]
    cache, ocache = make_caches(w, w.visible_chunks)
    names = ("k_codes", "v_codes", "k_scales", "v_scales", "k_gscale", "v_gscale")
    before = {n: getattr(cache, n).clone() for n in names}
    rows = sample_rows(w, 6, seed=11)
    first = None
    for step in list(range(4)) + [4, 5]:
        qb = synthetic.queries(w, 0, step)
        out = cache.attention(dev_bf16(qb), w.q_chunk, w.n_sink, w.window)
        assert cache.read_status() == 0
        want = attention_rows_threaded(qb, ocache, w.q_chunk, w.n_sink, w.window, rows)
        assert_attention_close(gather_rows(out.cpu().numpy(), rows), want, f"fewstep step {step}")
        if step == 0:
            first = out.clone()
    for n in names:
        assert torch.equal(getattr(cache, n).view(torch.uint8), before[n].view(torch.uint8)), n
    again = cache.attention(dev_bf16(synthetic.queries(w, 0, 0)), w.q_chunk, w.n_sink, w.window)
    assert torch.equal(again.view(torch.int32), first.view(torch.int32))


def _scaled_case(q_scale_fn, k_factor):
    """tiny-shaped case (2 heads, ragged tiles, two runs) with K multiplied by ``k_factor`` and
    each query row multiplied element-wise by ``q_scale_fn(shape)``."""
    from tests._bf16 import bf16_bits_to_f32, f32_to_bf16_bits
    w = dataclasses.replace(W["tiny"], key="scaled", batch=2, heads=3, chunk_tokens=200, capacity=6,
                            q_chunk=4, n_sink=1, window=2, q_tokens=300)
    cache, ocache = make_caches(w, [])
    for slot in w.visible_chunks:
        k, v = synthetic.chunk_kv(w, slot)
        k = f32_to_bf16_bits(bf16_bits_to_f32(k) * np.float32(k_factor))
        cache.quantize(slot, dev_bf16(k), dev_bf16(v))
        ocache.append(slot, k, v)
    q = bf16_bits_to_f32(synthetic.queries(w))
    qb = f32_to_bf16_bits((q * q_scale_fn(q.shape)).astype(np.float32))
    out = cache.attention(dev_bf16(qb), w.q_chunk, w.n_sink, w.window)
    assert cache.read_status() == 0
    rows = head_rows(w, [(b, h) for b in range(w.batch) for h in range(w.heads)])
    want = attention_rows_threaded(qb, ocache, w.q_chunk, w.n_sink, w.window, rows)
    return gather_rows(out.cpu().numpy(), rows), want


def test_tiny_queries_against_large_keys():
    # |q| ~ 2^-20 (all of fp16's subnormal range and below without a prescale) against keys
    # scaled by 2^20: the logits stay of order one, so a query rounded to fp16 subnormals would
    # move them by several per cent
    got, want = _scaled_case(lambda s: np.float32(2.0 ** -20), 2.0 ** 20)
    assert_attention_close(got, want, "tiny q")


def test_query_rows_of_very_different_magnitudes_in_one_tile():
    # every row gets its own scale 2^r, r in [-40, 20], and every element a further 2^-u,
    # u in [0, 40]: the tiles mix rows of very different size, and rows mix elements far below
    # their largest; keys are scaled down so that the largest rows keep moderate logits
    rng = np.random.default_rng(7)

    def scale(shape):
        B, Lq, H, d = shape
        r = rng.integers(-40, 21, size=(B, Lq, H, 1))
        u = rng.integers(0, 41, size=(B, Lq, H, d))
        u[..., 0] = 0  # each row keeps one element at its own scale
        return np.ldexp(np.float32(1.0), (r - u).astype(np.int32)).astype(np.float32)

    got, want = _scaled_case(scale, 2.0 ** -20)
    assert_attention_close(got, want, "mixed-magnitude q")
