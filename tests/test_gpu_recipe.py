"""GPU parity of the cache recipe options (reading note, "The inference infrastructure": K-smoothing
of K and adaptive scale selection of V within each chunk; "Engineering details of NVFP4 training":
candidate scale magnitudes {4, 6}).

The quantised bytes (codes, E4M3 scales, FP32 scales) and the channel means are compared with the
oracle bit for bit; attention over a smoothed cache is compared with the oracle's fp64 attention
over x_hat' + mu with the tolerance of the plain path."""
import ctypes
import dataclasses

import numpy as np
import pytest

import nvfp4_quantised_kv_b200 as nk
import oracle
from nvfp4_quantised_kv_b200 import KVCache, synthetic
from tests import special_chunks as sc
from tests._bf16 import bf16_bits_to_f32, f32_to_bf16_bits
from tests.gpu_util import (assert_attention_close, assert_cache_equal, attention_rows_threaded,
                            dev_bf16, gather_rows, head_rows, sample_rows)

pytestmark = pytest.mark.gpu

W = synthetic.WORKLOADS
OPTIONS = [(True, False), (False, True), (True, True)]


def _offset_kv(w, slot, layer=0):
    """The workload's chunk with a per-(chunk, head, channel) offset added to K (the structure
    K-smoothing removes): offsets N(0, 4) drawn from the chunk's own seed."""
    k, v = synthetic.chunk_kv(w, slot, layer)
    rng = np.random.default_rng(1000 + 97 * slot + layer)
    off = rng.standard_normal((1, 1, w.heads, w.head_dim)) * 4.0
    k = f32_to_bf16_bits((bf16_bits_to_f32(k) + off).astype(np.float32))
    return k, v


def _caches(w, slots, smooth, adaptive, offset=True, layer=0):
    cache = KVCache(w.batch, w.heads, w.chunk_tokens, w.capacity, q_tokens_max=w.q_tokens,
                    smooth_k=smooth, adaptive_v=adaptive)
    ocache = oracle.Cache(w.batch, w.heads, w.head_dim, w.chunk_tokens, w.capacity, smooth_k=smooth,
                          adaptive_v=adaptive)
    for slot in slots:
        k, v = _offset_kv(w, slot, layer) if offset else synthetic.chunk_kv(w, slot, layer)
        cache.quantize(slot, dev_bf16(k), dev_bf16(v))
        ocache.append(slot, k, v)
    return cache, ocache


def _assert_means_equal(cache, ocache, slots):
    got = cache.k_mean.cpu().numpy()
    for s in slots:
        assert np.array_equal(got[:, :, s].view(np.uint32), ocache.k_mean[:, :, s].view(np.uint32)), s


@pytest.mark.parametrize("smooth,adaptive", OPTIONS)
@pytest.mark.parametrize("key,slots", [("tiny", [0, 1, 2, 3]), ("1.3b", [3]), ("fewstep", [6])])
def test_recipe_quantize_matches_oracle_bit_for_bit(key, slots, smooth, adaptive):
    w = W[key]
    cache, ocache = _caches(w, slots, smooth, adaptive)
    assert cache.quantize_launches() == (3 if smooth else 2)
    assert_cache_equal(cache, ocache, slots)
    if smooth:
        _assert_means_equal(cache, ocache, slots)
    assert cache.read_status() == 0


@pytest.mark.parametrize("name", ["fixed0", "fixed-20", "fixed-100", "ties0", "underflow", "tiny_scale"])
def test_recipe_special_chunks_match_oracle(name):
    chunk = {"fixed0": lambda: sc.fixed_point_chunk(0), "fixed-20": lambda: sc.fixed_point_chunk(-20),
             "fixed-100": lambda: sc.fixed_point_chunk(-100), "ties0": lambda: sc.tie_chunk(0),
             "underflow": sc.underflow_chunk, "tiny_scale": sc.tiny_scale_chunk}[name]()
    chunk = sc.pad_tokens(chunk)
    L = chunk.shape[1]
    neg = chunk ^ np.uint16(0x8000)
    cache = KVCache(1, 1, L, 2, smooth_k=True, adaptive_v=True)
    ocache = oracle.Cache(1, 1, 128, L, 2, smooth_k=True, adaptive_v=True)
    cache.quantize(1, dev_bf16(chunk), dev_bf16(neg))
    ocache.append(1, chunk, neg)
    assert_cache_equal(cache, ocache, [1])
    _assert_means_equal(cache, ocache, [1])
    assert int(cache.k_codes[:, :, :L].abs().sum()) == 0


def test_recipe_token_stride_and_ragged_length():
    import torch
    w = dataclasses.replace(W["tiny"], heads=3, chunk_tokens=200, batch=2, capacity=2)
    k, v = _offset_kv(w, 1)
    qkv = torch.zeros(w.batch, w.chunk_tokens, 3, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    qkv[:, :, 1] = dev_bf16(k)
    qkv[:, :, 2] = dev_bf16(v)
    cache = KVCache(w.batch, w.heads, w.chunk_tokens, 2, smooth_k=True, adaptive_v=True)
    cache.quantize(1, qkv[:, :, 1], qkv[:, :, 2])
    ocache = oracle.Cache(w.batch, w.heads, 128, w.chunk_tokens, 2, smooth_k=True, adaptive_v=True)
    ocache.append(1, k, v)
    assert_cache_equal(cache, ocache, [1])
    _assert_means_equal(cache, ocache, [1])


def _adversarial_keys(B, L, H, seed):
    """Keys whose channels stress an exact sum: eight kinds, by channel mod 8 (uint16 [B, L, H, 128])."""
    rng = np.random.default_rng(seed)
    x = f32_to_bf16_bits((rng.standard_normal((B, L, H, 128)) * 3.0 + 1.0).astype(np.float32))
    sign = lambda n: rng.integers(0, 2, n).astype(np.uint16) << 15
    n = B * L * H
    big = f32_to_bf16_bits(np.float32(2.0 ** 100))
    for c in range(128):
        kind = c % 8
        col = x[:, :, :, c].reshape(-1).copy()
        if kind == 1:    # +-2^100 amid unit values: the large terms cancel
            col[::7] = big
            col[3::7] = big | np.uint16(0x8000)
        elif kind == 2:  # any finite bit pattern
            col = rng.integers(0, 0x7F80, n).astype(np.uint16) | sign(n)
        elif kind == 3:  # subnormal values only
            col = rng.integers(1, 0x80, n).astype(np.uint16) | sign(n)
        elif kind == 4:  # +0 and -0
            col = np.where(rng.integers(0, 2, n) == 1, 0x8000, 0).astype(np.uint16)
        elif kind == 5:  # the largest finite values of both signs
            col = np.uint16(0x7F7F) | sign(n)
        elif kind == 6:  # any bit pattern, Inf and NaN included (summed as the numbers their bits spell)
            col = rng.integers(0, 0x10000, n).astype(np.uint16)
        elif kind == 7:  # unit values with one 2^-39 or 2^-40 value per 64 keys (widest exact span, and one more)
            col[:] = f32_to_bf16_bits(np.float32(1.0))
            col[5::64] = f32_to_bf16_bits(np.float32(2.0 ** -39 if c % 16 == 7 else 2.0 ** -40))
        x[:, :, :, c] = col.reshape(B, L, H)
    return x


@pytest.mark.parametrize("B,H,L", [(2, 3, 130), (2, 3, 1310), (1, 1, 10000)])
def test_recipe_key_mean_is_exact_on_adversarial_channels(B, H, L):
    """The channel means of keys built to defeat a rounded sum (cancellation, subnormals, signed
    zeros, the largest values, any bit pattern) equal the oracle's exact mean rounded once, bit for
    bit.  1310 and 10000 keys end on a ragged 64-key slice and are split over a cluster of CTAs on a
    GPU with enough SMs; 10000 keys on one head also wrap each CTA's 16-stage ring."""
    k = _adversarial_keys(B, L, H, 20 + L)
    v = f32_to_bf16_bits(np.random.default_rng(L).standard_normal((B, L, H, 128)).astype(np.float32))
    cache = KVCache(B, H, L, 2, smooth_k=True)
    cache.quantize(1, dev_bf16(k), dev_bf16(v))
    got = cache.k_mean.cpu().numpy()[:, :, 1]
    want = oracle.key_mean(k)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_recipe_static_scratch_matches_workspace_call():
    import torch
    w = W["1.3b"]
    ref, _ = _caches(w, [], True, True)
    alt = KVCache(w.batch, w.heads, w.chunk_tokens, w.capacity, smooth_k=True, adaptive_v=True)
    k, v = _offset_kv(w, 2)
    kd, vd = dev_bf16(k), dev_bf16(v)
    ref.quantize(2, kd, vd)
    rc = nk.lib().nvfp4_kv_quantize_static_scratch(ctypes.byref(alt.desc), 2, kd.data_ptr(), vd.data_ptr(),
                                                   kd.stride(1), None)
    assert rc == nk.OK
    torch.cuda.synchronize()
    for name in ("k_codes", "v_codes", "k_scales", "v_scales", "k_gscale", "v_gscale", "k_mean"):
        assert torch.equal(getattr(ref, name).view(torch.uint8), getattr(alt, name).view(torch.uint8)), name


def test_recipe_dequantize_adds_the_chunk_mean():
    w = W["tiny"]
    cache, ocache = _caches(w, [0, 1, 2, 3], True, True)
    for which in ("k", "v"):
        got = cache.dequantize(which).cpu().numpy().astype(np.float64)
        want = ocache.dequantize(which)  # fp64, x_hat' + mu for K
        # one fp32 rounding of x_hat' * g, then (K) one of the sum with mu
        tol = 2.0 ** -23 * (np.abs(want) + (np.abs(want - np.repeat(ocache.k_mean, w.chunk_tokens, axis=2))
                                            if which == "k" else 0.0))
        assert np.all(np.abs(got - want) <= tol + 1e-30), which


EDGE = {
    "ragged_two_runs": dict(batch=2, heads=3, chunk_tokens=200, capacity=6, q_chunk=4, n_sink=1, window=2,
                            q_tokens=300),
    "sink_inside_window": dict(batch=1, heads=2, chunk_tokens=136, capacity=5, q_chunk=2, n_sink=2, window=5,
                               q_tokens=129),
    "self_only": dict(batch=1, heads=1, chunk_tokens=130, capacity=3, q_chunk=1, n_sink=0, window=1, q_tokens=1),
    "first_chunk": dict(batch=1, heads=2, chunk_tokens=256, capacity=3, q_chunk=0, n_sink=1, window=3,
                        q_tokens=256),
    "aligned_chunks": dict(batch=1, heads=2, chunk_tokens=128, capacity=6, q_chunk=5, n_sink=1, window=3,
                           q_tokens=200),
}


@pytest.mark.parametrize("name", sorted(EDGE))
def test_smoothed_attention_edge_shapes_all_rows(name):
    w = dataclasses.replace(W["tiny"], key=name, **EDGE[name])
    cache, ocache = _caches(w, w.visible_chunks, True, True)
    qb = synthetic.queries(w)
    out = cache.attention(dev_bf16(qb), w.q_chunk, w.n_sink, w.window)
    assert cache.read_status() == 0
    rows = head_rows(w, [(b, h) for b in range(w.batch) for h in range(w.heads)])
    want = attention_rows_threaded(qb, ocache, w.q_chunk, w.n_sink, w.window, rows)
    assert_attention_close(gather_rows(out.cpu().numpy(), rows), want, name)


@pytest.mark.parametrize("key,layer", [("1.3b", 0), ("rollout", 5)])
def test_smoothed_attention_full_size(key, layer):
    w = W[key]
    cache, ocache = _caches(w, w.visible_chunks, True, True, layer=layer)
    qb = synthetic.queries(w, layer)
    out = cache.attention(dev_bf16(qb), w.q_chunk, w.n_sink, w.window)
    assert cache.read_status() == 0
    rows = np.concatenate([head_rows(w, [(0, w.heads - 1)]), sample_rows(w, 6, seed=4)])
    want = attention_rows_threaded(qb, ocache, w.q_chunk, w.n_sink, w.window, rows)
    assert_attention_close(gather_rows(out.cpu().numpy(), rows), want, key)


def test_smoothing_matters_and_plain_caches_are_unchanged():
    import torch
    w = dataclasses.replace(W["tiny"], key="m", **EDGE["ragged_two_runs"])
    smooth, _ = _caches(w, w.visible_chunks, True, False)
    plain, oplain = _caches(w, w.visible_chunks, False, False)
    q = dev_bf16(synthetic.queries(w))
    a = smooth.attention(q, w.q_chunk, w.n_sink, w.window)
    b = plain.attention(q, w.q_chunk, w.n_sink, w.window)
    assert not torch.equal(a, b)
    # the plain cache still matches the plain oracle
    rows = head_rows(w, [(1, 2)])
    want = attention_rows_threaded(synthetic.queries(w), oplain, w.q_chunk, w.n_sink, w.window, rows)
    assert_attention_close(gather_rows(b.cpu().numpy(), rows), want, "plain")
