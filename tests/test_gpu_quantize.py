"""GPU parity of the quantiser and of the dequantisation step: codes, E4M3 scales and FP32
scales bit-identical to the oracle on the same seeded inputs; dequantised values equal to
the oracle's exact fp64 values rounded once to fp32."""
import dataclasses

import numpy as np
import pytest

import oracle
from nvfp4_quantised_kv_b200 import KVCache, debug_encode, quantize_layers, synthetic
from tests import special_chunks as sc
from tests.gpu_util import assert_cache_equal, dev_bf16, make_caches

pytestmark = pytest.mark.gpu


def _sweep_values():
    """Every finite bf16 value, dense neighbourhoods of every E2M1 / E4M3 rounding boundary
    (+-512 ulps), and random finite fp32 bit patterns."""
    rng = np.random.default_rng(123)
    bf = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    vals = [bf[np.isfinite(bf)]]
    e2 = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0]
    e4 = sorted(set(sc.e4m3_positive_values()))
    e4_mid = [(a + b) / 2 for a, b in zip([0.0] + e4[:-1], e4)] + [448.0, 464.0]
    centers = np.array(e2 + e4_mid, np.float32)
    off = np.arange(-512, 513, dtype=np.int64)
    for c in centers:
        u = np.int64(np.float32(c).view(np.uint32)) + off
        u = u[(u > 0) & (u < 0x7F800000)].astype(np.uint32)
        v = u.view(np.float32)
        vals += [v, -v]
    r = rng.integers(0, 2 ** 32, size=1 << 22, dtype=np.uint64).astype(np.uint32).view(np.float32)
    vals.append(r[np.isfinite(r)])
    return np.concatenate(vals)


def test_device_conversions_match_the_format_definition():
    import torch
    x = _sweep_values()
    e2, e4 = debug_encode(torch.from_numpy(x).cuda())
    e2, e4 = e2.cpu().numpy(), e4.cpu().numpy()
    want2 = oracle.e2m1_encode_array(x)
    want4 = oracle.e4m3_encode_array(x)
    bad2 = np.nonzero(e2 != want2)[0]
    bad4 = np.nonzero(e4 != want4)[0]
    assert bad2.size == 0, (x[bad2[:8]], e2[bad2[:8]], want2[bad2[:8]])
    assert bad4.size == 0, (x[bad4[:8]], e4[bad4[:8]], want4[bad4[:8]])


@pytest.mark.parametrize("key,slots", [("tiny", [0, 1, 2, 3]), ("1.3b", [0, 3]), ("5b", [1, 6]),
                                       ("fewstep", [6]), ("rollout", [39])])
def test_quantize_matches_oracle_bit_for_bit(key, slots):
    w = synthetic.WORKLOADS[key]
    cache, ocache = make_caches(w, slots)
    assert_cache_equal(cache, ocache, slots)
    assert cache.read_status() == 0


# Chunks of up to 16 x 448 tokens per (b, h) are quantised by one thread-block cluster in a single
# pass; longer ones by the two-pass kernels.  Every special chunk runs through both.
TWO_PASS_TOKENS = 7200


@pytest.mark.parametrize("path", ["cluster", "two_pass", "layers"])
@pytest.mark.parametrize("name", ["fixed0", "fixed-20", "fixed17", "fixed-100", "ties0", "ties-9",
                                  "underflow", "tiny_scale"])
def test_special_chunks_match_oracle(name, path):
    chunk = {"fixed0": lambda: sc.fixed_point_chunk(0), "fixed-20": lambda: sc.fixed_point_chunk(-20),
             "fixed17": lambda: sc.fixed_point_chunk(17), "fixed-100": lambda: sc.fixed_point_chunk(-100),
             "ties0": lambda: sc.tie_chunk(0), "ties-9": lambda: sc.tie_chunk(-9),
             "underflow": sc.underflow_chunk, "tiny_scale": sc.tiny_scale_chunk}[name]()
    chunk = sc.pad_tokens(chunk)
    if path == "two_pass":  # long enough that no cluster holds a (b, h, tensor) in shared memory
        reps = -(-TWO_PASS_TOKENS // chunk.shape[1])
        chunk = np.ascontiguousarray(np.tile(chunk, (1, reps, 1, 1)))
    L = chunk.shape[1]
    cache = KVCache(1, 1, L, 2)
    ocache = oracle.Cache(1, 1, 128, L, 2)
    neg = chunk ^ np.uint16(0x8000)  # V gets the negated chunk
    if path == "layers":  # the single-launch multi-layer path, as the second of two layers
        other = KVCache(1, 1, L, 2)
        quantize_layers([other, cache], 1, [dev_bf16(neg), dev_bf16(chunk)], [dev_bf16(chunk), dev_bf16(neg)])
    else:
        assert cache.quantize_launches() == (1 if path == "cluster" else 2)
        cache.quantize(1, dev_bf16(chunk), dev_bf16(neg))
    ocache.append(1, chunk, neg)
    assert_cache_equal(cache, ocache, [1])
    # the slot not written stays untouched
    assert int(cache.k_codes[:, :, :L].abs().sum()) == 0


def test_long_chunk_two_pass_path_matches_oracle():
    w = dataclasses.replace(synthetic.WORKLOADS["tiny"], heads=2, chunk_tokens=TWO_PASS_TOKENS + 8, capacity=2)
    cache, ocache = make_caches(w, [1])
    assert cache.quantize_launches() == 2
    assert_cache_equal(cache, ocache, [1])
    assert cache.read_status() == 0


def test_token_stride_fused_qkv_layout():
    import torch
    w = dataclasses.replace(synthetic.WORKLOADS["tiny"], heads=3, chunk_tokens=96, batch=2)
    k, v = synthetic.chunk_kv(w, 0)
    qkv = torch.zeros(w.batch, w.chunk_tokens, 3, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    qkv[:, :, 1] = dev_bf16(k)
    qkv[:, :, 2] = dev_bf16(v)
    cache = KVCache(w.batch, w.heads, w.chunk_tokens, 2)
    cache.quantize(1, qkv[:, :, 1], qkv[:, :, 2])
    ocache = oracle.Cache(w.batch, w.heads, 128, w.chunk_tokens, 2)
    ocache.append(1, k, v)
    assert_cache_equal(cache, ocache, [1])


def test_dequantize_matches_oracle_exact_values():
    w = synthetic.WORKLOADS["tiny"]
    cache, ocache = make_caches(w, [0, 1, 2, 3])
    for which in ("k", "v"):
        got = cache.dequantize(which).cpu().numpy()
        want = ocache.dequantize(which).astype(np.float32)
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), which
    got = cache.dequantize("v", first_slot=2, n_slots=2).cpu().numpy()
    want = ocache.dequantize("v")[:, :, 2 * w.chunk_tokens:].astype(np.float32)
    assert np.array_equal(got, want)


def test_quantize_is_deterministic():
    w = synthetic.WORKLOADS["5b"]
    cache, _ = make_caches(w, [])
    k, v = synthetic.chunk_kv(w, 2)
    kd, vd = dev_bf16(k), dev_bf16(v)
    cache.quantize(2, kd, vd)
    first = [t.clone() for t in (cache.k_codes, cache.v_scales, cache.k_gscale)]
    cache.quantize(2, kd, vd)
    for a, b in zip(first, (cache.k_codes, cache.v_scales, cache.k_gscale)):
        assert bool((a == b).all())


@pytest.mark.parametrize("batch,heads,chunk_tokens,layers", [(1, 2, 64, 3), (2, 3, 300, 2), (1, 1, 2, 5)])
def test_quantize_layers_matches_oracle_bit_for_bit(batch, heads, chunk_tokens, layers):
    # one launch for every layer's new chunk (ragged last parts, many slices, 2-token chunks)
    w = dataclasses.replace(synthetic.WORKLOADS["tiny"], batch=batch, heads=heads, chunk_tokens=chunk_tokens,
                            capacity=3)
    caches = [KVCache(batch, heads, chunk_tokens, 3) for _ in range(layers)]
    kv = [synthetic.chunk_kv(w, 2, layer) for layer in range(layers)]
    quantize_layers(caches, 2, [dev_bf16(k) for k, _ in kv], [dev_bf16(v) for _, v in kv])
    for layer in range(layers):
        ocache = oracle.Cache(batch, heads, 128, chunk_tokens, 3)
        ocache.append(2, *kv[layer])
        assert_cache_equal(caches[layer], ocache, [2])
        assert int(caches[layer].k_codes[:, :, :2 * chunk_tokens].abs().sum()) == 0  # other slots untouched
    assert caches[0].read_status() == 0


def test_quantize_layers_full_size_equals_per_layer_calls():
    # four 1.3B-class layers in one launch; layer 0 against the oracle, all against the per-layer call
    w = synthetic.WORKLOADS["1.3b"]
    layers = 4
    caches = [KVCache(w.batch, w.heads, w.chunk_tokens, w.capacity) for _ in range(layers)]
    refs = [KVCache(w.batch, w.heads, w.chunk_tokens, w.capacity) for _ in range(layers)]
    kv = [tuple(dev_bf16(x) for x in synthetic.chunk_kv(w, 3, layer)) for layer in range(layers)]
    ws = quantize_layers(caches, 3, [k for k, _ in kv], [v for _, v in kv])
    quantize_layers(caches, 3, [k for k, _ in kv], [v for _, v in kv], workspace=ws)  # reused scratch
    for c, r, (k, v) in zip(caches, refs, kv):
        r.quantize(3, k, v)
        for name in ("k_codes", "v_codes", "k_scales", "v_scales", "k_gscale", "v_gscale"):
            assert bool((getattr(c, name) == getattr(r, name)).all()), name
    ocache = oracle.Cache(w.batch, w.heads, 128, w.chunk_tokens, w.capacity)
    ocache.append(3, *synthetic.chunk_kv(w, 3, 0))
    assert_cache_equal(caches[0], ocache, [3])
    assert caches[0].read_status() == 0


def test_quantize_layers_at_the_rollout_step_size():
    # the benchmark's launch: every one of 30 layers' new 4680-token chunk (12 heads) into slot 39 of
    # 40-slot caches in one launch; three layers against the oracle, every layer against the
    # per-layer call
    import torch
    w = synthetic.WORKLOADS["rollout"]
    caches = [KVCache(w.batch, w.heads, w.chunk_tokens, w.capacity) for _ in range(w.layers)]
    ks, vs = [], []
    for layer in range(w.layers):
        k, v = synthetic.device_chunk_kv(w, w.q_chunk, layer)
        ks.append(k)
        vs.append(v)
    quantize_layers(caches, w.q_chunk, ks, vs)
    assert caches[0].read_status() == 0
    ref = KVCache(w.batch, w.heads, w.chunk_tokens, w.capacity)
    t0 = w.q_chunk * w.chunk_tokens
    for layer in range(w.layers):
        ref.quantize(w.q_chunk, ks[layer], vs[layer])
        for name in ("k_codes", "v_codes", "k_scales", "v_scales"):
            assert torch.equal(getattr(caches[layer], name)[:, :, t0:], getattr(ref, name)[:, :, t0:]), (layer, name)
        for name in ("k_gscale", "v_gscale"):
            assert torch.equal(getattr(caches[layer], name)[:, :, w.q_chunk].view(torch.int32),
                               getattr(ref, name)[:, :, w.q_chunk].view(torch.int32)), (layer, name)
    for layer in (0, 17, 29):
        kb = ks[layer].view(torch.int16).cpu().numpy().view(np.uint16)
        vb = vs[layer].view(torch.int16).cpu().numpy().view(np.uint16)
        ocache = oracle.Cache(w.batch, w.heads, 128, w.chunk_tokens, w.capacity)
        ocache.append(w.q_chunk, kb, vb)
        assert_cache_equal(caches[layer], ocache, [w.q_chunk])
