"""GPU parity of the NVFP4 KV attention against the fp64 oracle over the same dequantised
cache: max-abs <= 1e-2 and relative Frobenius <= 5e-3, on the five workloads (sampled rows
at full size) and on small edge cases compared row for row; masked chunks have no effect."""
import dataclasses

import numpy as np
import pytest

import oracle
from nvfp4_quantised_kv_b200 import synthetic
from tests.gpu_util import (assert_attention_close, dev_bf16, gather_rows, make_caches,
                            sample_rows)

pytestmark = pytest.mark.gpu

W = synthetic.WORKLOADS


def _run(w, slots=None, rows=None, softmax_scale=0.0, out_dtype=None, layer=0, step=0):
    slots = w.visible_chunks if slots is None else slots
    cache, ocache = make_caches(w, slots, layer)
    qb = synthetic.queries(w, layer, step)
    out = cache.attention(dev_bf16(qb), w.q_chunk, w.n_sink, w.window, softmax_scale,
                          out_dtype=out_dtype)
    assert cache.read_status() == 0
    if rows is None:
        rows = np.array([(b, h, i) for b in range(w.batch) for h in range(w.heads)
                         for i in range(w.q_tokens)], np.int32)
    want = oracle.attention_rows(qb, ocache, w.q_chunk, w.n_sink, w.window, rows, softmax_scale)
    got = gather_rows(out.float().cpu().numpy(), rows)
    return got, want, cache, ocache, out, qb


def test_tiny_workload_all_rows():
    got, want, *_ = _run(W["tiny"])
    assert_attention_close(got, want, "tiny")


EDGE = {
    # two runs (sink, then a window), ragged last tiles, a chunk boundary inside a tile, B=2
    "ragged_two_runs": dict(batch=2, heads=3, chunk_tokens=200, capacity=6, q_chunk=4, n_sink=1,
                            window=2, q_tokens=300),
    # 2-token chunks: every KV tile spans many chunks with different FP32 scales
    "many_chunks_per_tile": dict(batch=1, heads=2, chunk_tokens=2, capacity=100, q_chunk=99,
                                 n_sink=3, window=60, q_tokens=130),
    # sink overlaps the window: chunks counted once
    "sink_inside_window": dict(batch=1, heads=2, chunk_tokens=136, capacity=5, q_chunk=2, n_sink=2,
                               window=5, q_tokens=129),
    # no sink, window of one chunk: the query chunk attends to itself only
    "self_only": dict(batch=1, heads=1, chunk_tokens=130, capacity=3, q_chunk=1, n_sink=0, window=1,
                      q_tokens=1),
    # query chunk at slot 0
    "first_chunk": dict(batch=1, heads=2, chunk_tokens=256, capacity=3, q_chunk=0, n_sink=1, window=3,
                        q_tokens=256),
    # 148 heads of two query tiles (128 + 72 rows): one two-tile CTA per head on a 148-SM B200,
    # so the ragged tile sits in the second softmax warpgroup
    "ragged_pairs": dict(batch=1, heads=148, chunk_tokens=64, capacity=3, q_chunk=2, n_sink=1, window=2,
                         q_tokens=200),
}


@pytest.mark.parametrize("name", sorted(EDGE))
def test_edge_shapes_all_rows(name):
    w = dataclasses.replace(W["tiny"], key=name, **EDGE[name])
    got, want, *_ = _run(w)
    assert_attention_close(got, want, name)


@pytest.mark.parametrize("key,per_head", [("1.3b", 12), ("5b", 8), ("fewstep", 8)])
def test_full_size_workloads_sampled_rows(key, per_head):
    w = W[key]
    rows = sample_rows(w, per_head, seed=w.seed)
    got, want, *_ = _run(w, rows=rows)
    assert_attention_close(got, want, key)


def test_rollout_step_one_layer_sampled_rows():
    # 40 resident chunks; only the 8 visible ones hold data, the rest stay zero
    w = W["rollout"]
    rows = sample_rows(w, 8, seed=3)
    got, want, *_ = _run(w, rows=rows, layer=17)
    assert_attention_close(got, want, "rollout")


def test_masked_chunks_have_no_effect_on_the_output():
    import torch
    w = dataclasses.replace(W["tiny"], **EDGE["ragged_two_runs"])
    _, _, cache, ocache, out, qb = _run(w, slots=list(range(w.capacity)))
    hidden = [c for c in range(w.capacity) if c not in w.visible_chunks]
    assert hidden
    g = torch.Generator(device="cuda").manual_seed(5)
    for c in hidden:
        t0, t1 = c * w.chunk_tokens, (c + 1) * w.chunk_tokens
        for t in (cache.k_codes, cache.v_codes, cache.k_scales, cache.v_scales):
            t[:, :, t0:t1] = torch.randint(0, 256, t[:, :, t0:t1].shape, generator=g, device="cuda",
                                           dtype=torch.uint8)
        cache.k_gscale[:, :, c] = float("nan")
        cache.v_gscale[:, :, c] = float("inf")
    again = cache.attention(dev_bf16(qb), w.q_chunk, w.n_sink, w.window)
    assert torch.equal(out.view(torch.int32), again.view(torch.int32))


def test_output_is_deterministic_and_bf16_output_is_rounded_fp32():
    import torch
    w = dataclasses.replace(W["tiny"], **EDGE["ragged_two_runs"])
    _, _, cache, _, out, qb = _run(w)
    q = dev_bf16(qb)
    again = cache.attention(q, w.q_chunk, w.n_sink, w.window)
    assert torch.equal(out.view(torch.int32), again.view(torch.int32))
    ob = cache.attention(q, w.q_chunk, w.n_sink, w.window, out_dtype=torch.bfloat16)
    assert torch.equal(ob.view(torch.int16), out.to(torch.bfloat16).view(torch.int16))


def test_output_guard_rows_stay_untouched():
    # the output lives between two guard batches filled with a canary pattern
    import torch
    w = dataclasses.replace(W["tiny"], **EDGE["ragged_two_runs"])
    cache, _ = make_caches(w, w.visible_chunks)
    q = dev_bf16(synthetic.queries(w))
    big = torch.empty(w.batch + 2, w.q_tokens, w.heads, 128, dtype=torch.float32, device="cuda")
    big.view(torch.int32).fill_(0x7FC0DEAD)
    out = big[1:w.batch + 1]
    cache.attention(q, w.q_chunk, w.n_sink, w.window, out=out)
    assert cache.read_status() == 0
    guard = torch.cat([big[0], big[w.batch + 1]]).view(torch.int32)
    assert bool((guard == 0x7FC0DEAD).all())
    assert bool(torch.isfinite(out).all())


def test_query_token_stride_and_softmax_scale():
    import torch
    w = dataclasses.replace(W["tiny"], batch=2, heads=3)
    cache, ocache = make_caches(w, w.visible_chunks)
    qb = synthetic.queries(w)
    qkv = torch.zeros(w.batch, w.q_tokens, 3, w.heads, 128, dtype=torch.bfloat16, device="cuda")
    qkv[:, :, 0] = dev_bf16(qb)
    for scale in (0.0, 0.05):
        out = cache.attention(qkv[:, :, 0], w.q_chunk, w.n_sink, w.window, softmax_scale=scale)
        rows = np.array([(b, h, i) for b in range(w.batch) for h in range(w.heads)
                         for i in range(w.q_tokens)], np.int32)
        want = oracle.attention_rows(qb, ocache, w.q_chunk, w.n_sink, w.window, rows, scale)
        assert_attention_close(gather_rows(out.cpu().numpy(), rows), want, f"scale {scale}")


def test_queries_beyond_fp16_range_use_an_exact_power_of_two_prescale():
    # |q| up to ~2^22 (beyond fp16) with K scaled down by the same factor: logits stay moderate
    from tests._bf16 import bf16_bits_to_f32, f32_to_bf16_bits
    w = dataclasses.replace(W["tiny"], **EDGE["ragged_two_runs"])
    cache, ocache = make_caches(w, [])
    for slot in w.visible_chunks:
        k, v = synthetic.chunk_kv(w, slot)
        k = f32_to_bf16_bits(bf16_bits_to_f32(k) * np.float32(2.0 ** -20))
        cache.quantize(slot, dev_bf16(k), dev_bf16(v))
        ocache.append(slot, k, v)
    qb = f32_to_bf16_bits(bf16_bits_to_f32(synthetic.queries(w)) * np.float32(2.0 ** 20))
    out = cache.attention(dev_bf16(qb), w.q_chunk, w.n_sink, w.window)
    assert cache.read_status() == 0
    rows = np.array([(b, h, i) for b in range(w.batch) for h in range(w.heads)
                     for i in range(w.q_tokens)], np.int32)
    want = oracle.attention_rows(qb, ocache, w.q_chunk, w.n_sink, w.window, rows)
    assert_attention_close(gather_rows(out.cpu().numpy(), rows), want, "large q")


# ---- multi-shot attention sink (paper page, section 4.2; reading note, "Multi-shot attention
# sinks"): global sink U the current shot's sink U window, through the slot-list entry point.
MS = dataclasses.replace(W["tiny"], key="multishot", batch=1, heads=2, chunk_tokens=64, capacity=12,
                         q_chunk=9, n_sink=1, window=2, q_tokens=100)


def _ms_case(slots_listed, layer=0):
    w = MS
    vis = sorted(set(slots_listed))
    cache, ocache = make_caches(w, vis, layer)
    qb = synthetic.queries(w, layer)
    out = cache.attention_slots(dev_bf16(qb), slots_listed)
    assert cache.read_status() == 0
    rows = np.array([(b, h, i) for b in range(w.batch) for h in range(w.heads)
                     for i in range(w.q_tokens)], np.int32)
    want = oracle.attention_rows_slots(qb, ocache, slots_listed, rows)
    return gather_rows(out.float().cpu().numpy(), rows), want, cache, qb


def test_multishot_sink_three_runs_all_rows():
    # global sink {0}, shot sink (start 4, length 2), window {8, 9}: runs [0], [4, 5], [8, 9]
    slots = oracle.multishot_chunks(9, 1, 2, 4, 2, MS.capacity)
    assert slots == [0, 4, 5, 8, 9]
    got, want, *_ = _ms_case(slots)
    assert_attention_close(got, want, "multishot 3 runs")


def test_slot_list_four_runs_out_of_order_with_repeats():
    got, want, *_ = _ms_case([9, 0, 3, 6, 7, 3, 9, 0])
    assert_attention_close(got, want, "slot list 4 runs")


def test_multishot_binding_matches_the_oracle_set():
    import torch
    _, _, cache, qb = _ms_case(oracle.multishot_chunks(9, 1, 2, 4, 2, MS.capacity))
    a = cache.attention_multishot(dev_bf16(qb), 9, 1, 2, 4, 2)
    b = cache.attention_slots(dev_bf16(qb), [0, 4, 5, 8, 9])
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_window_slot_list_equals_the_window_call_bit_for_bit():
    import torch
    w = dataclasses.replace(W["tiny"], **EDGE["ragged_two_runs"])
    cache, _ = make_caches(w, w.visible_chunks)
    q = dev_bf16(synthetic.queries(w))
    a = cache.attention(q, w.q_chunk, w.n_sink, w.window)
    b = cache.attention_slots(q, list(reversed(w.visible_chunks)))
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))
