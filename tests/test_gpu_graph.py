"""The hot path captured in a CUDA graph (the benchmark's graph-replay record): a step of the
multi-layer quantiser and the attention calls, replayed, writes the same bytes as the same calls
made one by one on a stream."""
import dataclasses

import pytest

import nvfp4_quantised_kv_b200 as nk
from nvfp4_quantised_kv_b200 import synthetic
from tests.gpu_util import dev_bf16

pytestmark = pytest.mark.gpu


def _state(w, layers, seed_shift):
    import torch
    caches, ks, vs, qs, outs = [], [], [], [], []
    for layer in range(layers):
        ws = dataclasses.replace(w, seed=w.seed + seed_shift)
        c = nk.KVCache(w.batch, w.heads, w.chunk_tokens, w.capacity, q_tokens_max=w.q_tokens)
        for slot in w.visible_chunks:
            if slot != w.q_chunk:
                k, v = synthetic.chunk_kv(ws, slot, layer)
                c.quantize(slot, dev_bf16(k), dev_bf16(v))
        k, v = synthetic.chunk_kv(ws, w.q_chunk, layer)
        caches.append(c)
        ks.append(dev_bf16(k))
        vs.append(dev_bf16(v))
        qs.append(dev_bf16(synthetic.queries(ws, layer)))
        outs.append(torch.empty(w.batch, w.q_tokens, w.heads, 128, dtype=torch.float32, device="cuda"))
    return caches, ks, vs, qs, outs


def _step(w, caches, ks, vs, qs, outs, qws):
    nk.quantize_layers(caches, w.q_chunk, ks, vs, workspace=qws)
    for c, q, o in zip(caches, qs, outs):
        c.attention(q, w.q_chunk, w.n_sink, w.window, out=o)


def test_graph_replay_matches_stream_calls():
    import torch
    # three layers of a shape whose attention splits work items between CTAs (combine kernel
    # on the path): 2 heads x 3 query tiles over 12 KV tiles
    w = dataclasses.replace(synthetic.WORKLOADS["tiny"], key="graph", batch=1, heads=2, chunk_tokens=400,
                            capacity=5, q_chunk=4, n_sink=1, window=3, q_tokens=300)
    eager = _state(w, 3, 0)
    qws = nk.quantize_layers(eager[0], w.q_chunk, eager[1], eager[2])  # workspace
    _step(w, *eager, qws)
    torch.cuda.synchronize()

    graph = _state(w, 3, 0)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        _step(w, *graph, qws)  # warm-up outside the capture
    torch.cuda.synchronize()
    for c in graph[0]:  # the warm-up already wrote the new slot: clear it so the replay rewrites it
        t0 = w.q_chunk * w.chunk_tokens
        for t in (c.k_codes, c.v_codes, c.k_scales, c.v_scales):
            t[:, :, t0:].zero_()
        c.k_gscale[:, :, w.q_chunk] = 0
        c.v_gscale[:, :, w.q_chunk] = 0
    for o in graph[4]:
        o.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side, capture_error_mode="thread_local"):
        _step(w, *graph, qws)
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(eager[0], graph[0]):
        for name in ("k_codes", "v_codes", "k_scales", "v_scales", "k_gscale", "v_gscale"):
            assert torch.equal(getattr(a, name).view(torch.uint8), getattr(b, name).view(torch.uint8)), name
        assert a.read_status() == 0 and b.read_status() == 0
    for a, b in zip(eager[4], graph[4]):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    del g
