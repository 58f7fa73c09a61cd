"""Seeded synthetic inputs shaped like the video-DiT attention workloads.

This module only draws random numbers and rounds them to bf16; it holds none of the
NVFP4 method's arithmetic, and both the CUDA path and the CPU oracle consume exactly the
bytes it returns.  Arrays are numpy uint16 bf16 bit patterns in the [batch, tokens,
heads, head_dim] layout the library takes.

Value recipe (per workload): queries, keys and values are N(0, 1); a few "outlier"
channels per (tensor, layer, head) are multiplied by a gain, the same channels in every
chunk of that layer; optionally every (tensor, layer, head) is multiplied by a
log-normal magnitude.  Every chunk, tensor and layer has its own counter-derived seed,
so any chunk can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    key: str
    name: str
    batch: int
    heads: int
    chunk_tokens: int   # tokens per frame chunk (frames per chunk x tokens per latent frame)
    capacity: int       # chunk slots resident in the cache
    q_chunk: int        # slot of the query chunk
    n_sink: int         # global-sink chunks
    window: int         # window chunks, the query's own chunk included
    q_tokens: int
    layers: int
    seed: int
    kv_outliers: int    # outlier channels per (K or V, head)
    q_outliers: int     # outlier channels per (Q, head)
    gain: float         # outlier channel gain
    head_sigma: float   # sigma of the per-(tensor, head) log-normal magnitude (0: none)
    head_dim: int = 128
    attn_calls: int = 1  # attention calls per quantised chunk (denoising steps)

    @property
    def visible_chunks(self) -> list[int]:
        return [c for c in range(self.capacity)
                if c < self.n_sink or self.q_chunk - self.window < c <= self.q_chunk]

    @property
    def visible_tokens(self) -> int:
        return len(self.visible_chunks) * self.chunk_tokens


WORKLOADS = {
    # 2 heads, 64-token chunks, sink 1 + window 3, 64 queries; 2 outlier channels x20 in K/V
    "tiny": Workload("tiny", "tiny: B1 H2 d128, 4 chunks x 64 tokens, Lq 64", 1, 2, 64, 4, 3, 1, 3,
                     64, 1, seed=0, kv_outliers=2, q_outliers=0, gain=20.0, head_sigma=0.0),
    # 1.3B-class single layer: 1560 tokens/frame, 3-frame chunks, sink 1 + window 3
    "1.3b": Workload("1.3b", "1.3B-class layer: B1 H12 d128, chunk 4680, 4 chunks (18720 keys), Lq 4680",
                     1, 12, 4680, 4, 3, 1, 3, 4680, 1, seed=1, kv_outliers=1, q_outliers=1,
                     gain=16.0, head_sigma=0.0),
    # 5B-class single layer: 880 tokens/frame, 3-frame chunks, sink 1 + window 6
    "5b": Workload("5b", "5B-class layer: B1 H24 d128, chunk 2640, 7 chunks (18480 keys), Lq 2640",
                   1, 24, 2640, 7, 6, 1, 6, 2640, 1, seed=2, kv_outliers=1, q_outliers=1,
                   gain=16.0, head_sigma=0.5),
    # long rollout: 30 layers, 40 chunks resident (120 latent frames), sink 1 + window 7
    "rollout": Workload("rollout", "long rollout step t=39: 30 layers x H12 d128, chunk 4680, "
                        "40 chunks resident, sink 1 + window 7 (37440 keys), Lq 4680",
                        1, 12, 4680, 40, 39, 1, 7, 4680, 30, seed=3, kv_outliers=1, q_outliers=1,
                        gain=16.0, head_sigma=0.0),
    # real-time few-step decode: 1-frame query chunk, 4 then 2 denoising calls per chunk
    "fewstep": Workload("fewstep", "few-step decode: B1 H24 d128, Lq 880 (1 frame), chunk 2640, "
                        "7 chunks (18480 keys), 4+2 attention calls per chunk",
                        1, 24, 2640, 7, 6, 1, 6, 880, 1, seed=4, kv_outliers=1, q_outliers=1,
                        gain=16.0, head_sigma=0.0, attn_calls=6),
}

_TENSOR_ID = {"q": 0, "k": 1, "v": 2}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round to bf16 (nearest, ties to even) and return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _channel_gains(w: Workload, tensor: str, layer: int) -> np.ndarray:
    """[heads, head_dim] multiplier: outlier channels and the per-head magnitude."""
    tid = _TENSOR_ID[tensor]
    rng = _rng(w.seed, layer, 1_000_000 + tid)
    n_out = w.q_outliers if tensor == "q" else w.kv_outliers
    gains = np.ones((w.heads, w.head_dim), np.float64)
    for h in range(w.heads):
        if n_out:
            ch = rng.choice(w.head_dim, size=n_out, replace=False)
            gains[h, ch] = w.gain
    if w.head_sigma > 0:
        mag = rng.lognormal(0.0, w.head_sigma, size=w.heads)
        gains *= mag[:, None]
    return gains


def _draw(w: Workload, tensor: str, layer: int, slot: int, tokens: int) -> np.ndarray:
    rng = _rng(w.seed, layer, slot, _TENSOR_ID[tensor])
    x = rng.standard_normal((w.batch, tokens, w.heads, w.head_dim))
    x *= _channel_gains(w, tensor, layer)[None, None]
    return f32_to_bf16_bits(x.astype(np.float32))


def with_layers(w: Workload, layers: int) -> Workload:
    """The same workload with ``layers`` layers (each layer's shapes and inputs unchanged)."""
    if layers < 1:
        raise ValueError("layers must be positive")
    name = w.name.replace(f"{w.layers} layers", f"{layers} layer{'s' if layers > 1 else ''}")
    return dataclasses.replace(w, name=name, layers=layers)


def chunk_kv(w: Workload, slot: int, layer: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """bf16 K and V of chunk slot ``slot`` of layer ``layer``: two uint16 [B, Lc, H, d]."""
    return (_draw(w, "k", layer, slot, w.chunk_tokens), _draw(w, "v", layer, slot, w.chunk_tokens))


def queries(w: Workload, layer: int = 0, step: int = 0) -> np.ndarray:
    """bf16 queries of the query chunk (uint16 [B, Lq, H, d]); ``step`` picks a denoising step."""
    return _draw(w, "q", layer, 10_000 + step, w.q_tokens)


# ---- the same recipe drawn on the GPU (torch's counter-based generator), for inputs too large to
# draw on the host in reasonable time (the benchmark's 30-layer rollout).  Not the same bytes as
# the numpy draws above; the parity tests use those.
def _device_seed(*key: int) -> int:
    return int(np.random.SeedSequence(list(key)).generate_state(1, dtype=np.uint64)[0] >> 1)


def _device_draw(w: Workload, tensor: str, layer: int, slot: int, tokens: int, device):
    import torch
    g = torch.Generator(device=device).manual_seed(_device_seed(w.seed, layer, slot, _TENSOR_ID[tensor], 77))
    x = torch.randn((w.batch, tokens, w.heads, w.head_dim), generator=g, device=device, dtype=torch.float32)
    gains = torch.from_numpy(_channel_gains(w, tensor, layer).astype(np.float32)).to(device)
    return (x * gains).to(torch.bfloat16)


def device_chunk_kv(w: Workload, slot: int, layer: int = 0, device="cuda"):
    """bf16 CUDA tensors K, V [B, Lc, H, d] of chunk ``slot`` of layer ``layer``."""
    return (_device_draw(w, "k", layer, slot, w.chunk_tokens, device),
            _device_draw(w, "v", layer, slot, w.chunk_tokens, device))


def device_queries(w: Workload, layer: int = 0, step: int = 0, device="cuda"):
    """bf16 CUDA tensor of the query chunk [B, Lq, H, d]."""
    return _device_draw(w, "q", layer, 10_000 + step, w.q_tokens, device)
