"""Helpers for the GPU parity tests: move synthetic bytes to the device, build matching
CUDA and oracle caches, and compare results."""
import numpy as np

import oracle
from nvfp4_quantised_kv_b200 import KVCache, synthetic

# attention tolerance against the fp64 oracle over the same dequantised cache
MAX_ABS = 1e-2
REL_FRO = 5e-3


def dev_bf16(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def make_caches(w, slots, layer: int = 0):
    """CUDA cache and oracle cache holding the same synthetic chunks in ``slots``."""
    cache = KVCache(w.batch, w.heads, w.chunk_tokens, w.capacity, q_tokens_max=w.q_tokens)
    ocache = oracle.Cache(w.batch, w.heads, w.head_dim, w.chunk_tokens, w.capacity)
    for slot in slots:
        k, v = synthetic.chunk_kv(w, slot, layer)
        cache.quantize(slot, dev_bf16(k), dev_bf16(v))
        ocache.append(slot, k, v)
    return cache, ocache


def assert_cache_equal(cache, ocache, slots):
    """Codes, E4M3 scales and FP32 scales of ``slots`` are identical, bit for bit."""
    Lc = ocache.Lc
    for name in ("k_codes", "v_codes", "k_scales", "v_scales"):
        got = getattr(cache, name).cpu().numpy()
        want = getattr(ocache, name)
        for s in slots:
            a, b = got[:, :, s * Lc:(s + 1) * Lc], want[:, :, s * Lc:(s + 1) * Lc]
            bad = np.argwhere(a != b)
            assert bad.size == 0, f"{name} slot {s}: {len(bad)} bytes differ, first at {bad[:3].tolist()}"
    for name, oname in (("k_gscale", "k_g"), ("v_gscale", "v_g")):
        got = getattr(cache, name).cpu().numpy()
        want = getattr(ocache, oname)
        for s in slots:
            assert np.array_equal(got[:, :, s].view(np.uint32), want[:, :, s].view(np.uint32)), name


def sample_rows(w, per_head: int, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    rows = []
    fixed = sorted({0, min(127, w.q_tokens - 1), min(128, w.q_tokens - 1), w.q_tokens - 1})
    for b in range(w.batch):
        for h in range(w.heads):
            extra = rng.choice(w.q_tokens, size=max(0, per_head - len(fixed)), replace=False)
            for i in sorted(set(fixed) | set(int(e) for e in extra)):
                rows.append((b, h, i))
    return np.array(rows, np.int32)


def errors(got: np.ndarray, want: np.ndarray):
    d = got.astype(np.float64) - want
    return float(np.max(np.abs(d))), float(np.linalg.norm(d) / max(np.linalg.norm(want), 1e-300))


def assert_attention_close(got_rows: np.ndarray, want_rows: np.ndarray, what: str = ""):
    max_abs, rel = errors(got_rows, want_rows)
    assert np.all(np.isfinite(got_rows)), what
    assert max_abs <= MAX_ABS and rel <= REL_FRO, f"{what}: max_abs {max_abs:.3e} rel_fro {rel:.3e}"
    return max_abs, rel


def gather_rows(out: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """out is [B, Lq, H, d]; rows are (b, h, i) triples."""
    return np.stack([out[b, i, h] for b, h, i in rows])


def attention_rows_threaded(qb, ocache, q_chunk, n_sink, window, rows, softmax_scale=0.0,
                            threads=None):
    """The oracle's attention of ``rows``, with the rows split over host threads.

    Each thread calls the single-threaded oracle on its own share of the rows (the oracle keeps
    no state between calls and ctypes releases the interpreter lock), so the result is the same
    array the one-call form returns, only sooner.
    """
    import os
    from concurrent.futures import ThreadPoolExecutor
    threads = threads or max(1, min(32, os.cpu_count() or 1))
    parts = [p for p in np.array_split(rows, threads) if len(p)]
    with ThreadPoolExecutor(len(parts)) as ex:
        outs = list(ex.map(lambda p: oracle.attention_rows(qb, ocache, q_chunk, n_sink, window, p,
                                                            softmax_scale), parts))
    return np.concatenate(outs)


def head_rows(w, bh_list) -> np.ndarray:
    """Every query row (b, h, i) of the listed (b, h) pairs."""
    return np.array([(b, h, i) for b, h in bh_list for i in range(w.q_tokens)], np.int32)


def kv_tiles(chunk_tokens: int, slots) -> int:
    """128-key tiles of the visible chunks, which are merged into runs of consecutive slots; a
    tile never crosses a run boundary."""
    slots = sorted(set(slots))
    tiles, i = 0, 0
    while i < len(slots):
        k = i
        while k + 1 < len(slots) and slots[k + 1] == slots[k] + 1:
            k += 1
        tiles += -(-(k - i + 1) * chunk_tokens // 128)
        i = k + 1
    return tiles
