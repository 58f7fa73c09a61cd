"""ctypes front end of the CPU oracle (TEST INFRASTRUCTURE ONLY).

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may import
this package.  It is an independent, slow, single-threaded restatement of the NVFP4
KV-cache path; see ``nvfp4kv_oracle.cpp`` for what each function computes and which
page passage it follows.  Arrays are numpy arrays; bf16 data travels as uint16 bit
patterns.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_decode.restype = ctypes.c_double
        L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        for name in ("oracle_e2m1_encode_array", "oracle_e4m3_encode_array"):
            fn = getattr(L, name)
            fn.restype = None
            fn.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        L.oracle_quantize_chunk.restype = ctypes.c_int
        L.oracle_quantize_chunk.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                            ctypes.c_int32, ctypes.c_int32, ctypes.c_int64,
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_dequantize.restype = ctypes.c_int
        L.oracle_dequantize.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                        ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p]
        L.oracle_visible_chunks.restype = ctypes.c_int
        L.oracle_visible_chunks.argtypes = [ctypes.c_int32] * 4 + [ctypes.c_void_p]
        L.oracle_attention_rows.restype = ctypes.c_int
        L.oracle_attention_rows.argtypes = (
            [ctypes.c_void_p] + [ctypes.c_int32] * 4 + [ctypes.c_int64] + [ctypes.c_void_p] * 6 +
            [ctypes.c_int32] * 5 + [ctypes.c_double, ctypes.c_void_p, ctypes.c_int32,
                                    ctypes.c_void_p])
        L.oracle_multishot_chunks.restype = ctypes.c_int
        L.oracle_multishot_chunks.argtypes = [ctypes.c_int32] * 6 + [ctypes.c_void_p]
        L.oracle_attention_rows_slots.restype = ctypes.c_int
        L.oracle_attention_rows_slots.argtypes = (
            [ctypes.c_void_p] + [ctypes.c_int32] * 4 + [ctypes.c_int64] + [ctypes.c_void_p] * 6 +
            [ctypes.c_int32] * 2 + [ctypes.c_void_p, ctypes.c_int32, ctypes.c_double, ctypes.c_void_p,
                                    ctypes.c_int32, ctypes.c_void_p])
        L.oracle_key_mean.restype = ctypes.c_int
        L.oracle_key_mean.argtypes = [ctypes.c_void_p] + [ctypes.c_int32] * 4 + [ctypes.c_int64, ctypes.c_void_p]
        L.oracle_quantize_chunk_ex.restype = ctypes.c_int
        L.oracle_quantize_chunk_ex.argtypes = ([ctypes.c_void_p] + [ctypes.c_int32] * 4 +
                                               [ctypes.c_int64, ctypes.c_void_p, ctypes.c_int32] +
                                               [ctypes.c_void_p] * 3)
        L.oracle_attention_rows_slots_kmean.restype = ctypes.c_int
        L.oracle_attention_rows_slots_kmean.argtypes = (
            [ctypes.c_void_p] + [ctypes.c_int32] * 4 + [ctypes.c_int64] + [ctypes.c_void_p] * 7 +
            [ctypes.c_int32] * 2 + [ctypes.c_void_p, ctypes.c_int32, ctypes.c_double, ctypes.c_void_p,
                                    ctypes.c_int32, ctypes.c_void_p])
        del u8p
        _LIB = L
    return _LIB


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def e2m1_decode(code: int) -> float:
    return lib().oracle_e2m1_decode(code)


def e2m1_encode(v: float) -> int:
    return lib().oracle_e2m1_encode(v)


def e4m3_decode(code: int) -> float:
    return lib().oracle_e4m3_decode(code)


def e4m3_encode(v: float) -> int:
    return lib().oracle_e4m3_encode(v)


def e2m1_encode_array(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(x.shape, np.uint8)
    lib().oracle_e2m1_encode_array(_ptr(x), x.size, _ptr(out))
    return out


def e4m3_encode_array(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(x.shape, np.uint8)
    lib().oracle_e4m3_encode_array(_ptr(x), x.size, _ptr(out))
    return out


def key_mean(x_bf16: np.ndarray, token_stride: int | None = None) -> np.ndarray:
    """K-smoothing's channel mean of one chunk ``x_bf16`` (uint16 [B, L, H, d]): float32 [B, H, d],
    the exact mean rounded once to fp32 (nearest, ties to even)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    B, L, H, d = x.shape
    stride = H * d if token_stride is None else token_stride
    out = np.zeros((B, H, d), np.float32)
    if lib().oracle_key_mean(_ptr(x), B, L, H, d, stride, _ptr(out)) != 0:
        raise ValueError("oracle_key_mean rejected its arguments")
    return out


def quantize_chunk(x_bf16: np.ndarray, token_stride: int | None = None, mean: np.ndarray | None = None,
                   adaptive: bool = False):
    """Quantise one chunk ``x_bf16`` (uint16, shape [B, L, H, d]) of K or V.

    ``mean`` ([B, H, d] float32) quantises x - mean (K-smoothing); ``adaptive`` chooses each
    block's scale target from {6, 4}.  Returns ``(codes [B,H,L,d/2] u8, scales [B,H,L,d/16] u8,
    gscale [B,H] f32)``.
    """
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    B, L, H, d = x.shape
    stride = H * d if token_stride is None else token_stride
    codes = np.zeros((B, H, L, d // 2), np.uint8)
    scales = np.zeros((B, H, L, d // 16), np.uint8)
    g = np.zeros((B, H), np.float32)
    if mean is None and not adaptive:
        rc = lib().oracle_quantize_chunk(_ptr(x), B, L, H, d, stride, _ptr(codes), _ptr(scales), _ptr(g))
    else:
        mp = None
        if mean is not None:
            mean = np.ascontiguousarray(mean, dtype=np.float32)
            assert mean.shape == (B, H, d)
            mp = _ptr(mean)
        rc = lib().oracle_quantize_chunk_ex(_ptr(x), B, L, H, d, stride, mp, 1 if adaptive else 0,
                                            _ptr(codes), _ptr(scales), _ptr(g))
    if rc != 0:
        raise ValueError("oracle_quantize_chunk rejected its arguments")
    return codes, scales, g


class Cache:
    """Oracle-side NVFP4 cache for one tensor pair (K, V), laid out as the format states.

    ``smooth_k`` stores every chunk's K as x - mu with its channel mean mu (``k_mean``,
    [B, H, C, d] float32); ``adaptive_v`` chooses V's block scale targets from {6, 4}.
    """

    def __init__(self, B: int, H: int, d: int, chunk_tokens: int, capacity: int, smooth_k: bool = False,
                 adaptive_v: bool = False):
        self.B, self.H, self.d, self.Lc, self.C = B, H, d, chunk_tokens, capacity
        self.smooth_k, self.adaptive_v = smooth_k, adaptive_v
        T = chunk_tokens * capacity
        self.k_codes = np.zeros((B, H, T, d // 2), np.uint8)
        self.v_codes = np.zeros((B, H, T, d // 2), np.uint8)
        self.k_scales = np.zeros((B, H, T, d // 16), np.uint8)
        self.v_scales = np.zeros((B, H, T, d // 16), np.uint8)
        self.k_g = np.zeros((B, H, capacity), np.float32)
        self.v_g = np.zeros((B, H, capacity), np.float32)
        self.k_mean = np.zeros((B, H, capacity, d), np.float32) if smooth_k else None

    def append(self, slot: int, k_bf16: np.ndarray, v_bf16: np.ndarray) -> None:
        """Quantise a new chunk's K and V ([B, Lc, H, d] uint16) into chunk slot ``slot``."""
        t0, t1 = slot * self.Lc, (slot + 1) * self.Lc
        mu = None
        if self.smooth_k:
            mu = key_mean(k_bf16)
            self.k_mean[:, :, slot] = mu
        for x, codes, scales, g, m, ad in ((k_bf16, self.k_codes, self.k_scales, self.k_g, mu, False),
                                           (v_bf16, self.v_codes, self.v_scales, self.v_g, None, self.adaptive_v)):
            c, s, gg = quantize_chunk(x, mean=m, adaptive=ad)
            codes[:, :, t0:t1] = c
            scales[:, :, t0:t1] = s
            g[:, :, slot] = gg

    def dequantize(self, which: str) -> np.ndarray:
        """The keys or values the cache stands for, fp64 [B, H, T, d] (smoothed keys include mu)."""
        codes, scales, g = ((self.k_codes, self.k_scales, self.k_g) if which == "k" else
                            (self.v_codes, self.v_scales, self.v_g))
        out = np.zeros((self.B, self.H, self.Lc * self.C, self.d), np.float64)
        rc = lib().oracle_dequantize(_ptr(codes), _ptr(scales), _ptr(g), self.B, self.H, self.d,
                                     self.Lc, self.C, _ptr(out))
        if rc != 0:
            raise ValueError("oracle_dequantize rejected its arguments")
        if which == "k" and self.k_mean is not None:
            out += np.repeat(self.k_mean.astype(np.float64), self.Lc, axis=2)
        return out


def visible_chunks(q_chunk: int, n_sink: int, window: int, capacity: int) -> list[int]:
    out = np.zeros(max(capacity, 1), np.int32)
    n = lib().oracle_visible_chunks(q_chunk, n_sink, window, capacity, _ptr(out))
    if n < 0:
        raise ValueError("oracle_visible_chunks rejected its arguments")
    return [int(c) for c in out[:n]]


def multishot_chunks(q_chunk: int, n_sink: int, window: int, shot_start: int, shot_len: int,
                     capacity: int) -> list[int]:
    """Global sink U shot sink (start, len) U sliding window, each chunk once, ascending."""
    out = np.zeros(max(capacity, 1), np.int32)
    n = lib().oracle_multishot_chunks(q_chunk, n_sink, window, shot_start, shot_len, capacity, _ptr(out))
    if n < 0:
        raise ValueError("oracle_multishot_chunks rejected its arguments")
    return [int(c) for c in out[:n]]


def attention_rows_slots(q_bf16: np.ndarray, cache: Cache, slots, rows: np.ndarray,
                         softmax_scale: float = 0.0) -> np.ndarray:
    """fp64 attention of ``rows`` over the keys of the listed chunk slots (union, any order)."""
    q = np.ascontiguousarray(q_bf16, dtype=np.uint16)
    B, Lq, H, d = q.shape
    rows = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
    sl = np.ascontiguousarray(slots, dtype=np.int32).reshape(-1)
    out = np.zeros((rows.shape[0], d), np.float64)
    c = cache
    km = getattr(c, "k_mean", None)
    rc = lib().oracle_attention_rows_slots_kmean(
        _ptr(q), B, Lq, H, d, H * d, _ptr(c.k_codes), _ptr(c.k_scales), _ptr(c.k_g),
        None if km is None else _ptr(km),
        _ptr(c.v_codes), _ptr(c.v_scales), _ptr(c.v_g), c.Lc, c.C, _ptr(sl), sl.shape[0],
        float(softmax_scale), _ptr(rows), rows.shape[0], _ptr(out))
    if rc != 0:
        raise ValueError("oracle_attention_rows_slots rejected its arguments")
    return out


def attention_rows(q_bf16: np.ndarray, cache: Cache, q_chunk: int, n_sink: int, window: int,
                   rows: np.ndarray, softmax_scale: float = 0.0,
                   q_token_stride: int | None = None) -> np.ndarray:
    """fp64 attention for the query rows ``rows`` (int32 [n, 3] of (b, h, i)).

    ``q_bf16`` is uint16 of shape [B, Lq, H, d].  Returns float64 [n, d].
    """
    if getattr(cache, "k_mean", None) is not None:
        if q_token_stride is not None:
            raise ValueError("smoothed-key attention takes packed queries")
        return attention_rows_slots(q_bf16, cache, visible_chunks(q_chunk, n_sink, window, cache.C), rows,
                                    softmax_scale)
    q = np.ascontiguousarray(q_bf16, dtype=np.uint16)
    B, Lq, H, d = q.shape
    stride = H * d if q_token_stride is None else q_token_stride
    rows = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
    out = np.zeros((rows.shape[0], d), np.float64)
    c = cache
    rc = lib().oracle_attention_rows(
        _ptr(q), B, Lq, H, d, stride, _ptr(c.k_codes), _ptr(c.k_scales), _ptr(c.k_g),
        _ptr(c.v_codes), _ptr(c.v_scales), _ptr(c.v_g), c.Lc, c.C, q_chunk, n_sink, window,
        float(softmax_scale), _ptr(rows), rows.shape[0], _ptr(out))
    if rc != 0:
        raise ValueError("oracle_attention_rows rejected its arguments")
    return out
