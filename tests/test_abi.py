"""The C-ABI library loads on a machine without a GPU, exports every function its header
declares, sizes the cache by the pages' closed form, and rejects bad arguments before
touching CUDA."""
import ctypes
import os
import re

import pytest

import nvfp4_quantised_kv_b200 as nk
from nvfp4_quantised_kv_b200 import build as kbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "nvfp4kv.h")


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    return nk.lib()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(nvfp4[a-z_0-9]*)\s*\(", text,
                                 flags=re.M)))


def test_every_declared_symbol_is_exported(L):
    names = _declared_functions()
    assert len(names) >= 8
    for name in names:
        assert hasattr(L, name), name
    assert set(names) == set(nk.SIGNATURES)


def test_cache_sizes_follow_nine_eighths_closed_form(L):
    # reading note, "The inference infrastructure": K+V storage 4*Tc*H*d (bf16) -> 9/8*Tc*H*d
    Tc, H, d = 4680, 12, 128
    codes, scales, g = nk.cache_sizes(1, H, Tc, 1)
    assert 2 * (codes + scales) * 8 == 9 * Tc * H * d
    assert g == H * 4
    # the 30-layer, 40-chunk rollout cache: 9.70 GB NVFP4 against 34.5 GB of bf16
    codes, scales, g = nk.cache_sizes(1, 12, 4680, 40)
    total = 30 * 2 * (codes + scales + g)
    assert abs(total / 1e9 - 9.704) < 0.001
    assert abs(30 * 4 * 40 * 4680 * 12 * 128 / total - 3.556) < 0.001
    assert L.nvfp4kv_cache_sizes(1, 1, 24, 2, 1, None, None, None) == nk.ERR_INVALID_ARG
    assert L.nvfp4kv_cache_sizes(0, 1, 128, 2, 1, None, None, None) == nk.ERR_INVALID_ARG


def _desc(**kw):
    base = dict(batch=1, heads=2, head_dim=128, chunk_tokens=64, capacity_chunks=4,
                k_codes=0x10000, v_codes=0x20000, k_scales=0x30000, v_scales=0x40000,
                k_gscale=0x50000, v_gscale=0x60000, status=0x70000)
    base.update(kw)
    d = nk.CacheDesc()
    for k, v in base.items():
        setattr(d, k, v)
    return d


def _quant(L, d, slot=0, k=0x80000, v=0x90000, stride=256, ws=0xA0000, ws_bytes=1 << 20):
    return L.nvfp4_kv_quantize(ctypes.byref(d), slot, k, v, stride, ws, ws_bytes, None)


def _attn(L, d, q=0x80000, lq=64, stride=256, q_chunk=3, sink=1, window=3, out=0x90000,
          dtype=0, ws=0xA0000, ws_bytes=1 << 20):
    return L.nvfp4_kv_attention(ctypes.byref(d), q, lq, stride, q_chunk, sink, window, 0.0, out,
                                dtype, ws, ws_bytes, None)


def _attn_slots(L, d, slots, q=0x80000, lq=64, stride=256, out=0x90000, dtype=0):
    arr = (ctypes.c_int32 * max(len(slots), 1))(*slots)
    return L.nvfp4_kv_attention_slots(ctypes.byref(d), q, lq, stride, arr if slots else None, len(slots),
                                      0.0, out, dtype, 0xA0000, 1 << 20, None)


def test_attention_slot_list_argument_checks(L):
    d = _desc(capacity_chunks=12)
    assert _attn_slots(L, d, []) == nk.ERR_INVALID_ARG
    assert _attn_slots(L, d, [0, 12]) == nk.ERR_INVALID_ARG        # slot >= capacity
    assert _attn_slots(L, d, [-1]) == nk.ERR_INVALID_ARG
    assert _attn_slots(L, d, [0, 2, 4, 6, 8]) == nk.ERR_UNSUPPORTED  # five runs of slots
    assert _attn_slots(L, d, [0, 2, 4, 6, 7], lq=0) == nk.ERR_INVALID_ARG


def _attn_ms(L, d, q_chunk=9, sink=1, window=2, start=4, length=2, lq=64):
    return L.nvfp4_kv_attention_multishot(ctypes.byref(d), 0x80000, lq, 256, q_chunk, sink, window, start,
                                          length, 0.0, 0x90000, 0, 0xA0000, 1 << 30, None)


def test_multishot_argument_checks(L):
    # paper page, section 4.2: the shot's sink (start, len) is history of the query chunk
    d = _desc(capacity_chunks=12)
    assert _attn_ms(L, d, start=-1) == nk.ERR_INVALID_ARG
    assert _attn_ms(L, d, length=-1) == nk.ERR_INVALID_ARG
    assert _attn_ms(L, d, start=9, length=2) == nk.ERR_INVALID_ARG   # ends past the query chunk
    assert _attn_ms(L, d, q_chunk=12) == nk.ERR_INVALID_ARG
    assert _attn_ms(L, d, window=0) == nk.ERR_INVALID_ARG
    assert _attn_ms(L, d, sink=-1) == nk.ERR_INVALID_ARG
    assert _attn_ms(L, d, lq=0) == nk.ERR_INVALID_ARG
    assert L.nvfp4_kv_attention_multishot(None, 0x80000, 64, 256, 9, 1, 2, 4, 2, 0.0, 0x90000, 0, 0xA0000,
                                          1 << 30, None) == nk.ERR_INVALID_ARG


def test_quantize_argument_checks(L):
    assert L.nvfp4_kv_quantize(None, 0, 0x80000, 0x90000, 256, 0xA0000, 1 << 20, None) == nk.ERR_INVALID_ARG
    assert _quant(L, _desc(head_dim=64)) == nk.ERR_UNSUPPORTED
    assert _quant(L, _desc(chunk_tokens=63)) == nk.ERR_UNSUPPORTED
    assert _quant(L, _desc(k_codes=0x10008)) == nk.ERR_INVALID_ARG   # misaligned cache array
    assert _quant(L, _desc(status=None)) == nk.ERR_INVALID_ARG
    assert _quant(L, _desc(), slot=4) == nk.ERR_INVALID_ARG           # slot >= capacity
    assert _quant(L, _desc(), slot=-1) == nk.ERR_INVALID_ARG
    assert _quant(L, _desc(), k=0x80002) == nk.ERR_INVALID_ARG        # misaligned input
    assert _quant(L, _desc(), stride=255) == nk.ERR_INVALID_ARG       # stride < H*d
    assert _quant(L, _desc(), stride=260) == nk.ERR_INVALID_ARG       # stride not a multiple of 8
    assert _quant(L, _desc(), ws=None) == nk.ERR_WORKSPACE
    assert _quant(L, _desc(), ws_bytes=4) == nk.ERR_WORKSPACE


def test_attention_argument_checks(L):
    d = _desc()
    assert _attn(L, d, q_chunk=4) == nk.ERR_INVALID_ARG
    assert _attn(L, d, window=0) == nk.ERR_INVALID_ARG
    assert _attn(L, d, sink=-1) == nk.ERR_INVALID_ARG
    assert _attn(L, d, lq=0) == nk.ERR_INVALID_ARG
    assert _attn(L, d, dtype=7) == nk.ERR_INVALID_ARG
    assert _attn(L, d, out=0x90004) == nk.ERR_INVALID_ARG
    assert _attn(L, d, stride=100) == nk.ERR_INVALID_ARG
    assert _attn(L, _desc(head_dim=256)) == nk.ERR_UNSUPPORTED


def test_dequantize_and_status_argument_checks(L):
    d = _desc()
    assert L.nvfp4_kv_dequantize(ctypes.byref(d), 2, 0, 1, 0x90000, None) == nk.ERR_INVALID_ARG
    assert L.nvfp4_kv_dequantize(ctypes.byref(d), 0, 3, 2, 0x90000, None) == nk.ERR_INVALID_ARG
    assert L.nvfp4_kv_dequantize(ctypes.byref(d), 0, 0, 1, 0x90008, None) == nk.ERR_INVALID_ARG
    assert L.nvfp4kv_read_status(None, None, None) == nk.ERR_INVALID_ARG
    assert L.nvfp4kv_quantize_launches(None) == -nk.ERR_INVALID_ARG
    assert L.nvfp4kv_debug_wait_timeout(None, None) == nk.ERR_INVALID_ARG
    assert L.nvfp4kv_quantize_launches(ctypes.byref(_desc(head_dim=256))) == -nk.ERR_UNSUPPORTED
    assert L.nvfp4kv_debug_encode(None, 4, 0x1000, 0x2000, None) == nk.ERR_INVALID_ARG
    assert L.nvfp4kv_workspace_bytes(None, 64) == 0
    assert L.nvfp4kv_workspace_bytes(ctypes.byref(d), 64) >= 256


def test_valid_arguments_without_a_gpu_report_a_cuda_error(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _quant(L, _desc()) == nk.ERR_CUDA
    assert _attn(L, _desc()) == nk.ERR_CUDA
    # four runs, listed out of order and with repeats: valid, so it reaches the device check
    assert _attn_slots(L, _desc(capacity_chunks=12), [9, 0, 4, 5, 0, 7, 9]) == nk.ERR_CUDA
    assert _attn_ms(L, _desc(capacity_chunks=12)) == nk.ERR_CUDA
    assert _attn_ms(L, _desc(capacity_chunks=12), start=9, length=1) == nk.ERR_CUDA  # shot = query chunk
    assert L.nvfp4kv_quantize_launches(ctypes.byref(_desc())) == -nk.ERR_CUDA
    assert L.nvfp4kv_debug_wait_timeout(ctypes.byref(_desc()), None) == nk.ERR_CUDA


def test_strerror_covers_every_code(L):
    for code in range(6):
        assert nk.strerror(code) != "unknown status"
    assert nk.strerror(99) == "unknown status"


def test_recipe_flags_are_checked_before_any_launch(L):
    bad = _desc(flags=4)  # an unknown option bit
    assert L.nvfp4_kv_quantize(ctypes.byref(bad), 0, 0x80000, 0x90000, 256, 0xA0000, 1 << 20, None) == nk.ERR_INVALID_ARG
    no_mean = _desc(flags=nk.K_SMOOTH)  # smoothing without its mean array
    assert L.nvfp4_kv_quantize(ctypes.byref(no_mean), 0, 0x80000, 0x90000, 256, 0xA0000, 1 << 20,
                               None) == nk.ERR_INVALID_ARG
    odd = _desc(flags=nk.K_SMOOTH, k_mean=0xB0008)  # misaligned mean array
    assert L.nvfp4_kv_quantize(ctypes.byref(odd), 0, 0x80000, 0x90000, 256, 0xA0000, 1 << 20, None) == nk.ERR_INVALID_ARG
    # smoothed attention needs chunks of at least 128 tokens (a tile spans at most two chunks)
    short = _desc(flags=nk.K_SMOOTH, k_mean=0xB0000, chunk_tokens=64)
    out = (ctypes.c_int32 * 1)()
    rc = L.nvfp4_kv_attention(ctypes.byref(short), 0x80000, 64, 256, 1, 1, 2, 0.0, 0xC0000, 0, 0xA0000,
                              1 << 24, None)
    assert rc == nk.ERR_UNSUPPORTED
    del out
    # smoothed chunks beyond 2^23 keys: more than the exact channel sums have room for
    long_chunk = _desc(flags=nk.K_SMOOTH, k_mean=0xB0000, chunk_tokens=(1 << 23) + 2, capacity_chunks=1)
    assert _quant(L, long_chunk) == nk.ERR_UNSUPPORTED
    assert L.nvfp4_kv_dequantize(ctypes.byref(long_chunk), 0, 0, 1, 0x90000, None) == nk.ERR_UNSUPPORTED
    # the single-launch multi-layer quantiser takes plain caches only
    pair = (nk.CacheDesc * 2)(_desc(), _desc(flags=nk.V_ADAPTIVE_SCALE))
    ks = (ctypes.c_void_p * 2)(0x80000, 0x80000)
    assert L.nvfp4_kv_quantize_layers(pair, 2, 0, ks, ks, 256, 0xA0000, 1 << 20, None) == nk.ERR_UNSUPPORTED
