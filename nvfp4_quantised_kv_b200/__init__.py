"""Python binding of libnvfp4kv (include/nvfp4kv.h): argument marshalling only.

Every step of the NVFP4 KV path runs in the library's CUDA kernels; this module checks
tensor shapes, passes raw device pointers and the current torch CUDA stream through
ctypes, and turns status codes into exceptions.  torch provides device memory and
streams.  There is no fallback: if ``libnvfp4kv.so`` is missing or cannot be loaded, every
call raises.

    cache = KVCache(batch=1, heads=12, chunk_tokens=4680, capacity=4)
    cache.quantize(slot, k, v)                     # k, v: bf16 [B, Lc, H, 128] on cuda
    out = cache.attention(q, q_chunk=3, n_sink=1, window=3)   # q: bf16 [B, Lq, H, 128]
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnvfp4kv.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_CUDA = 3
ERR_DEVICE_TIMEOUT = 4
ERR_WORKSPACE = 5
OUT_F32 = 0
OUT_BF16 = 1
HEAD_DIM = 128
K_SMOOTH = 1  # recipe option: K-smoothing of K (channel mean per chunk, added back in attention)
V_ADAPTIVE_SCALE = 2  # recipe option: per-block scale target chosen from {6, 4} for V

# Every function the C header declares, with its ctypes signature.
_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


class CacheDesc(ctypes.Structure):
    """Mirror of ``nvfp4kv_cache``."""
    _fields_ = [("batch", _i32), ("heads", _i32), ("head_dim", _i32), ("chunk_tokens", _i32),
                ("capacity_chunks", _i32), ("k_codes", _vp), ("v_codes", _vp),
                ("k_scales", _vp), ("v_scales", _vp), ("k_gscale", _vp), ("v_gscale", _vp),
                ("status", _vp), ("flags", ctypes.c_uint32), ("k_mean", _vp)]


_CP = ctypes.POINTER(CacheDesc)
SIGNATURES = {
    "nvfp4kv_cache_sizes": (ctypes.c_int, [_i32, _i32, _i32, _i32, _i32, ctypes.POINTER(_sz),
                                           ctypes.POINTER(_sz), ctypes.POINTER(_sz)]),
    "nvfp4kv_workspace_bytes": (_sz, [_CP, _i32]),
    "nvfp4_kv_quantize": (ctypes.c_int, [_CP, _i32, _vp, _vp, _i64, _vp, _sz, _vp]),
    "nvfp4_kv_quantize_static_scratch": (ctypes.c_int, [_CP, _i32, _vp, _vp, _i64, _vp]),
    "nvfp4_kv_quantize_layers": (ctypes.c_int, [_CP, _i32, _i32, ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i64,
                                                _vp, _sz, _vp]),
    "nvfp4kv_quantize_layers_workspace_bytes": (_sz, [_CP, _i32]),
    "nvfp4_kv_attention": (ctypes.c_int, [_CP, _vp, _i32, _i64, _i32, _i32, _i32, ctypes.c_float,
                                          _vp, _i32, _vp, _sz, _vp]),
    "nvfp4_kv_attention_slots": (ctypes.c_int, [_CP, _vp, _i32, _i64, ctypes.POINTER(_i32), _i32,
                                                ctypes.c_float, _vp, _i32, _vp, _sz, _vp]),
    "nvfp4_kv_dequantize": (ctypes.c_int, [_CP, _i32, _i32, _i32, _vp, _vp]),
    "nvfp4kv_debug_encode": (ctypes.c_int, [_vp, _i64, _vp, _vp, _vp]),
    "nvfp4kv_quantize_launches": (ctypes.c_int, [_CP]),
    "nvfp4_kv_attention_multishot": (ctypes.c_int, [_CP, _vp, _i32, _i64, _i32, _i32, _i32, _i32, _i32,
                                                    ctypes.c_float, _vp, _i32, _vp, _sz, _vp]),
    "nvfp4kv_attention_plan": (ctypes.c_int, [_CP, _i32, _i32, _i32, _i32, _i32, ctypes.POINTER(_i32)]),
    "nvfp4kv_debug_wait_timeout": (ctypes.c_int, [_CP, _vp]),
    "nvfp4kv_read_status": (ctypes.c_int, [_CP, _vp, ctypes.POINTER(ctypes.c_uint32)]),
    "nvfp4kv_strerror": (ctypes.c_char_p, [ctypes.c_int]),
}

_LIB = None


class NvFp4KvError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} (status {code})")


def lib() -> ctypes.CDLL:
    """Load libnvfp4kv.so (in-tree).  Raises when it is not built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run `python -m nvfp4_quantised_kv_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def strerror(code: int) -> str:
    return lib().nvfp4kv_strerror(code).decode()


def _check(rc: int, what: str) -> None:
    if rc != OK:
        raise NvFp4KvError(rc, what)


def cache_sizes(batch: int, heads: int, chunk_tokens: int, capacity: int, head_dim: int = HEAD_DIM):
    """(codes, scales, gscale) bytes per tensor for a cache of this shape."""
    c, s, g = _sz(), _sz(), _sz()
    _check(lib().nvfp4kv_cache_sizes(batch, heads, head_dim, chunk_tokens, capacity,
                                     ctypes.byref(c), ctypes.byref(s), ctypes.byref(g)),
           "nvfp4kv_cache_sizes")
    return c.value, s.value, g.value


def _stream_handle(stream) -> ctypes.c_void_p:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _token_stride(t, name: str, tokens: int, heads: int) -> int:
    """Token stride (elements) of a bf16 [B, L, H, 128] view with contiguous heads."""
    import torch
    if t.dtype != torch.bfloat16 or not t.is_cuda or t.dim() != 4:
        raise ValueError(f"{name} must be a bf16 CUDA tensor of shape [B, L, H, {HEAD_DIM}]")
    B, L, H, d = t.shape
    if L != tokens or H != heads or d != HEAD_DIM:
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected [B, {tokens}, {heads}, {HEAD_DIM}]")
    sb, st, sh, se = t.stride()
    if se != 1 or sh != HEAD_DIM or (B > 1 and sb != L * st):
        raise ValueError(f"{name} needs contiguous heads and a uniform token stride")
    return st


def workspace_bytes(batch: int, heads: int, chunk_tokens: int, capacity: int, q_tokens: int) -> int:
    """Scratch bytes the calls on a cache of this shape need on the current device."""
    d = CacheDesc(batch, heads, HEAD_DIM, chunk_tokens, capacity, 16, 16, 16, 16, 16, 16, 16)
    n = lib().nvfp4kv_workspace_bytes(ctypes.byref(d), q_tokens)
    if n == 0:
        raise NvFp4KvError(ERR_INVALID_ARG, "nvfp4kv_workspace_bytes")
    return n


class KVCache:
    """One layer's NVFP4 KV cache; the arrays are torch CUDA tensors owned by this object."""

    def __init__(self, batch: int, heads: int, chunk_tokens: int, capacity: int,
                 q_tokens_max: int = 0, device=None, workspace=None, smooth_k: bool = False,
                 adaptive_v: bool = False):
        """``workspace``: an optional uint8 CUDA tensor used as this cache's scratch instead of one
        of its own (caches that run on one stream, one call at a time, may share it).
        ``smooth_k`` / ``adaptive_v``: the recipe options K_SMOOTH / V_ADAPTIVE_SCALE."""
        import torch
        self.batch, self.heads, self.chunk_tokens, self.capacity = batch, heads, chunk_tokens, capacity
        dev = torch.device("cuda") if device is None else torch.device(device)
        T = chunk_tokens * capacity
        cache_sizes(batch, heads, chunk_tokens, capacity)  # validates the shape
        u8 = dict(dtype=torch.uint8, device=dev)
        self.k_codes = torch.zeros(batch, heads, T, HEAD_DIM // 2, **u8)
        self.v_codes = torch.zeros(batch, heads, T, HEAD_DIM // 2, **u8)
        self.k_scales = torch.zeros(batch, heads, T, HEAD_DIM // 16, **u8)
        self.v_scales = torch.zeros(batch, heads, T, HEAD_DIM // 16, **u8)
        self.k_gscale = torch.zeros(batch, heads, capacity, dtype=torch.float32, device=dev)
        self.v_gscale = torch.zeros(batch, heads, capacity, dtype=torch.float32, device=dev)
        self.status = torch.zeros(4, dtype=torch.int32, device=dev)
        self.flags = (K_SMOOTH if smooth_k else 0) | (V_ADAPTIVE_SCALE if adaptive_v else 0)
        self.k_mean = (torch.zeros(batch, heads, capacity, HEAD_DIM, dtype=torch.float32, device=dev)
                       if smooth_k else None)
        self.desc = CacheDesc(batch, heads, HEAD_DIM, chunk_tokens, capacity,
                              self.k_codes.data_ptr(), self.v_codes.data_ptr(),
                              self.k_scales.data_ptr(), self.v_scales.data_ptr(),
                              self.k_gscale.data_ptr(), self.v_gscale.data_ptr(),
                              self.status.data_ptr(), self.flags,
                              self.k_mean.data_ptr() if smooth_k else None)
        self._ws = workspace
        self._ws_owned = workspace is None
        self.reserve_workspace(max(q_tokens_max, 1))

    def reserve_workspace(self, q_tokens: int) -> None:
        import torch
        need = lib().nvfp4kv_workspace_bytes(ctypes.byref(self.desc), q_tokens)
        if need == 0:
            raise NvFp4KvError(ERR_INVALID_ARG, "nvfp4kv_workspace_bytes")
        if self._ws is None or self._ws.numel() < need:
            if not self._ws_owned:
                raise ValueError(f"the shared workspace holds {self._ws.numel()} bytes, {need} are needed")
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.k_codes.device)

    @property
    def nbytes(self) -> int:
        arrays = [self.k_codes, self.v_codes, self.k_scales, self.v_scales, self.k_gscale, self.v_gscale]
        if self.k_mean is not None:
            arrays.append(self.k_mean)
        return sum(t.numel() * t.element_size() for t in arrays)

    def quantize(self, slot: int, k, v, stream=None) -> None:
        """Quantise bf16 K and V ([B, Lc, H, 128]) of a new chunk into chunk slot ``slot``."""
        ks = _token_stride(k, "k", self.chunk_tokens, self.heads)
        vs = _token_stride(v, "v", self.chunk_tokens, self.heads)
        if ks != vs:
            raise ValueError("k and v must share a token stride")
        _check(lib().nvfp4_kv_quantize(ctypes.byref(self.desc), slot, k.data_ptr(), v.data_ptr(), ks,
                                       self._ws.data_ptr(), self._ws.numel(), _stream_handle(stream)),
               "nvfp4_kv_quantize")

    def debug_wait_timeout(self, stream=None) -> None:
        """Fault injection: a kernel whose bounded wait runs out sets the device-timeout bit."""
        _check(lib().nvfp4kv_debug_wait_timeout(ctypes.byref(self.desc), _stream_handle(stream)),
               "nvfp4kv_debug_wait_timeout")

    def quantize_launches(self) -> int:
        """Kernels one ``quantize`` call launches for this cache on the current device (1 to 3)."""
        n = lib().nvfp4kv_quantize_launches(ctypes.byref(self.desc))
        if n < 0:
            raise NvFp4KvError(-n, "nvfp4kv_quantize_launches")
        return n

    def _out_for(self, q, out, out_dtype):
        import torch
        Lq = q.shape[1]
        if out is None:
            out = torch.empty(q.shape[0], Lq, self.heads, HEAD_DIM,
                              dtype=torch.float32 if out_dtype is None else out_dtype, device=q.device)
        if not out.is_contiguous() or out.shape != (q.shape[0], Lq, self.heads, HEAD_DIM):
            raise ValueError("out must be a contiguous [B, Lq, H, 128] tensor")
        code = {torch.float32: OUT_F32, torch.bfloat16: OUT_BF16}.get(out.dtype)
        if code is None:
            raise ValueError("out must be fp32 or bf16")
        return out, code

    def attention(self, q, q_chunk: int, n_sink: int, window: int, softmax_scale: float = 0.0,
                  out=None, out_dtype=None, stream=None):
        """Attention of bf16 queries ``q`` ([B, Lq, H, 128]) of chunk ``q_chunk`` over the
        sink + window chunks of the cache.  Returns ``out`` ([B, Lq, H, 128], fp32 by default)."""
        Lq = q.shape[1]
        qs = _token_stride(q, "q", Lq, self.heads)
        out, code = self._out_for(q, out, out_dtype)
        self.reserve_workspace(Lq)
        _check(lib().nvfp4_kv_attention(ctypes.byref(self.desc), q.data_ptr(), Lq, qs, q_chunk, n_sink,
                                        window, float(softmax_scale), out.data_ptr(), code,
                                        self._ws.data_ptr(), self._ws.numel(), _stream_handle(stream)),
               "nvfp4_kv_attention")
        return out

    def attention_slots(self, q, slots, softmax_scale: float = 0.0, out=None, out_dtype=None,
                        stream=None):
        """Attention of ``q`` over the keys of the listed chunk slots (any order, repeats once)."""
        Lq = q.shape[1]
        qs = _token_stride(q, "q", Lq, self.heads)
        out, code = self._out_for(q, out, out_dtype)
        sl = (_i32 * max(len(slots), 1))(*[int(x) for x in slots])
        self.reserve_workspace(Lq)
        _check(lib().nvfp4_kv_attention_slots(ctypes.byref(self.desc), q.data_ptr(), Lq, qs, sl, len(slots),
                                              float(softmax_scale), out.data_ptr(), code,
                                              self._ws.data_ptr(), self._ws.numel(), _stream_handle(stream)),
               "nvfp4_kv_attention_slots")
        return out

    def attention_multishot(self, q, q_chunk: int, n_sink: int, window: int, shot_start: int,
                            shot_len: int, softmax_scale: float = 0.0, out=None, out_dtype=None,
                            stream=None):
        """Multi-shot attention sink: the library attends to the global sink {c < n_sink}, the
        current shot's sink {shot_start <= c < shot_start + shot_len} and the window
        {q_chunk - window < c <= q_chunk}, each chunk once."""
        Lq = q.shape[1]
        qs = _token_stride(q, "q", Lq, self.heads)
        out, code = self._out_for(q, out, out_dtype)
        self.reserve_workspace(Lq)
        _check(lib().nvfp4_kv_attention_multishot(ctypes.byref(self.desc), q.data_ptr(), Lq, qs, q_chunk,
                                                  n_sink, window, shot_start, shot_len, float(softmax_scale),
                                                  out.data_ptr(), code, self._ws.data_ptr(), self._ws.numel(),
                                                  _stream_handle(stream)),
               "nvfp4_kv_attention_multishot")
        return out

    def dequantize(self, which: str, first_slot: int = 0, n_slots: int | None = None, stream=None):
        """fp32 [B, H, n_slots*Lc, 128] dequantised K (``which='k'``) or V."""
        import torch
        n = self.capacity - first_slot if n_slots is None else n_slots
        out = torch.empty(self.batch, self.heads, n * self.chunk_tokens, HEAD_DIM, dtype=torch.float32,
                          device=self.k_codes.device)
        _check(lib().nvfp4_kv_dequantize(ctypes.byref(self.desc), 0 if which == "k" else 1, first_slot,
                                         n, out.data_ptr(), _stream_handle(stream)),
               "nvfp4_kv_dequantize")
        return out

    def read_status(self, stream=None) -> int:
        """Synchronise the stream and return (and clear) the device status word."""
        v = ctypes.c_uint32(0)
        _check(lib().nvfp4kv_read_status(ctypes.byref(self.desc), _stream_handle(stream), ctypes.byref(v)),
               "nvfp4kv_read_status")
        return v.value


def quantize_layers(caches, slot: int, ks, vs, workspace=None, stream=None):
    """Quantise the new chunk of every layer in one launch: bf16 ``ks[l]``, ``vs[l]``
    ([B, Lc, H, 128]) into chunk slot ``slot`` of ``caches[l]`` (caches of one shape)."""
    import torch
    n = len(caches)
    if n == 0 or len(ks) != n or len(vs) != n:
        raise ValueError("one K and one V tensor per cache")
    c0 = caches[0]
    strides = {_token_stride(t, "k/v", c0.chunk_tokens, c0.heads) for t in list(ks) + list(vs)}
    if len(strides) != 1:
        raise ValueError("every K and V tensor must share one token stride")
    descs = (CacheDesc * n)(*[c.desc for c in caches])
    need = lib().nvfp4kv_quantize_layers_workspace_bytes(descs, n)
    if need == 0:
        raise NvFp4KvError(ERR_INVALID_ARG, "nvfp4kv_quantize_layers_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=c0.k_codes.device)
    kp = (_vp * n)(*[t.data_ptr() for t in ks])
    vp = (_vp * n)(*[t.data_ptr() for t in vs])
    _check(lib().nvfp4_kv_quantize_layers(descs, n, slot, kp, vp, strides.pop(), workspace.data_ptr(),
                                          workspace.numel(), _stream_handle(stream)),
           "nvfp4_kv_quantize_layers")
    return workspace


def attention_plan(cache_desc, q_tokens: int, kv_tiles: int, n_sms: int = 0, cta: int = -1, seg: int = -1):
    """The attention work split (``nvfp4kv_attention_plan``): a list of 8 ints."""
    out = (_i32 * 8)()
    _check(lib().nvfp4kv_attention_plan(ctypes.byref(cache_desc), q_tokens, kv_tiles, n_sms, cta, seg, out),
           "nvfp4kv_attention_plan")
    return list(out)


def debug_encode(x, stream=None):
    """Device E2M1 and E4M3 codes of the fp32 CUDA tensor ``x`` (diagnostic probe)."""
    import torch
    x = x.contiguous()
    e2 = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    e4 = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    _check(lib().nvfp4kv_debug_encode(x.data_ptr(), x.numel(), e2.data_ptr(), e4.data_ptr(),
                                      _stream_handle(stream)), "nvfp4kv_debug_encode")
    return e2, e4
