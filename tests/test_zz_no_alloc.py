"""The quantiser entry point that takes no workspace (nvfp4_kv_quantize_static_scratch).

It serves callers that cannot allocate device memory: code that runs inside a memory arena
planned before this library was linked, plugins whose host framework owns every device
allocation, and real-time loops that must not allocate.  It keeps its scratch (the per-slice
amax partials of the two-pass quantiser) in a fixed device array inside the library.  These
tests call it through the C ABI and check that it writes exactly the bytes the workspace
version writes, on calls in a row that all use the array with different layouts (so each call
finds the previous call's partials there), including one at the largest accepted size, and that
caches too large for the fixed array are refused before anything runs.
"""
import ctypes

import pytest

import nvfp4_quantised_kv_b200 as nk
from nvfp4_quantised_kv_b200 import synthetic

ARRAYS = ("k_codes", "v_codes", "k_scales", "v_scales", "k_gscale", "v_gscale")
SCRATCH_BYTES = 64 * 1024


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _partial_bytes(batch, heads, chunk_tokens):
    return 2 * batch * heads * (-(-chunk_tokens // 128)) * 4


def _inputs(batch, heads, chunk_tokens, seed):
    import torch
    g = torch.Generator(device="cuda").manual_seed(seed)
    shape = (batch, chunk_tokens, heads, 128)
    k = torch.randn(shape, generator=g, device="cuda").mul_(3.0).to(torch.bfloat16)
    v = torch.randn(shape, generator=g, device="cuda").to(torch.bfloat16)
    return k, v


@pytest.mark.gpu
def test_static_scratch_quantize_matches_workspace_quantize_on_calls_in_a_row():
    import torch
    nk.lib()
    w = synthetic.WORKLOADS["1.3b"]
    # (batch, heads, chunk_tokens, slot): three shapes that all take the two-pass path and lay
    # their partials out differently; the last one needs exactly the whole fixed array
    calls = [(w.batch, w.heads, w.chunk_tokens, 3), (1, 2, 7208, 1), (1, 64, 16384, 0)]
    assert _partial_bytes(*calls[-1][:3]) == SCRATCH_BYTES
    for i, (batch, heads, lc, slot) in enumerate(calls):
        ref = nk.KVCache(batch, heads, lc, slot + 1)
        alt = nk.KVCache(batch, heads, lc, slot + 1)
        assert ref.quantize_launches() == 2 and alt.quantize_launches() == 2
        if i == 0:
            import numpy as np
            kb, vb = synthetic.chunk_kv(w, slot)
            kd = torch.from_numpy(np.ascontiguousarray(kb).view(np.int16)).cuda().view(torch.bfloat16)
            vd = torch.from_numpy(np.ascontiguousarray(vb).view(np.int16)).cuda().view(torch.bfloat16)
        else:
            kd, vd = _inputs(batch, heads, lc, seed=i)
        ref.quantize(slot, kd, vd)  # the workspace entry point
        rc = nk.lib().nvfp4_kv_quantize_static_scratch(ctypes.byref(alt.desc), slot, kd.data_ptr(),
                                                       vd.data_ptr(), kd.stride(1), _stream())
        assert rc == nk.OK, nk.strerror(rc)
        torch.cuda.synchronize()
        for name in ARRAYS:  # quantised bytes are compared bit for bit, as for the workspace path
            a, b = getattr(ref, name), getattr(alt, name)
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), (i, name)
        assert float(alt.k_gscale[..., slot].abs().sum()) > 0.0
        assert alt.read_status() == 0 and ref.read_status() == 0
        del ref, alt, kd, vd


def test_static_scratch_refuses_caches_beyond_its_fixed_size():
    nk.lib()
    # one partial slot more than the fixed array holds
    d = nk.CacheDesc(1, 64, 128, 16384 + 128, 2, 0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x60000,
                     0x70000)
    assert _partial_bytes(1, 64, 16384 + 128) > SCRATCH_BYTES
    rc = nk.lib().nvfp4_kv_quantize_static_scratch(ctypes.byref(d), 0, 0x80000, 0x90000, 64 * 128, None)
    assert rc == nk.ERR_WORKSPACE
