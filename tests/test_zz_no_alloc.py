"""The quantiser entry point that takes no workspace (nvfp4_kv_quantize_static_scratch).

It serves callers that cannot allocate device memory: code that runs inside a memory arena
planned before this library was linked, plugins whose host framework owns every device
allocation, and real-time loops that must not allocate.  It keeps its scratch in a fixed
device array inside the library.  These tests call it through the C ABI and check that it
writes exactly the bytes the workspace version writes, on two calls in a row (the second
call finds the first call's leftovers in the shared array), and that caches too large for
the fixed array are refused before anything runs.
"""
import ctypes

import pytest

import nvfp4_quantised_kv_b200 as nk
from nvfp4_quantised_kv_b200 import synthetic

ARRAYS = ("k_codes", "v_codes", "k_scales", "v_scales", "k_gscale", "v_gscale")


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
def test_static_scratch_quantize_matches_workspace_quantize_on_two_calls():
    import numpy as np
    import torch
    nk.lib()
    calls = [("1.3b", 3), ("tiny", 1)]  # a large call, then a small one on a different cache
    for key, slot in calls:
        w = synthetic.WORKLOADS[key]
        ref = nk.KVCache(w.batch, w.heads, w.chunk_tokens, w.capacity)
        alt = nk.KVCache(w.batch, w.heads, w.chunk_tokens, w.capacity)
        k, v = synthetic.chunk_kv(w, slot)
        kd = torch.from_numpy(np.ascontiguousarray(k).view(np.int16)).cuda().view(torch.bfloat16)
        vd = torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).cuda().view(torch.bfloat16)
        ref.quantize(slot, kd, vd)  # the workspace entry point
        rc = nk.lib().nvfp4_kv_quantize_static_scratch(ctypes.byref(alt.desc), slot, kd.data_ptr(),
                                                       vd.data_ptr(), kd.stride(1), _stream())
        assert rc == nk.OK, nk.strerror(rc)
        torch.cuda.synchronize()
        for name in ARRAYS:  # quantised bytes are compared bit for bit, as for the workspace path
            a, b = getattr(ref, name), getattr(alt, name)
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), (key, name)
        assert float(alt.k_gscale[..., slot].abs().sum()) > 0.0
        assert alt.read_status() == 0 and ref.read_status() == 0


def test_static_scratch_refuses_caches_beyond_its_fixed_size():
    nk.lib()
    d = nk.CacheDesc(1, 9000, 128, 64, 2, 0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x60000,
                     0x70000)
    rc = nk.lib().nvfp4_kv_quantize_static_scratch(ctypes.byref(d), 0, 0x80000, 0x90000,
                                                   9000 * 128, None)
    assert rc == nk.ERR_WORKSPACE
