"""Every finite fp32 value through the device's E2M1 and E4M3 conversions against the oracle's
codecs.

The oracle's encoders round to the nearest representable magnitude (ties to the even code) and
saturate, so on non-negative inputs each is a non-decreasing step function of the value, and fp32
bit patterns of non-negative values order like the values.  Bisection over bit patterns finds,
with the oracle itself, the first pattern of every code; the expected code of any non-negative
pattern is then the number of those thresholds at or below it.  Negative inputs take the sign bit
on top of the magnitude code, which the test checks against the oracle on a sample.  The device
codes of all 2^32 - 2^24 finite patterns are compared with that on the GPU, slice by slice.
"""
import struct

import numpy as np
import pytest

import oracle
from nvfp4_quantised_kv_b200 import debug_encode

pytestmark = pytest.mark.gpu

POS_FINITE_END = 0x7F800000  # +inf; every smaller non-negative pattern is finite


def _f(bits: int) -> float:
    return struct.unpack("<f", struct.pack("<I", bits))[0]


def _thresholds(encode, n_codes):
    """First non-negative fp32 bit pattern whose oracle code is >= c, for c = 1 .. n_codes - 1."""
    out = []
    for c in range(1, n_codes):
        lo, hi = 0, POS_FINITE_END - 1
        if encode(_f(hi)) < c:
            break
        while lo < hi:  # smallest pattern p with encode(p) >= c
            mid = (lo + hi) // 2
            if encode(_f(mid)) >= c:
                hi = mid
            else:
                lo = mid + 1
        out.append(lo)
    return out


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_every_finite_fp32_converts_as_the_oracle(fmt):
    import torch
    enc = oracle.e2m1_encode if fmt == "e2m1" else oracle.e4m3_encode
    n_codes, sign = (8, 0x8) if fmt == "e2m1" else (127, 0x80)
    thr = _thresholds(enc, n_codes)
    assert len(thr) == n_codes - 1 and thr == sorted(thr)
    # the thresholds are where the oracle's code changes: one pattern below each has the code below
    for c, t in enumerate(thr, start=1):
        assert enc(_f(t)) == c and enc(_f(t - 1)) == c - 1
    # negative inputs: the sign bit on top of the magnitude code (checked on a sample)
    rng = np.random.default_rng(17)
    pos = rng.integers(0, POS_FINITE_END, size=1 << 16, dtype=np.uint64).astype(np.uint32)
    neg = (pos | np.uint32(0x80000000)).view(np.float32)
    codec_array = oracle.e2m1_encode_array if fmt == "e2m1" else oracle.e4m3_encode_array
    assert np.array_equal(codec_array(neg), codec_array(pos.view(np.float32)) | np.uint8(sign))

    dev = torch.device("cuda")
    t_dev = torch.tensor(thr, dtype=torch.int64, device=dev)
    step = 1 << 26
    bad = checked = 0
    for base in range(0, POS_FINITE_END, step):
        n = min(step, POS_FINITE_END - base)
        bits = torch.arange(base, base + n, dtype=torch.int64, device=dev)
        want = torch.searchsorted(t_dev, bits, right=True).to(torch.uint8)
        for neg_half in (False, True):
            b32 = (bits | 0x80000000) if neg_half else bits
            x = b32.to(torch.int32).view(torch.float32)  # the low 32 bits, reinterpreted
            e2, e4 = debug_encode(x)
            got = e2 if fmt == "e2m1" else e4
            exp = want | sign if neg_half else want
            bad += int((got != exp).sum())
            checked += got.numel()
        del bits, want
    assert checked == 2 * POS_FINITE_END  # every finite pattern of both signs
    assert bad == 0
