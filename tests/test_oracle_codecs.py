"""Pins of the oracle's E2M1 / E4M3 codecs against the pages' format facts and torch's
float8_e4m3fn conversion (an independent library routine)."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.conftest import read_golden


def test_e2m1_decode_matches_value_table():
    for code, value in read_golden("e2m1_values.txt"):
        got = oracle.e2m1_decode(int(code))
        assert got == float(value)
        assert math.copysign(1.0, got) == math.copysign(1.0, float(value))


def test_e2m1_encode_roundtrips_every_code():
    for code in range(16):
        assert oracle.e2m1_encode(oracle.e2m1_decode(code)) == code


def test_e2m1_ties_and_saturation():
    for value, code in read_golden("e2m1_ties.txt"):
        assert oracle.e2m1_encode(float(value)) == int(code), value
    assert oracle.e2m1_encode(float("inf")) == 7
    assert oracle.e2m1_encode(float("-inf")) == 15


def test_e2m1_encode_is_nearest_on_random_values():
    grid = np.array([float(v) for _, v in read_golden("e2m1_values.txt")][:8])
    rng = np.random.default_rng(7)
    xs = rng.uniform(-7.0, 7.0, 4000).astype(np.float32)
    for x in xs:
        code = oracle.e2m1_encode(float(x))
        mag = abs(float(x))
        best = np.min(np.abs(grid - mag))
        assert abs(abs(oracle.e2m1_decode(code)) - mag) == best
        assert (code >= 8) == (x < 0)


def test_e4m3_decode_matches_torch_for_all_codes():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for code in range(256):
        got = oracle.e4m3_decode(code)
        if code in (0x7F, 0xFF):
            assert math.isnan(got) and math.isnan(ref[code])
        else:
            assert got == ref[code], code


def test_e4m3_format_extremes():
    # largest finite magnitude is M_FP8 = 448 (paper page, section 2.2); smallest subnormal 2^-9
    finite = [abs(oracle.e4m3_decode(c)) for c in range(127)]
    assert max(finite) == 448.0
    assert min(v for v in finite if v > 0) == 2.0 ** -9
    assert len(set(finite)) == 127  # 0x00..0x7E are distinct, ascending magnitudes
    assert finite == sorted(finite)


def _e4m3_sweep_values():
    mags = np.array([abs(oracle.e4m3_decode(c)) for c in range(127)], dtype=np.float64)
    mids = (mags[1:] + mags[:-1]) / 2
    rng = np.random.default_rng(3)
    rand = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(464.0), 20000))
    vals = np.concatenate([mags, mids, np.nextafter(mids.astype(np.float32), 0),
                           np.nextafter(mids.astype(np.float32), 1000), rand])
    return vals.astype(np.float32)


def test_e4m3_encode_matches_torch_in_range():
    vals = _e4m3_sweep_values()
    vals = vals[vals <= 464.0]
    vals = np.concatenate([vals, -vals])
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in vals], dtype=np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (vals[bad[:5]], got[bad[:5]], ref[bad[:5]])


@pytest.mark.parametrize("v", [448.0, 449.0, 464.0, 465.0, 1e6, float("inf")])
def test_e4m3_encode_saturates_to_448(v):
    assert oracle.e4m3_encode(v) == 0x7E
    assert oracle.e4m3_encode(-v) == 0xFE
