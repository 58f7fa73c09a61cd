"""The arithmetic fact behind the channel-mean kernel's fast path (host-side, no GPU): the fp64 sum
of at most 64 bf16 values whose non-zero magnitudes lie within 40 binades (exponent span <= 39) is
exact in any order of additions, so the kernel may add a slice's values in fp64 and move the result
into its integer bins; one binade more and an fp64 sum can lose a value.

Every bf16 value is m * 2^(p - 133) with m < 256; within a span of 39 every partial sum is a whole
number of the smallest value's unit below 64 * 256 * 2^39 = 2^53, which fp64 holds exactly."""
from fractions import Fraction

import numpy as np
import pytest

from tests._bf16 import bf16_bits_to_f32

SLICE = 64
SPAN = 39


def _pos(bits):
    """p of |v| = m * 2^(p - 133) for a finite non-zero bf16 bit pattern."""
    e = (bits >> 7) & 0xFF
    return int(e) - 1 if e else 0


def _random_slice(rng, span, n):
    """n finite bf16 patterns (some zeros) whose non-zero positions lie in [p0, p0 + span]."""
    p0 = int(rng.integers(0, 254 - span))
    pos = rng.integers(p0, p0 + span + 1, n)
    frac = rng.integers(0, 128, n)
    bits = np.where(pos == 0, frac, ((pos + 1) << 7) | frac).astype(np.uint16)  # p = 0: subnormal or e = 1
    bits |= (rng.integers(0, 2, n) << 15).astype(np.uint16)
    bits[rng.random(n) < 0.05] = 0
    return bits


def _exact(vals):
    return sum((Fraction(float(v)) for v in vals), Fraction(0))


def test_any_order_of_fp64_additions_is_exact_within_the_span():
    rng = np.random.default_rng(5)
    for trial in range(400):
        n = int(rng.integers(1, SLICE + 1))
        bits = _random_slice(rng, SPAN if trial % 2 else int(rng.integers(0, SPAN + 1)), n)
        nz = [_pos(b & 0x7FFF) for b in bits if b & 0x7FFF]
        if nz:
            assert max(nz) - min(nz) <= SPAN
        vals = bf16_bits_to_f32(bits).astype(np.float64)
        want = _exact(vals)
        for order in range(3):
            v = vals[rng.permutation(n)] if order else vals
            acc = [0.0, 0.0, 0.0, 0.0]  # four interleaved accumulators, then a pairwise finish
            for i, x in enumerate(v):
                acc[i % 4] += float(x)
            assert Fraction((acc[0] + acc[1]) + (acc[2] + acc[3])) == want
            run = 0.0
            for x in v:
                run += float(x)
            assert Fraction(run) == want


@pytest.mark.parametrize("k", [-80, -40, 0, 80])
def test_the_widest_span_holds_and_one_more_binade_fails(k):
    # 63 values 1.9921875 * 2^k (m = 255) and one 1.0078125 * 2^(k - span) (m = 129, an odd
    # significand): the exact sum, 63 * 255 * 2^span + 129 units, needs 54 bits at span 40, so the
    # running fp64 sum drops the small value's last bit; at span 39 it needs 53 and is kept
    big = 1.9921875 * 2.0 ** k
    for span, exact in ((SPAN, True), (SPAN + 1, False)):
        small = 1.0078125 * 2.0 ** (k - span)
        vals = np.array([big] * 63 + [small])
        f32 = vals.astype(np.float32)
        assert np.array_equal(f32.astype(np.float64), vals) and not np.any(f32.view(np.uint32) & 0xFFFF)  # bf16 values
        bits = (f32.view(np.uint32) >> 16).astype(np.uint16)
        assert _pos(int(bits[0])) - _pos(int(bits[-1])) == span
        run = 0.0
        for x in vals:
            run += float(x)
        assert (Fraction(run) == _exact(vals)) is exact, span
