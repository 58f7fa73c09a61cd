"""Host logic of the attention launch (no GPU): the persistent CTAs' ranges of (work item, KV tile)
units cover every query tile of every (b, h) against every KV tile exactly once, through the same
mapping functions the kernels run (nvfp4kv_attention_plan with an explicit SM count never touches
a device); the ranges have near-equal weighted cost; split items get distinct partial slots."""
import ctypes

import pytest

import nvfp4_quantised_kv_b200 as nk
from tests.test_abi import _desc

W_PAIR, W_SINGLE = 9, 7  # the planner's relative cost of a KV tile of a two-tile / one-tile item


def _plan(L, d, lq, nt, sms, cta=-1, seg=-1):
    out = (ctypes.c_int32 * 8)()
    rc = L.nvfp4kv_attention_plan(ctypes.byref(d), lq, nt, sms, cta, seg, out)
    return rc, list(out)


@pytest.fixture(scope="module")
def L():
    return nk.lib()


def _segments(L, d, lq, nt, sms):
    rc, out = _plan(L, d, lq, nt, sms)
    assert rc == nk.OK
    g = out[0]
    segs = []
    for c in range(g):
        rc, o = _plan(L, d, lq, nt, sms, c)
        assert rc == nk.OK
        for k in range(o[1]):
            rc, o2 = _plan(L, d, lq, nt, sms, c, k)
            assert rc == nk.OK
            segs.append((c, k, o2[2], o2[3], o2[4], o2[5], o2[6], o2[7]))
    return out, segs


SHAPES = [(64, 1, 2, 2), (4680, 1, 12, 147), (2640, 1, 24, 145), (880, 1, 24, 145), (4680, 1, 12, 293),
          (300, 2, 3, 6), (130, 1, 2, 120), (1, 1, 1, 2), (256, 1, 2, 3), (200, 1, 148, 2),
          (38400, 1, 1, 9), (5000, 4, 16, 40), (257, 1, 7, 1)]


@pytest.mark.parametrize("lq,batch,heads,nt", SHAPES)
@pytest.mark.parametrize("sms", [148, 132, 8, 1])
def test_every_unit_is_covered_once_with_balanced_ranges(L, lq, batch, heads, nt, sms):
    d = _desc(batch=batch, heads=heads)
    head, segs = _segments(L, d, lq, nt, sms)
    n_ctas, launches = head[0], head[1]
    n_qt = -(-lq // 128)
    seen = set()
    cost = [0] * n_ctas
    slots = {}
    for c, k, bh, row0, nq, t0, t1, slot in segs:
        assert 0 <= bh < batch * heads and row0 % 256 == 0 and nq in (1, 2)
        assert nq == min(2, n_qt - row0 // 128)
        assert 0 <= t0 < t1 <= nt
        full = t0 == 0 and t1 == nt
        assert (slot == -1) == full
        if not full:
            # only a CTA's first and last segments can be partial; slot 2c for the first
            assert slot in (2 * c, 2 * c + 1)
            assert slot == 2 * c if k == 0 else slot == 2 * c + 1
            assert slot not in slots
            slots[slot] = (bh, row0)
        for q in range(nq):
            for t in range(t0, t1):
                key = (bh, row0 // 128 + q, t)
                assert key not in seen
                seen.add(key)
        cost[c] += (t1 - t0) * (W_PAIR if nq == 2 else W_SINGLE)
    assert len(seen) == batch * heads * n_qt * nt
    # CTA c starts at the first unit at or after weighted position floor(W c / G), so every range
    # is within one unit's weight of W / G
    assert max(cost) - min(cost) <= 2 * W_PAIR
    assert launches == (2 if slots else 1)
    # every split item has at least two parts
    parts = {}
    for bh, row0 in slots.values():
        parts[(bh, row0)] = parts.get((bh, row0), 0) + 1
    assert all(n >= 2 for n in parts.values())


def test_benchmarked_shapes_fill_every_sm(L):
    for lq, heads, nt in [(4680, 12, 147), (2640, 24, 145), (880, 24, 145), (4680, 12, 293)]:
        _, out = _plan(L, _desc(batch=1, heads=heads), lq, nt, 148)
        assert out[0] == 148


def test_plan_argument_checks(L):
    d = _desc()
    assert _plan(L, d, 0, 2, 148)[0] == nk.ERR_INVALID_ARG
    assert _plan(L, d, 64, 0, 148)[0] == nk.ERR_INVALID_ARG
    assert _plan(L, d, 64, 2, 148, 99)[0] == nk.ERR_INVALID_ARG
    assert _plan(L, d, 64, 2, 148, 0, 5)[0] == nk.ERR_INVALID_ARG
    assert L.nvfp4kv_attention_plan(ctypes.byref(d), 64, 2, 148, -1, -1, None) == nk.ERR_INVALID_ARG
    assert L.nvfp4kv_attention_plan(None, 64, 2, 148, -1, -1, (ctypes.c_int32 * 8)()) == nk.ERR_INVALID_ARG
    # more (item, KV tile) units than the planner's 64-bit weighted arithmetic takes
    big = _desc(batch=65535, heads=65535)
    assert _plan(L, big, 1 << 24, (1 << 24) - 1, 148)[0] == nk.ERR_UNSUPPORTED


def test_planning_a_very_large_launch_is_cheap(L):
    import time
    d = _desc(batch=64, heads=64)
    t0 = time.perf_counter()
    rc, out = _plan(L, d, 16384 + 77, 300, 148)  # 64*64 heads x 65 items x 300 KV tiles
    assert rc == nk.OK and out[0] == 148
    for c in (0, 77, 147):
        assert _plan(L, d, 16384 + 77, 300, 148, c)[0] == nk.OK
    assert time.perf_counter() - t0 < 0.5
