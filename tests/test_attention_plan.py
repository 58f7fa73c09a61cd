"""Host logic of the attention launch (no GPU): the work split into two-tile and one-tile CTAs
covers every query tile of every (b, h) exactly once, through the same mapping function the
kernel runs (nvfp4kv_attention_plan with an explicit SM count never touches a device)."""
import ctypes

import pytest

import nvfp4_quantised_kv_b200 as nk
from tests.test_abi import _desc


def _plan(L, d, lq, sms, cta):
    out = (ctypes.c_int32 * 4)()
    rc = L.nvfp4kv_attention_plan(ctypes.byref(d), lq, sms, cta, out)
    return rc, list(out)


@pytest.fixture(scope="module")
def L():
    return nk.lib()


SHAPES = [(64, 1, 2), (4680, 1, 12), (2640, 1, 24), (880, 1, 24), (300, 2, 3), (130, 1, 2), (1, 1, 1),
          (256, 1, 2), (200, 1, 148), (38400, 1, 1), (5000, 4, 16), (257, 1, 7), (4680, 3, 5)]


@pytest.mark.parametrize("lq,batch,heads", SHAPES)
@pytest.mark.parametrize("sms", [148, 132, 8, 1])
def test_every_query_tile_is_covered_once(L, lq, batch, heads, sms):
    d = _desc(batch=batch, heads=heads)
    rc, out = _plan(L, d, lq, sms, -1)
    assert rc == nk.OK
    n_ctas = out[0]
    n_qt = -(-lq // 128)
    seen = set()
    for c in range(n_ctas):
        rc, (_, bh, row0, nq) = _plan(L, d, lq, sms, c)
        assert rc == nk.OK
        assert 0 <= bh < batch * heads and nq in (1, 2) and row0 % 128 == 0
        for t in range(row0 // 128, row0 // 128 + nq):
            assert 0 <= t < n_qt
            assert (bh, t) not in seen
            seen.add((bh, t))
    assert len(seen) == batch * heads * n_qt
    # two-tile CTAs come first, so the longest work items start in the first wave
    nqs = [_plan(L, d, lq, sms, c)[1][3] for c in range(n_ctas)]
    assert nqs == sorted(nqs, reverse=True)


def test_the_1p3b_layer_splits_into_one_wave_of_pairs_and_one_of_singles(L):
    d = _desc(batch=1, heads=12)
    _, out = _plan(L, d, 4680, 148, -1)
    assert out[0] == 296
    assert sum(_plan(L, d, 4680, 148, c)[1][3] == 2 for c in range(296)) == 148


def test_plan_argument_checks(L):
    d = _desc()
    assert _plan(L, d, 0, 148, -1)[0] == nk.ERR_INVALID_ARG
    assert _plan(L, d, 64, 148, 99)[0] == nk.ERR_INVALID_ARG
    assert L.nvfp4kv_attention_plan(ctypes.byref(d), 64, 148, -1, None) == nk.ERR_INVALID_ARG
    assert L.nvfp4kv_attention_plan(None, 64, 148, -1, (ctypes.c_int32 * 4)()) == nk.ERR_INVALID_ARG


@pytest.mark.parametrize("lq,heads,pairs", [(4680, 12, 148), (2640, 24, 240), (880, 24, 72)])
def test_benchmarked_shapes_plan_as_documented(L, lq, heads, pairs):
    d = _desc(batch=1, heads=heads)
    n = _plan(L, d, lq, 148, -1)[1][0]
    assert sum(_plan(L, d, lq, 148, c)[1][3] == 2 for c in range(n)) == pairs


def test_planning_a_very_large_launch_is_cheap(L):
    import time
    d = _desc(batch=64, heads=64)
    t0 = time.perf_counter()
    rc, out = _plan(L, d, 16384 + 77, 148, -1)  # 64*64 heads x 129 query tiles
    assert rc == nk.OK and out[0] > 0
    assert time.perf_counter() - t0 < 0.5
