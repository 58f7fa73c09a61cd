"""Failure detection without a GPU fault: a kernel whose bounded wait is made to run out (nothing
arrives at its barrier) reports NVFP4KV_ERR_DEVICE_TIMEOUT through the cache's status word, the
read clears it, and the same context then runs the hot path normally."""
import time

import numpy as np
import pytest

import nvfp4_quantised_kv_b200 as nk
import oracle
from nvfp4_quantised_kv_b200 import synthetic
from tests.gpu_util import assert_attention_close, dev_bf16, gather_rows, make_caches

pytestmark = pytest.mark.gpu


def test_a_wait_that_runs_out_sets_the_timeout_bit_and_the_context_stays_usable():
    w = synthetic.WORKLOADS["tiny"]
    cache, ocache = make_caches(w, w.visible_chunks)
    assert cache.read_status() == 0
    t0 = time.perf_counter()
    cache.debug_wait_timeout()
    status = cache.read_status()  # waits for the stream
    waited = time.perf_counter() - t0
    assert status == 1 << nk.ERR_DEVICE_TIMEOUT
    assert 0.5 < waited < 30.0   # the kernels' wait limit is one second
    assert cache.read_status() == 0  # reading cleared it
    qb = synthetic.queries(w)
    out = cache.attention(dev_bf16(qb), w.q_chunk, w.n_sink, w.window)
    assert cache.read_status() == 0
    rows = np.array([(b, h, i) for b in range(w.batch) for h in range(w.heads)
                     for i in range(w.q_tokens)], np.int32)
    want = oracle.attention_rows(qb, ocache, w.q_chunk, w.n_sink, w.window, rows)
    assert_attention_close(gather_rows(out.cpu().numpy(), rows), want, "after the timeout")
