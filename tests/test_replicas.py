"""The multi-GPU plumbing of bench.py on CPU: two gloo ranks (the path has no exchange step, so
`bench.py --gpus N` runs N replicas; only the timing reduction crosses ranks)."""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 0.25 * rank], torch.device("cpu"))
        out.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_timings_reduce_to_the_slowest_rank_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    env_root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    os.environ.setdefault("PYTHONPATH", env_root)
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results[0] == results[1] == [2.0, 5.0, 0.25]


def test_single_process_reduction_is_the_identity():
    import torch
    import bench
    assert bench.max_over_ranks([3.0, 1.5], torch.device("cpu")) == [3.0, 1.5]


@pytest.mark.parametrize("world", [1, 2, 8])
def test_whole_job_rate_counts_every_rank(world):
    import bench
    # each rank processes 1e12 FLOP per step; the slowest rank takes 2 ms
    assert bench.whole_job_rate(1e12, world, 2.0) == pytest.approx(world * 5e14)


def test_replicas_draw_distinct_inputs():
    import bench
    seeds = {bench.replica_seed(1, s, r) for s in range(4) for r in range(8)}
    assert len(seeds) == 32
