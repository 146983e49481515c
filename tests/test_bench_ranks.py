"""Host logic of the multi-rank bench: timings reduce to the slowest rank, and the whole-job rate
counts the work of every rank (independent replicas, weak scaling).  Two gloo ranks on CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        # rank r reports timings (1 + r, 10 - r, 5): the reduction must give (world, 10, 5) everywhere
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 5.0], world, "cpu")
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_max_over_ranks_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert res[r] == [float(world), 10.0, 5.0]


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks([3.0, 1.5], 1, "cpu") == [3.0, 1.5]


def test_job_rate_weak_scaling():
    # 2e12 flop per rank in 10 ms: 200 TFLOP/s per rank; N ranks at the same time give N times that
    assert bench.job_rate(1, 2e12, 10.0) == pytest.approx(2e14)
    assert bench.job_rate(8, 2e12, 10.0) == pytest.approx(1.6e15)
    # the slowest rank sets the time: doubling it halves the rate
    assert bench.job_rate(4, 2e12, 20.0) == pytest.approx(bench.job_rate(4, 2e12, 10.0) / 2)
