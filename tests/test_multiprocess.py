"""Multi-rank host logic of the benchmark under gloo, world size 2, on CPU:
replicas time independently; the job's time is the slowest rank's and the
job's value counts every rank's work."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    local_ms = 10.0 + 2.0 * rank
    ms = bench.max_over_ranks(local_ms, world)
    value = bench.job_value(1e12, ms, world)
    bench.barrier(world)
    out.put((rank, ms, value))
    dist.destroy_process_group()


def test_two_rank_aggregation_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in res:
        assert ms == pytest.approx(12.0)
        assert value == pytest.approx(2 * 1e12 / 12e-3 / 1e12)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_value(2e12, 4.0, 1) == pytest.approx(500.0)
