"""Multi-rank plumbing of the benchmark on CPU (gloo, world size 2).

Each rank runs the whole workload (independent replicas, weak scaling); the only
cross-rank step is the max over ranks of the timed duration.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = [12.5, 30.0][rank]
        got = bench.max_over_ranks(ms, torch.device("cpu"))
        rate = bench.weak_scaling_rate(1.0e12, 10, world, got)
        q.put((rank, got, rate))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_rate_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, got, rate in res:
        assert got == 30.0
        assert rate == pytest.approx(1.0e12 * 10 * 2 / 0.030)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(7.0, torch.device("cpu")) == 7.0
    assert bench.weak_scaling_rate(2.0, 3, 1, 1000.0) == pytest.approx(6.0)
