"""Multi-rank paths on CPU (gloo).

The benchmark's headline runs one independent sequence per rank (weak
scaling); its decode batch is split by sequence and its 128K block by kv head
(global_gqa_b200/shard.py).  These tests run real gloo ranks: every rank
computes its own share, the shares are gathered, and together they must cover
every (sequence, kv head) unit of the workload exactly once; the timed
duration is the maximum over ranks.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import inputs
from global_gqa_b200 import shard


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _run(world, target):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    return sorted(q.get(timeout=10) for _ in range(world))


def _init(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))


def _timing_worker(rank, world, port, q):
    _init(rank, world, port)
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
    res = _run(2, _timing_worker)
    for rank, got, rate in res:
        assert got == 30.0
        assert rate == pytest.approx(1.0e12 * 10 * 2 / 0.030)


def _cover_worker(rank, world, port, q):
    _init(rank, world, port)
    try:
        dec, lng = inputs.DECODE_B64, inputs.LONG_128K
        mine = {
            "decode": shard.rank_units(dec.B, dec.Hkv, world, rank, "sequence"),
            "long": shard.rank_units(lng.B, lng.Hkv, world, rank, "kv_head"),
        }
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        q.put((rank, gathered))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 8])
def test_shards_cover_every_unit_once_gloo(world):
    """The 64-sequence decode split by sequence and the 128K block split by kv
    head (16 kv heads) over 2, 3 and 8 gloo ranks."""
    dec, lng = inputs.DECODE_B64, inputs.LONG_128K
    res = _run(world, _cover_worker)
    for rank, gathered in res:
        assert gathered == res[0][1]                 # every rank sees the same assignment
        for key, B, Hkv in (("decode", dec.B, dec.Hkv), ("long", lng.B, lng.Hkv)):
            units = [u for g in gathered for u in g[key]]
            assert len(units) == len(set(units)) == B * Hkv
            assert set(units) == {(b, h) for b in range(B) for h in range(Hkv)}
            sizes = [len(g[key]) for g in gathered]
            assert max(sizes) - min(sizes) <= max(B, Hkv)  # balanced to one sequence or one kv head


def test_split_is_contiguous_and_balanced():
    for n in (0, 1, 7, 16, 64):
        for world in (1, 2, 3, 8):
            ranges = [shard.split(n, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [e - s for s, e in ranges]
            assert max(sizes) - min(sizes) <= 1
    assert shard.kv_head_shard(16, 2, 3, 0) == {"kv": (0, 6), "q": (0, 12)}
    assert shard.kv_head_shard(16, 2, 3, 2) == {"kv": (11, 16), "q": (22, 32)}
    with pytest.raises(ValueError):
        shard.split(4, 2, 2)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(7.0, torch.device("cpu")) == 7.0
    assert bench.weak_scaling_rate(2.0, 3, 1, 1000.0) == pytest.approx(6.0)
