"""Multi-rank host logic of bench.py on CPU ranks (gloo, world size 2).

The attention path shards into independent problems (layers, sequences), so
the only cross-rank steps are the barrier around the timed region and the
max-over-ranks of the step time.  These tests run that logic on two CPU
processes, and check that a rank that leaves early makes the other rank's
next collective fail with an error instead of hanging.
"""

import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=timeout_s))


def _worker_max(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    import bench

    _init(rank, world, port, 30)
    try:
        bench.barrier(world)
        m = bench.max_over_ranks(10.0 + rank, world)
        shards = bench.shard_units(48, rank, world)
        q.put((rank, m, shards, bench.rank_layer(rank)))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_sharding():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker_max, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(world))
    assert [o[1] for o in out] == [11.0, 11.0]  # max over ranks, seen by every rank
    all_units = sorted(u for o in out for u in o[2])
    assert all_units == list(range(48))  # every unit exactly once
    assert out[0][3] != out[1][3]  # each rank times its own layer


def test_shard_units_uneven():
    import sys

    sys.path.insert(0, ROOT)
    import bench

    for n in (1, 5, 48, 49):
        for world in (1, 2, 3, 8):
            parts = [bench.shard_units(n, r, world) for r in range(world)]
            assert sorted(u for p in parts for u in p) == list(range(n))
            assert max(map(len, parts)) - min(map(len, parts)) <= 1


def _put_and_exit(q, item):
    q.put(item)
    q.close()
    q.join_thread()  # flush before the hard exit
    os._exit(0)


def _worker_leaves(rank, world, port, q):
    _init(rank, world, port, 5)
    if rank == 1:
        _put_and_exit(q, (rank, "left"))  # leaves between steps, without joining the barrier
    try:
        dist.barrier()
        msg = "no error"
    except Exception as e:  # the timeout (or the peer's exit) surfaces as an error
        msg = "error: " + type(e).__name__
    _put_and_exit(q, (rank, msg))


def test_rank_leaving_early_fails_the_barrier_instead_of_hanging():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker_leaves, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode is not None, "a rank hung"
    res = dict(q.get(timeout=10) for _ in range(world))
    assert res[1] == "left"
    assert res[0].startswith("error"), res[0]
