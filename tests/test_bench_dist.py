"""The benchmark's multi-rank plumbing on CPU: two gloo ranks agree on the
slowest rank's time, and the whole-job value counts every rank's units over
that time (weak scaling, no collective on the data path)."""

import multiprocessing as mp
import os
import socket
import sys
from pathlib import Path

import torch

ROOT = Path(__file__).resolve().parents[1]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, times, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, str(ROOT))
    import bench

    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    slowest = d.max(times[rank], torch.device("cpu"))
    value = bench.aggregate_value(1000.0, d.world, slowest)
    d.barrier()
    d.close()
    q.put((rank, slowest, value))


def test_two_gloo_ranks_take_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    times = [0.5, 2.0]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _, _ in out] == [0, 1]
    for _, slowest, value in out:
        assert slowest == 2.0
        assert value == 1000.0 * 2 / 2.0


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, str(ROOT))
    import bench

    d = bench.Dist()
    assert d.world == int(os.environ.get("WORLD_SIZE", "1"))
    if d.world == 1:
        d.init("gloo")
        assert not d.pg
        assert d.max(3.25, torch.device("cpu")) == 3.25
        assert bench.aggregate_value(10.0, 1, 2.0) == 5.0
