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


def test_reference_arm_prints_one_contract_line():
    """bench.py --impl reference (the oracle on the host cores) prints one JSON
    line with the contract's keys, on the bench workload's config."""
    import json
    import subprocess

    out = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--impl", "reference", "--steps", "1", "--warmup",
                          "1", "--cpu-seconds", "0.5", "--workload", "d2048_h16_n1024_dv128"], capture_output=True,
                         text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["config"]["workload"] == "d2048_h16_n1024_dv128"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
