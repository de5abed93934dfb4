"""The multi-GPU partition of one layer call (sparse_memory_linear_pkm_b200/shard.py),
on CPU with two gloo ranks.

Each rank runs its share with the oracle standing in for the CUDA library
(test-side compute only), takes the real collective step (the all-reduce of
the rows' sums of squares in the column split with the epilogue), and the
assembled outputs must equal one unsharded oracle call: y and M_T of the rows
and heads splits exactly (the same per-(b, h) arithmetic), and of the column
split within 1e-12 relative (the mean of squares is summed in another order).
"""

import multiprocessing as mp
import os
import socket
import sys
from pathlib import Path

import numpy as np
import pytest

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))

from sparse_memory_linear_pkm_b200.shard import (Partition, layer_forward_sharded, place_outputs,  # noqa: E402
                                                 plan_partition, shard_inputs)

EPS = 1e-6


def _inputs(B, T, H, sqrt_n, d_v, seed, gate):
    rng = np.random.default_rng(seed)
    f = np.float32
    d = dict(kp=rng.standard_normal((B, T, H, 2 * sqrt_n)).astype(f), qp=rng.standard_normal((B, T, H, 2 * sqrt_n)).astype(f),
             v=rng.standard_normal((B, T, H, d_v)).astype(f),
             alpha=np.exp(-np.log1p(np.exp(rng.standard_normal((B, T, H))))).astype(f),
             beta=rng.uniform(0, 1, (B, T, H)).astype(f),
             M0=(0.02 * rng.standard_normal((H, sqrt_n * sqrt_n, d_v))).astype(f))
    d["g"] = rng.standard_normal((B, T, H, d_v)).astype(f) if gate else None
    return d


class OracleOps:
    """A rank's compute by the oracle (numpy in, numpy out)."""

    def __init__(self, oracle):
        self.o = oracle

    def layer_forward(self, kp, qp, v, alpha, beta, M0, W, R, g=None, eps=EPS):
        c = np.ascontiguousarray
        out = self.o.layer_forward(c(kp), c(qp), c(v), c(alpha), c(beta), c(M0), W, R,
                                   g=None if g is None else c(g), eps=eps)
        return out["y"], out["M_T"].astype(np.float64)

    def row_sumsq(self, y):
        return np.sum(y * y, axis=-1)

    def rmsnorm_gate_rows(self, y, g, ss, d_total, eps):
        return g * y / np.sqrt(ss / d_total + eps)[..., None]


def _worker(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank))
    import datetime

    import torch
    import torch.distributed as dist

    import oracle as oracle_pkg

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        B, T, H, sqrt_n, d_v, W, R, gate, col_align = case
        inp = _inputs(B, T, H, sqrt_n, d_v, seed=11, gate=gate)
        part = plan_partition(B, H, d_v, world, col_align)
        loc = shard_inputs(part, rank, inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], inp["M0"], inp["g"])
        calls = []

        def all_reduce(ss):
            calls.append(ss.shape)
            t = torch.from_numpy(np.ascontiguousarray(ss, dtype=np.float64))
            dist.all_reduce(t, op=dist.ReduceOp.SUM)
            return t.numpy()

        y, M_T = layer_forward_sharded(part, rank, loc["kp"], loc["qp"], loc["v"], loc["alpha"], loc["beta"],
                                       loc["M0"], W, R, g=loc.get("g"), eps=EPS,
                                       ops=OracleOps(oracle_pkg.get()), all_reduce=all_reduce)
        q.put((rank, part.mode, y, M_T, calls))
    finally:
        dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASES = {
    # B, T, H, sqrt_n, d_v, W, R, epilogue, column alignment
    "rows": (2, 9, 1, 8, 32, 5, 3, True, 16),
    "heads": (1, 9, 2, 8, 32, 5, 3, True, 16),
    "columns_epilogue": (1, 11, 1, 8, 64, 6, 4, True, 16),
    "columns_no_epilogue": (1, 11, 1, 8, 64, 6, 4, False, 32),
}


@pytest.mark.parametrize("name", list(CASES))
def test_two_ranks_equal_one_call(oracle, name):
    case = CASES[name]
    B, T, H, sqrt_n, d_v, W, R, gate, col_align = case
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, case, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted((q.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    mode = out[0][1]
    assert mode == name.split("_")[0]
    inp = _inputs(B, T, H, sqrt_n, d_v, seed=11, gate=gate)
    ref = oracle.layer_forward(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], inp["M0"], W, R, g=inp["g"],
                               eps=EPS)
    part = plan_partition(B, H, d_v, 2, col_align)
    y = np.full((B, T, H, d_v), np.nan)
    M_T = np.full((B, H, sqrt_n * sqrt_n, d_v), np.nan)
    for rank, _, y_loc, M_loc, calls in out:
        place_outputs(part, rank, y, M_T, y_loc, M_loc)
        # the column split with the epilogue takes exactly one collective step: B*T*H sums
        assert calls == ([(B, T, H)] if part.needs_all_reduce and gate else [])
    assert not np.isnan(y).any() and not np.isnan(M_T).any()
    if mode == "columns" and gate:
        np.testing.assert_allclose(y, ref["y"], rtol=1e-12, atol=1e-15)
    else:
        assert np.array_equal(y, ref["y"])
    assert np.array_equal(M_T, ref["M_T"].astype(np.float64))


def test_plan_partition():
    assert plan_partition(8, 16, 128, 4).mode == "rows"
    assert plan_partition(1, 8, 512, 4).mode == "heads"
    p = plan_partition(1, 2, 2048, 8)
    assert p.mode == "columns" and p.needs_all_reduce
    # the long-context workload over 8 GPUs: 256 columns each, whole 128-byte bf16 segments
    assert [p.ranges(r)[4:] for r in range(8)] == [(256 * r, 256 * (r + 1)) for r in range(8)]
    # uneven batch rows: contiguous, covering every row once
    p = plan_partition(5, 1, 64, 2)
    assert [p.ranges(r)[:2] for r in range(2)] == [(0, 2), (2, 5)]
    assert not plan_partition(8, 1, 64, 1).needs_all_reduce
    with pytest.raises(ValueError):
        plan_partition(1, 1, 96, 2)  # 96 columns do not split into two multiples of 64
    with pytest.raises(ValueError):
        Partition("rows", 2, 2, 1, 64).ranges(2)
