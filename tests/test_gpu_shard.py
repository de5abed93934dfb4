"""The column split of one layer call (shard.py) through the C ABI on one GPU:
the ranks' shares run as independent calls one after another (nothing waits
on anything else), their rows' sums of squares are added as the all-reduce
would, and the assembled outputs match the unsharded call and the oracle."""

import numpy as np
import pytest
import torch

from parity_helpers import assert_rel_close, f32, tol_for
from sparse_memory_linear_pkm_b200 import shard, synth

pytestmark = pytest.mark.gpu


def test_row_sumsq_and_slice_epilogue_match_oracle(sdm, oracle, cuda_device):
    gen = torch.Generator().manual_seed(3)
    y = torch.randn((37, 96), generator=gen)
    g = torch.randn((37, 96), generator=gen).to(torch.bfloat16)
    ss = sdm.row_sumsq(y.to(cuda_device))
    sdm.stream_check()
    np.testing.assert_allclose(ss.cpu().numpy(), (y.double() ** 2).sum(-1).numpy(), rtol=1e-6)
    want = oracle.rmsnorm_gate(f32(y), f32(g))
    halves = []
    for c0, c1 in ((0, 32), (32, 96)):  # a 32 + 64 column split of the rows
        yh = y[:, c0:c1].contiguous().to(cuda_device)
        sdm.rmsnorm_gate_rows(yh, g[:, c0:c1].contiguous().to(cuda_device), ss, 96)
        halves.append(yh.cpu())
    sdm.stream_check()
    assert_rel_close(torch.cat(halves, 1).numpy(), want, 1e-5, "epilogue on column slices")


@pytest.mark.parametrize("world", [2, 4])
def test_column_split_equals_one_call(sdm, oracle, cuda_device, world):
    shape = synth.WORKLOADS["long_t1m_n262144_dv2048"].replace(B=1, T=40, H=1, sqrt_n=32, d_v=512)
    inp = synth.make_inputs(shape, seed=5, device=cuda_device, with_gate=True)
    part = shard.plan_partition(shape.B, shape.H, shape.d_v, world)
    assert part.mode == "columns" and part.needs_all_reduce
    y_full, M_full = sdm.layer_forward(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], inp["M0"], shape.W,
                                       shape.R, g=inp["g"])
    ops = shard.CudaOps()
    parts, ss = [], None
    for rank in range(world):  # each rank's call up to its collective step
        loc = {k: t.contiguous() for k, t in shard.shard_inputs(part, rank, inp["kp"], inp["qp"], inp["v"], inp["alpha"],
                                                                inp["beta"], inp["M0"], inp["g"]).items()}
        y, M_T = ops.layer_forward(loc["kp"], loc["qp"], loc["v"], loc["alpha"], loc["beta"], loc["M0"], shape.W,
                                   shape.R)
        s = ops.row_sumsq(y)
        ss = s if ss is None else ss + s
        parts.append((loc, y, M_T))
    y_all = torch.empty_like(y_full)
    M_all = torch.empty_like(M_full)
    for rank, (loc, y, M_T) in enumerate(parts):  # after the all-reduce
        ops.rmsnorm_gate_rows(y, loc["g"], ss, shape.d_v, 1e-6)
        shard.place_outputs(part, rank, y_all, M_all, y, M_T)
    sdm.stream_check()
    # the state columns evolve alone: bit for bit; y differs from one call only in summation order
    assert torch.equal(M_all, M_full)
    assert_rel_close(y_all.cpu().numpy(), y_full.cpu().numpy(), 1e-5, "y (column split vs one call)")
    ref = oracle.layer_forward(f32(inp["kp"]), f32(inp["qp"]), f32(inp["v"]), f32(inp["alpha"]), f32(inp["beta"]),
                               f32(inp["M0"]), shape.W, shape.R, g=f32(inp["g"]), state_bf16=True)
    assert_rel_close(y_all.cpu().numpy(), ref["y"], tol_for(shape.state_dtype), "y (column split vs oracle)")
