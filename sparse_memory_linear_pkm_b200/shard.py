"""One layer call spread over the GPUs of a node, one process per GPU.

Every (b, h) sequence of the recurrence is independent, and within one (b, h)
every column of d_v evolves on its own given the per-token scalars (the
selection weights, alpha and beta): the write of SDM explainer section 3.1
step 2 and the read of step 3 act column by column. Only the optional RMS-norm
epilogue of step 3 couples the columns of a row, through the row's mean of
squares. So a call splits over ranks in one of three ways, each the natural
shard of a parallel layout upstream:

  rows     contiguous batch rows per rank (data parallel); no collective.
  heads    contiguous heads per rank (head parallel, the projections produce
           k', q', v per head); no collective.
  columns  contiguous d_v column slices per rank (the v projection is column
           parallel), with k', q', alpha and beta replicated, so every rank
           selects the same slots, and the state M0 / M_T and g sharded by
           columns; with the epilogue, one all-reduce of each row's sum of
           squares (B*T*H floats) per call.

`plan_partition` picks rows when there are at least as many batch rows as
ranks, else heads, else columns (the long-context workload: B*H = 2). The
functions here only slice and combine; every step of a rank's share runs in
the CUDA library (or in whatever `ops` the caller passes).
"""

from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class Partition:
    """How one call of shape (B, T, H, ..., d_v) is split over `world` ranks."""

    mode: str  # "rows", "heads" or "columns"
    world: int
    B: int
    H: int
    d_v: int
    col_align: int = 64

    def bounds(self, rank: int, n: int, align: int = 1):
        """[lo, hi) of rank's contiguous share of n items (multiples of align)."""
        units = n // align
        lo = units * rank // self.world
        hi = units * (rank + 1) // self.world
        return lo * align, hi * align

    def ranges(self, rank: int):
        """(b0, b1, h0, h1, c0, c1): the batch rows, heads and columns rank owns."""
        if not 0 <= rank < self.world:
            raise ValueError(f"rank {rank} outside [0, {self.world})")
        b0, b1, h0, h1, c0, c1 = 0, self.B, 0, self.H, 0, self.d_v
        if self.mode == "rows":
            b0, b1 = self.bounds(rank, self.B)
        elif self.mode == "heads":
            h0, h1 = self.bounds(rank, self.H)
        else:
            c0, c1 = self.bounds(rank, self.d_v, self.col_align)
        return b0, b1, h0, h1, c0, c1

    @property
    def needs_all_reduce(self) -> bool:
        """Whether the epilogue needs the cross-rank sum of squares."""
        return self.mode == "columns" and self.world > 1


def plan_partition(B: int, H: int, d_v: int, world: int, col_align: int = 64) -> Partition:
    """Rows when B >= world, else heads when H >= world, else d_v columns in
    slices that are multiples of col_align (so each rank's slice still fills
    whole 128-byte row segments of the state)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    if B >= world:
        return Partition("rows", world, B, H, d_v, col_align)
    if H >= world:
        return Partition("heads", world, B, H, d_v, col_align)
    if d_v % col_align or d_v // col_align < world:
        raise ValueError(f"cannot split d_v = {d_v} into {world} slices of multiples of {col_align} columns")
    return Partition("columns", world, B, H, d_v, col_align)


def shard_inputs(part: Partition, rank: int, kp, qp, v, alpha, beta, M0, g=None) -> dict:
    """Rank's share of global inputs (kp, qp [B,T,H,2 sqrt_n]; v, g [B,T,H,d_v];
    alpha, beta [B,T,H]; M0 [H,N,d_v]). Works on numpy arrays and torch
    tensors; the caller makes the slices contiguous where it needs to."""
    b0, b1, h0, h1, c0, c1 = part.ranges(rank)
    out = {"kp": kp[b0:b1, :, h0:h1], "qp": qp[b0:b1, :, h0:h1], "alpha": alpha[b0:b1, :, h0:h1],
           "beta": beta[b0:b1, :, h0:h1], "v": v[b0:b1, :, h0:h1, c0:c1], "M0": M0[h0:h1, :, c0:c1]}
    if g is not None:
        out["g"] = g[b0:b1, :, h0:h1, c0:c1]
    return out


def place_outputs(part: Partition, rank: int, y_global, M_T_global, y_local, M_T_local) -> None:
    """Writes rank's outputs (y [B',T,H',d'], M_T [B',H',N,d']) into the global
    arrays (y [B,T,H,d_v], M_T [B,H,N,d_v])."""
    b0, b1, h0, h1, c0, c1 = part.ranges(rank)
    y_global[b0:b1, :, h0:h1, c0:c1] = y_local
    M_T_global[b0:b1, h0:h1, :, c0:c1] = M_T_local


class CudaOps:
    """A rank's compute through the CUDA library (C ABI)."""

    def __init__(self, **layer_kw):
        self.layer_kw = layer_kw

    def layer_forward(self, kp, qp, v, alpha, beta, M0, W, R, g=None, eps=1e-6):
        from . import layer_forward

        return layer_forward(kp, qp, v, alpha, beta, M0, W, R, g=g, eps=eps, **self.layer_kw)

    def row_sumsq(self, y):
        from . import row_sumsq

        return row_sumsq(y)

    def rmsnorm_gate_rows(self, y, g, ss, d_total, eps):
        from . import rmsnorm_gate_rows

        return rmsnorm_gate_rows(y, g, ss, d_total, eps)


def all_reduce_sum(ss, group=None):
    """In-place sum of ss over the ranks of the process group (NCCL for CUDA
    tensors, gloo for CPU ones)."""
    import torch.distributed as dist

    dist.all_reduce(ss, op=dist.ReduceOp.SUM, group=group)
    return ss


def layer_forward_sharded(part: Partition, rank: int, kp, qp, v, alpha, beta, M0, W: int, R: int, g=None,
                          eps: float = 1e-6, ops=None, all_reduce=None):
    """Runs rank's share of one layer call on its input shard (see
    shard_inputs) and returns its (y, M_T) shard. Every rank calls this
    once per layer call, in the same order (the column mode with the epilogue
    takes one collective step: the all-reduce of the rows' sums of squares)."""
    ops = ops if ops is not None else CudaOps()
    all_reduce = all_reduce if all_reduce is not None else all_reduce_sum
    if not part.needs_all_reduce or g is None:
        return ops.layer_forward(kp, qp, v, alpha, beta, M0, W, R, g=g, eps=eps)
    y, M_T = ops.layer_forward(kp, qp, v, alpha, beta, M0, W, R, g=None, eps=eps)
    ss = ops.row_sumsq(y)
    ss = all_reduce(ss)
    y = ops.rmsnorm_gate_rows(y, g, ss, part.d_v, eps)
    return y, M_T
