"""Seeded synthetic inputs for the SDM recurrent core.

This module is shared by the tests, the benchmark and the oracle checks. It
holds only shapes and random-number recipes -- none of the method's
arithmetic. Every tensor has its own generator stream derived from
(seed, tensor id), so a slice of one tensor never depends on another's size.

Workloads (isoFLOP sizing of the SDM explainer, section 3.2: d_qk_total = d/2
split over H heads gives 2*sqrtN per head, d_v_total = d gives d_v per head;
W = R = d_qk of the dense baseline = 64). Value recipes for every workload:
scores of keys and queries i.i.d. N(0,1); v ~ N(0,1); alpha = exp(-softplus(z))
with z ~ N(0,1); beta ~ U(0,1); M0 ~ N(0, 0.02^2); gate g ~ N(0,1) when the
epilogue runs. Values are rounded to the input/state dtype after drawing.
"""

from __future__ import annotations

import dataclasses

import torch

F32 = "f32"
BF16 = "bf16"
_TORCH_DTYPE = {F32: torch.float32, BF16: torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Shape:
    """One SDM layer call: B batch rows, T tokens, H heads, N = sqrt_n^2 slots
    of d_v columns per head, W write and R read slots per token-head."""

    name: str
    B: int
    T: int
    H: int
    sqrt_n: int
    d_v: int
    W: int
    R: int
    in_dtype: str = BF16
    state_dtype: str = F32

    @property
    def N(self) -> int:
        return self.sqrt_n * self.sqrt_n

    @property
    def tokens(self) -> int:
        return self.B * self.T

    @property
    def token_heads(self) -> int:
        return self.B * self.T * self.H

    def replace(self, **kw) -> "Shape":
        return dataclasses.replace(self, **kw)

    def torch_in(self) -> torch.dtype:
        return _TORCH_DTYPE[self.in_dtype]

    def torch_state(self) -> torch.dtype:
        return _TORCH_DTYPE[self.state_dtype]


# The five workloads, named by what they are.
WORKLOADS = {
    "tiny_n1024_dv16": Shape("tiny_n1024_dv16", B=1, H=2, T=256, sqrt_n=32, d_v=16, W=8, R=8,
                             in_dtype=F32, state_dtype=F32),
    "d2048_h16_n1024_dv128": Shape("d2048_h16_n1024_dv128", B=8, H=16, T=4096, sqrt_n=32, d_v=128,
                                   W=64, R=64, in_dtype=BF16, state_dtype=F32),
    "d2048_h4_n16384_dv512": Shape("d2048_h4_n16384_dv512", B=8, H=4, T=8192, sqrt_n=128, d_v=512,
                                   W=64, R=64, in_dtype=BF16, state_dtype=F32),
    "d4096_h8_n16384_dv512": Shape("d4096_h8_n16384_dv512", B=4, H=8, T=32768, sqrt_n=128, d_v=512,
                                   W=64, R=64, in_dtype=BF16, state_dtype=F32),
    "long_t1m_n262144_dv2048": Shape("long_t1m_n262144_dv2048", B=1, H=2, T=1 << 20, sqrt_n=512,
                                     d_v=2048, W=64, R=64, in_dtype=BF16, state_dtype=BF16),
}
WORKLOAD_ORDER = list(WORKLOADS)

# Tensor ids for the per-tensor generator streams.
_STREAM = {"kp": 1, "qp": 2, "v": 3, "z": 4, "beta": 5, "M0": 6, "g": 7}


def _gen(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000003 + _STREAM[name])
    return g


def make_inputs(shape: Shape, seed: int = 0, device="cpu", with_gate: bool = False) -> dict:
    """Draws all inputs of one layer call on ``device``.

    Returns kp, qp [B,T,H,2*sqrt_n], v [B,T,H,d_v], alpha, beta [B,T,H] in the
    input dtype, M0 [H,N,d_v] in the state dtype and, with ``with_gate``,
    g [B,T,H,d_v]. Values depend on the device's generator (CPU and CUDA
    streams differ), so a check uses one device's draw throughout.
    """
    dev = torch.device(device)
    B, T, H = shape.B, shape.T, shape.H
    tin, tst = shape.torch_in(), shape.torch_state()
    out = {}
    score_shape = (B, T, H, 2 * shape.sqrt_n)
    out["kp"] = torch.randn(score_shape, generator=_gen(seed, "kp", dev), device=dev).to(tin)
    out["qp"] = torch.randn(score_shape, generator=_gen(seed, "qp", dev), device=dev).to(tin)
    out["v"] = torch.randn((B, T, H, shape.d_v), generator=_gen(seed, "v", dev), device=dev).to(tin)
    z = torch.randn((B, T, H), generator=_gen(seed, "z", dev), device=dev)
    out["alpha"] = torch.exp(-torch.nn.functional.softplus(z)).to(tin)
    out["beta"] = torch.rand((B, T, H), generator=_gen(seed, "beta", dev), device=dev).to(tin)
    out["M0"] = (0.02 * torch.randn((H, shape.N, shape.d_v), generator=_gen(seed, "M0", dev),
                                    device=dev)).to(tst)
    if with_gate:
        out["g"] = torch.randn((B, T, H, shape.d_v), generator=_gen(seed, "g", dev), device=dev).to(tin)
    return out


def to_numpy_f32(t: torch.Tensor):
    """Exact widening of a (bf16 or fp32) tensor to a float32 numpy array."""
    return t.detach().to("cpu", torch.float32).contiguous().numpy()
