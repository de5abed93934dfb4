"""Shared pieces of the GPU-vs-oracle parity tests (test-side only)."""

from __future__ import annotations

import numpy as np
import torch

from sparse_memory_linear_pkm_b200 import synth

# Tolerances fixed for this path: relative to max|reference| for the outputs y
# and the final state; fp32 state 1e-4, bf16 state 2e-2. Softmax weights: the
# fp32 kernel rounds each selected score to fp32 (|error| <= 2^-24 |s|, scores
# are O(10)) and evaluates expf and one division, so |dw| <= 1e-6 absolute.
TOL_F32_STATE = 1e-4
TOL_BF16_STATE = 2e-2
TOL_WEIGHTS = 1e-6


def tol_for(state_dtype: str) -> float:
    return TOL_BF16_STATE if state_dtype == synth.BF16 else TOL_F32_STATE


def f32(t: torch.Tensor) -> np.ndarray:
    return synth.to_numpy_f32(t)


def assert_rel_close(got: np.ndarray, want: np.ndarray, tol: float, what: str):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    scale = max(np.abs(want).max(), 1e-30)
    err = np.abs(got - want).max() if got.size else 0.0
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    assert err <= tol * scale, f"{what}: max|diff| {err:.3e} > {tol:.1e} * max|ref| {scale:.3e}"


def random_selection(gen: torch.Generator, B, T, H, N, K):
    """Distinct uniform slots per token-head and positive weights summing to 1."""
    keys = torch.rand((B * T * H, N), generator=gen) if N <= 4096 else None
    if keys is not None:
        idx = torch.argsort(keys, dim=1)[:, :K].to(torch.int32)
    else:
        idx = torch.empty((B * T * H, K), dtype=torch.int32)
        for u in range(B * T * H):
            idx[u] = torch.randperm(N, generator=gen)[:K].to(torch.int32)
    w = torch.rand((B * T * H, K), generator=gen) + 0.05
    w = w / w.sum(-1, keepdim=True)
    return idx.reshape(B, T, H, K).contiguous(), w.reshape(B, T, H, K).contiguous()


def scan_inputs(shape: synth.Shape, seed: int):
    """Selection-independent inputs of one sdm_scan call, on the CPU."""
    gen = torch.Generator().manual_seed(seed)
    idx_w, w_w = random_selection(gen, shape.B, shape.T, shape.H, shape.N, shape.W)
    idx_r, w_r = random_selection(gen, shape.B, shape.T, shape.H, shape.N, shape.R)
    base = synth.make_inputs(shape, seed=seed, device="cpu")
    M = torch.stack([base["M0"]] * shape.B).contiguous()
    return dict(idx_w=idx_w, w_w=w_w, idx_r=idx_r, w_r=w_r, v=base["v"], alpha=base["alpha"],
                beta=base["beta"], M=M)


def oracle_on_compact_state(oracle, idx_w, w_w, idx_r, w_r, v, alpha, beta, M0_rows_fn, state_bf16, g=None,
                            eps=1e-6):
    """Runs the oracle recurrence on the rows the selection touches only.

    The recurrence reads and writes only selected rows, so renumbering the
    touched slots of each (b, h) densely and running on that compact state is
    the same computation on fewer rows. M0_rows_fn(b, h, slots) returns the
    initial values of those rows (float32 [len, d_v]). Returns y and a dict
    {(b, h): (slots, final rows)}.
    """
    B, T, H, W = idx_w.shape
    R = idx_r.shape[-1]
    d_v = v.shape[-1]
    touched = {}
    width = 0
    for b in range(B):
        for h in range(H):
            s = np.unique(np.concatenate([idx_w[b, :, h].ravel(), idx_r[b, :, h].ravel()]))
            touched[(b, h)] = s
            width = max(width, len(s))
    Mc = np.zeros((B, H, width, d_v), dtype=np.float32)
    cw = np.empty_like(idx_w)
    cr = np.empty_like(idx_r)
    for (b, h), s in touched.items():
        Mc[b, h, :len(s)] = M0_rows_fn(b, h, s)
        lut = {int(x): i for i, x in enumerate(s)}
        cw[b, :, h] = np.vectorize(lut.__getitem__)(idx_w[b, :, h])
        cr[b, :, h] = np.vectorize(lut.__getitem__)(idx_r[b, :, h])
    y, MT, _ = oracle.scan(cw, w_w, cr, w_r, v, alpha, beta, Mc, g=g, eps=eps, state_bf16=state_bf16)
    rows = {k: (s, MT[k[0], k[1], :len(s)]) for k, s in touched.items()}
    return y, rows
