"""The block-scaled fp8 state (E4M3 codes, one power-of-two scale per 16 row
values) against the oracle, through the C ABI.

Two bounds, both derived from the E4M3 grid rather than measured:

* One step from the same state. The kernel forms a written row in fp32
  (factored form), the oracle by the pages' two-step write in double; the two
  pre-quantisation values differ by a few fp32 roundings. Rounding both to
  nearest on the E4M3 grid then gives values at most one grid step apart (one
  step of the coarser grid when the two sides pick different block exponents,
  which happens only when the block maximum sits on the exponent threshold).
  So every decoded value of a written row is within one step, taken at the
  larger of the two magnitudes and the larger of the two exponents, and each
  y value within sum_r |q_r| * (that step of row r) plus fp32 read rounding.
  Each step starts from the oracle's state, so the bound does not compound.

* Many steps against the unrounded double recurrence. Quantising x adds at most
  half a step: max(2^-4 |x|, 2^-10 * 2^e) (normal and subnormal E4M3), and
  2^e < max_block|x| / 232 because the exponent is the smallest with
  max_block|x| <= 464 * 2^e. A write contracts an earlier error by
  a = alpha (1 - beta k) and adds a new one, so the error bound E of every
  state value obeys E <- a E + half_step(|x_exact| + a E); y errs by at most
  sum_r |q_r| E[r]. Small slack terms cover the kernel's fp32 arithmetic.
"""

import numpy as np
import pytest
import torch

from parity_helpers import f32
from sparse_memory_linear_pkm_b200 import synth

pytestmark = pytest.mark.gpu

FP32_SLACK = 1e-6  # relative: fp32 products, sums and fp32 softmax weights against double


def _dequant(oracle, codes, exps):
    return oracle.dequantize_fp8blk(codes, exps)


def _step_of(mag, e):
    """Spacing of the E4M3 grid scaled by 2^e at magnitude mag (subnormal
    spacing 2^-9 below 2^-6, 2^(j-3) in the binade [2^j, 2^(j+1)))."""
    s = np.ldexp(mag, -e)
    _, k = np.frexp(np.where(s > 0, s, 1.0))
    j = np.maximum(np.where(s > 0, k - 1, -6), -6)
    return np.ldexp(1.0, (j - 3) + e)


def _half_step_bound(a):
    """Upper bound of the quantisation error of values with magnitude <= a
    [..., d_v] (blocks of 16 along the last axis)."""
    blk = a.reshape(a.shape[:-1] + (-1, 16)).max(axis=-1)
    floor = np.repeat(np.ldexp(blk / 232.0, -10), 16, axis=-1)
    return np.maximum(np.ldexp(a, -4), floor)


def _buf(codes, exps, device):
    return torch.from_numpy(np.concatenate([codes.reshape(-1), exps.reshape(-1).view(np.uint8)])).to(device)


def _split(buf, codes_shape, exps_shape):
    got = buf.cpu().numpy()
    n = int(np.prod(codes_shape))
    return got[:n].reshape(codes_shape), got[n:].view(np.int8).reshape(exps_shape)


def _setup(oracle, seed, **kw):
    shape = synth.WORKLOADS["d2048_h16_n1024_dv128"].replace(**kw)
    inp = synth.make_inputs(shape, seed=seed, device="cpu")
    M0 = f32(inp["M0"])
    codes, exps = oracle.quantize_fp8blk(np.broadcast_to(M0[None], (shape.B,) + M0.shape).copy())
    idx_w, w_w = oracle.pkm_topk(f32(inp["kp"]), shape.W)
    idx_r, w_r = oracle.pkm_topk(f32(inp["qp"]), shape.R)
    return shape, inp, codes, exps, (idx_w, w_w, idx_r, w_r)


def _gpu_step(sdm, d, t, buf, shape):
    sl = {k: d[k][:, t:t + 1].contiguous() for k in ("kp", "qp", "v", "alpha", "beta")}
    y = sdm.layer_step(sl["kp"], sl["qp"], sl["v"], sl["alpha"], sl["beta"], buf, shape.W, shape.R)
    sdm.stream_check()
    return y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("W", [64, 16])
def test_decode_fp8_step_within_one_grid_step(sdm, oracle, cuda_device, W):
    shape, inp, codes, exps, (idx_w, w_w, idx_r, w_r) = _setup(oracle, 41, B=2, T=6, H=2, W=W, R=W)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    v, alpha, beta = f32(inp["v"]), f32(inp["alpha"]), f32(inp["beta"])
    for t in range(shape.T):
        buf = _buf(codes, exps, cuda_device)
        y = _gpu_step(sdm, d, t, buf, shape)
        gc, ge = _split(buf, codes.shape, exps.shape)
        sl = slice(t, t + 1)
        oy, oc, oe = oracle.scan_fp8blk(idx_w[:, sl], w_w[:, sl], idx_r[:, sl], w_r[:, sl], v[:, sl], alpha[:, sl],
                                        beta[:, sl], codes, exps)
        written = np.zeros(codes.shape[:3], dtype=bool)
        for b in range(shape.B):
            for h in range(shape.H):
                written[b, h, idx_w[b, t, h]] = True
        # rows the step does not write are left bit for bit
        assert np.array_equal(gc[~written], codes[~written]) and np.array_equal(ge[~written], exps[~written])
        Dk, Do = _dequant(oracle, gc, ge), _dequant(oracle, oc, oe)
        e_max = np.repeat(np.maximum(ge, oe).astype(np.int64), 16, axis=-1)
        step = _step_of(np.maximum(np.abs(Dk), np.abs(Do)), e_max) * (1 + FP32_SLACK)
        step[~written] = 0.0
        diff = np.abs(Dk - Do)
        assert np.all(diff <= step), ("state", t, float((diff - step).max()))
        ybound = np.zeros_like(oy)
        for b in range(shape.B):
            for h in range(shape.H):
                q = np.abs(w_r[b, t, h])[:, None]
                rows = idx_r[b, t, h]
                ybound[b, 0, h] = (q * step[b, h, rows]).sum(0) + 4 * FP32_SLACK * (q * np.abs(Do[b, h, rows])).sum(0)
        dy = np.abs(y - oy)
        assert np.all(dy <= ybound + 1e-30), ("y", t, float((dy - ybound).max()))
        codes, exps = oc, oe  # the next step starts from the oracle's state


def test_decode_fp8_state_error_against_exact_recurrence(sdm, oracle, cuda_device):
    shape, inp, codes, exps, (idx_w, w_w, idx_r, w_r) = _setup(oracle, 43, B=2, T=8, H=2)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    v, alpha, beta = (f32(inp[k]).astype(np.float64) for k in ("v", "alpha", "beta"))
    buf = _buf(codes, exps, cuda_device)
    M = _dequant(oracle, codes, exps)  # the exact recurrence starts from the same decoded state
    E = np.zeros_like(M)
    worst = 0.0
    for t in range(shape.T):
        y = _gpu_step(sdm, d, t, buf, shape)
        sl = slice(t, t + 1)
        M_old = M
        oy, M = oracle.scan_f64(idx_w[:, sl], w_w[:, sl], idx_r[:, sl], w_r[:, sl], v[:, sl], alpha[:, sl],
                                beta[:, sl], M_old)
        E_new = E.copy()
        for b in range(shape.B):
            for h in range(shape.H):
                a_t, b_t = alpha[b, t, h], beta[b, t, h]
                for j, i in enumerate(idx_w[b, t, h]):
                    cw = b_t * w_w[b, t, h, j]
                    aw = a_t * (1.0 - cw)
                    carried = aw * E[b, h, i]
                    slack = FP32_SLACK * (aw * (np.abs(M_old[b, h, i]) + E[b, h, i]) + cw * np.abs(v[b, t, h]))
                    E_new[b, h, i] = carried + slack + _half_step_bound(np.abs(M[b, h, i]) + carried + slack)
        E = E_new
        gc, ge = _split(buf, codes.shape, exps.shape)
        Dk = _dequant(oracle, gc, ge)
        err = np.abs(Dk - M)
        assert np.all(err <= E), ("state", t, float((err - E).max()))
        for b in range(shape.B):
            for h in range(shape.H):
                q = np.abs(w_r[b, t, h])[:, None]
                rows = idx_r[b, t, h]
                bound = (q * E[b, h, rows]).sum(0) + 4 * FP32_SLACK * (q * (np.abs(M[b, h, rows]) + E[b, h, rows])).sum(0)
                dy = np.abs(y[b, 0, h] - oy[b, 0, h])
                assert np.all(dy <= bound + 1e-30), ("y", t, b, h, float((dy - bound).max()))
        worst = max(worst, float(np.abs(y - oy).max() / max(np.abs(oy).max(), 1e-30)))
    # the fp8 state's read error, relative to the largest read value, stays at the format's precision
    assert worst < 0.25, worst


# ---- the fp8 state in whole-sequence calls (sdm_layer_forward, pipelined kernel)

def _whole_setup(oracle, seed, T, W, sqrt_n=8):
    shape = synth.WORKLOADS["d2048_h16_n1024_dv128"].replace(B=2, T=T, H=2, sqrt_n=sqrt_n, d_v=256, W=W, R=W)
    inp = synth.make_inputs(shape, seed=seed, device="cpu")
    M0 = f32(inp["M0"])
    c0, e0 = oracle.quantize_fp8blk(M0)  # M0 [H, N, d_v] as the fp8 state
    return shape, inp, c0, e0


@pytest.mark.parametrize("T,W", [(1, 16), (37, 16), (64, 64), (150, 24)])
def test_whole_sequence_fp8_state_equals_chained_decode_steps(sdm, oracle, cuda_device, T, W):
    """One sdm_layer_forward over T tokens on the fp8 state (pipelined kernel)
    leaves the state bit for bit where T single-token decode steps leave it:
    both decode a unit with its block exponent, write it in fp32 with the same
    operations and re-quantise it with the same rule. y differs only in the
    order of the fp32 read sums. With N = 64 slots and W = R up to 64, slots
    collide within and across tokens all the time."""
    shape, inp, c0, e0 = _whole_setup(oracle, 60 + T, T, W)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    M0 = _buf(c0, e0, cuda_device)
    y_full, M_full = sdm.layer_forward(d["kp"], d["qp"], d["v"], d["alpha"], d["beta"], M0, shape.W, shape.R)
    sdm.stream_check()
    assert sdm.scan_variant(sdm.make_shape(shape.B, T, shape.H, shape.sqrt_n, W, W, shape.d_v, torch.bfloat16,
                                           torch.uint8)) == "pipelined"
    # the decode chain starts from M0 in every batch row (codes of all rows, then their exponents)
    cb = np.broadcast_to(c0[None], (shape.B,) + c0.shape)
    eb = np.broadcast_to(e0[None], (shape.B,) + e0.shape)
    buf = _buf(cb, eb, cuda_device)
    ys = [_gpu_step(sdm, d, t, buf, shape) for t in range(T)]
    assert torch.equal(M_full.reshape(-1), buf), "state differs from the chained decode steps"
    y_chain = np.concatenate(ys, axis=1)
    got = y_full.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(got, y_chain, rtol=1e-5, atol=1e-6 * np.abs(y_chain).max())


def test_whole_sequence_fp8_state_error_against_exact_recurrence(sdm, oracle, cuda_device):
    """The whole-sequence call against the unrounded double recurrence from the
    same decoded start, with the compounding bound of the module docstring
    checked on every token's y and on the final state."""
    shape, inp, c0, e0 = _whole_setup(oracle, 71, 24, 32, sqrt_n=16)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    y_full, M_full = sdm.layer_forward(d["kp"], d["qp"], d["v"], d["alpha"], d["beta"], _buf(c0, e0, cuda_device),
                                       shape.W, shape.R)
    sdm.stream_check()
    y_full = y_full.cpu().numpy().astype(np.float64)
    idx_w, w_w = oracle.pkm_topk(f32(inp["kp"]), shape.W)
    idx_r, w_r = oracle.pkm_topk(f32(inp["qp"]), shape.R)
    v, alpha, beta = (f32(inp[k]).astype(np.float64) for k in ("v", "alpha", "beta"))
    D0 = _dequant(oracle, c0, e0)
    M = np.ascontiguousarray(np.broadcast_to(D0[None], (shape.B,) + D0.shape))
    E = np.zeros_like(M)
    for t in range(shape.T):
        sl = slice(t, t + 1)
        M_old = M
        oy, M = oracle.scan_f64(idx_w[:, sl], w_w[:, sl], idx_r[:, sl], w_r[:, sl], v[:, sl], alpha[:, sl],
                                beta[:, sl], M_old)
        E_new = E.copy()
        for b in range(shape.B):
            for h in range(shape.H):
                a_t, b_t = alpha[b, t, h], beta[b, t, h]
                for j, i in enumerate(idx_w[b, t, h]):
                    cw = b_t * w_w[b, t, h, j]
                    aw = a_t * (1.0 - cw)
                    carried = aw * E[b, h, i]
                    slack = FP32_SLACK * (aw * (np.abs(M_old[b, h, i]) + E[b, h, i]) + cw * np.abs(v[b, t, h]))
                    E_new[b, h, i] = carried + slack + _half_step_bound(np.abs(M[b, h, i]) + carried + slack)
        E = E_new
        for b in range(shape.B):
            for h in range(shape.H):
                q = np.abs(w_r[b, t, h])[:, None]
                rows = idx_r[b, t, h]
                bound = (q * E[b, h, rows]).sum(0) + 4 * FP32_SLACK * (q * (np.abs(M[b, h, rows]) + E[b, h, rows])).sum(0)
                dy = np.abs(y_full[b, t, h] - oy[b, 0, h])
                assert np.all(dy <= bound + 1e-30), ("y", t, b, h, float((dy - bound).max()))
    n = shape.B * shape.H * shape.N * shape.d_v
    got = M_full.reshape(-1).cpu().numpy()
    Dk = _dequant(oracle, got[:n].reshape(M.shape), got[n:].view(np.int8).reshape(M.shape[:-1] + (shape.d_v // 16,)))
    err = np.abs(Dk - M)
    assert np.all(err <= E), ("state", float((err - E).max()))


def test_whole_sequence_fp8_state_rejected_where_unsupported(sdm, cuda_device):
    shape = synth.WORKLOADS["d2048_h16_n1024_dv128"].replace(B=1, T=4, H=1, sqrt_n=8, d_v=128, W=8, R=8)
    inp = synth.make_inputs(shape, seed=1, device=cuda_device)
    M0 = sdm.quantize_fp8blk(inp["M0"].float().contiguous())
    with pytest.raises(sdm.SdmError, match="multiple of 256"):  # 16-byte exponent rows
        sdm.layer_forward(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], M0, shape.W, shape.R)
    with pytest.raises(sdm.SdmError, match="pipelined variant only"):
        sdm.layer_forward(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], M0, shape.W, shape.R,
                          variant="streaming")
