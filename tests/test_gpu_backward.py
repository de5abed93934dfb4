"""Backward kernels against the oracle's derivatives, through the C ABI.

sdm_scan_backward and sdm_pkm_topk_backward are compared element by element
with oracle.scan_backward / oracle.pkm_topk_backward (double precision, pinned
by finite differences) on the same seeded inputs. The GPU recomputes the
forward in fp32, so the tolerance is the fp32-state forward's: 1e-4 * max|ref|.
"""

import numpy as np
import pytest
import torch

from parity_helpers import TOL_F32_STATE, assert_rel_close, f32, scan_inputs
from sparse_memory_linear_pkm_b200 import synth

pytestmark = pytest.mark.gpu

TOL_BWD = TOL_F32_STATE
# softmax derivative: fp32 products and one fp32 sum of K terms per token-head
TOL_TOPK_BWD = 1e-5

BWD = [
    # sqrt_n, d_v, W, R, in, T, B, H, M_in shared by the batch
    (32, 128, 64, 64, "bf16", 300, 2, 2, False),  # three checkpoint chunks and a ragged tail
    (8, 32, 5, 3, "f32", 41, 2, 1, True),
    (64, 64, 16, 16, "bf16", 150, 1, 2, False),  # N = 4096
    (8, 32, 40, 36, "f32", 33, 1, 1, False),  # W, R above one warp of entries
    (4, 16, 16, 16, "f32", 129, 1, 1, False),  # W = N: every slot written every token
    (16, 48, 12, 4, "f32", 1, 1, 3, True),  # one token
    (32, 16, 8, 8, "f32", 256, 1, 2, False),  # T a multiple of the chunk
    (8, 32, 5, 4, "bf16", 70, 2, 1, False),  # W + R odd: padded staging
    (16, 32, 128, 96, "f32", 20, 1, 2, False),  # W, R above 64: several rounds of entries per lane
    # N = 16384: state and adjoint tiles in global memory
    (128, 64, 16, 16, "bf16", 150, 1, 2, False),  # 32-column tiles, one chunk
    (128, 48, 8, 8, "f32", 70, 2, 1, True),  # d_v not a multiple of 32: 16-column tiles
    (128, 32, 64, 64, "bf16", 600, 1, 1, False),  # two chunks of 512
]


def _bwd_inputs(case, seed):
    sqrt_n, d_v, W, R, tin, T, B, H, shared = case
    shape = synth.Shape("t", B=B, T=T, H=H, sqrt_n=sqrt_n, d_v=d_v, W=W, R=R, in_dtype=tin, state_dtype="f32")
    inp = scan_inputs(shape, seed=seed)
    gen = torch.Generator().manual_seed(seed + 1)
    M0 = inp["M"][0]
    if shared:
        M_in = M0.clone()
        M_full = torch.stack([M0] * B)
    else:
        M_full = (inp["M"] + 0.05 * torch.randn(inp["M"].shape, generator=gen)).contiguous()
        M_in = M_full
    dy = torch.randn((B, T, H, d_v), generator=gen)
    dM_T = 0.3 * torch.randn((B, H, shape.N, d_v), generator=gen)
    return shape, inp, M_in, M_full, dy, dM_T


def _gpu_backward(sdm, dev, inp, M_in, dy, dM_T):
    d = {k: v.to(dev) for k, v in inp.items() if k != "M"}
    out = sdm.scan_backward(d["idx_w"], d["w_w"], d["idx_r"], d["w_r"], d["v"], d["alpha"], d["beta"], M_in.to(dev),
                            dy.to(dev), dM_T.to(dev).clone())
    sdm.stream_check()
    return out


def _oracle_backward(oracle, inp, M_full, dy, dM_T):
    return oracle.scan_backward(inp["idx_w"].numpy(), inp["w_w"].numpy().astype(np.float64), inp["idx_r"].numpy(),
                                inp["w_r"].numpy().astype(np.float64), f32(inp["v"]), f32(inp["alpha"]),
                                f32(inp["beta"]), f32(M_full), f32(dy), f32(dM_T))


@pytest.mark.parametrize("case", BWD, ids=lambda c: "-".join(map(str, c)))
def test_scan_backward_matches_oracle(sdm, oracle, cuda_device, case):
    shape, inp, M_in, M_full, dy, dM_T = _bwd_inputs(case, seed=sum(case[:4]) + case[5])
    got = _gpu_backward(sdm, cuda_device, inp, M_in, dy, dM_T)
    want = _oracle_backward(oracle, inp, M_full, dy, dM_T)
    for k in ("dv", "dalpha", "dbeta", "dw_w", "dw_r", "dM0"):
        assert_rel_close(got[k].cpu().numpy(), want[k], TOL_BWD, k)


def test_scan_backward_deterministic(sdm, cuda_device):
    case = (32, 64, 16, 16, "bf16", 200, 2, 2, False)
    _, inp, M_in, _, dy, dM_T = _bwd_inputs(case, seed=11)
    a = _gpu_backward(sdm, cuda_device, inp, M_in, dy, dM_T)
    b = _gpu_backward(sdm, cuda_device, inp, M_in, dy, dM_T)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_scan_backward_rejects_bf16_state(sdm, cuda_device):
    sh = sdm.make_shape(1, 4, 1, 32, 8, 8, 64, torch.float32, torch.bfloat16)
    with pytest.raises(sdm.SdmError, match="fp32 state"):
        sdm.scan_backward_workspace_bytes(sh)


def test_scan_backward_out_of_range_flagged(sdm, cuda_device):
    case = (8, 32, 4, 4, "f32", 9, 1, 1, False)
    _, inp, M_in, _, dy, dM_T = _bwd_inputs(case, seed=2)
    inp["idx_w"][0, 3, 0, 1] = 64  # N = 64
    inp["idx_r"][0, 5, 0, 2] = -3
    d = {k: v.to(cuda_device) for k, v in inp.items() if k != "M"}
    out = sdm.scan_backward(d["idx_w"], d["w_w"], d["idx_r"], d["w_r"], d["v"], d["alpha"], d["beta"],
                            M_in.to(cuda_device), dy.to(cuda_device), dM_T.to(cuda_device).clone())
    with pytest.raises(sdm.SdmError, match="DEVICE_FAULT"):
        sdm.stream_check()
    assert all(torch.isfinite(t).all() for t in out.values())


@pytest.mark.parametrize("sqrt_n,K", [(32, 64), (8, 5), (128, 64), (4, 16), (1, 1), (16, 256)])
def test_pkm_topk_backward_matches_oracle(sdm, oracle, cuda_device, sqrt_n, K):
    B, T, H = 2, 37, 3
    g = torch.Generator().manual_seed(sqrt_n + K)
    x = torch.randn((B, T, H, 2 * sqrt_n), generator=g)
    idx, w = oracle.pkm_topk(f32(x), K)
    dw = torch.randn((B, T, H, K), generator=g)
    w32 = torch.from_numpy(w.astype(np.float32))
    got = sdm.pkm_topk_backward(torch.from_numpy(idx).to(cuda_device), w32.to(cuda_device), dw.to(cuda_device),
                                sqrt_n)
    sdm.stream_check()
    want = oracle.pkm_topk_backward(idx, w32.numpy().astype(np.float64), f32(dw), sqrt_n)
    assert_rel_close(got.cpu().numpy(), want, TOL_TOPK_BWD, "dscores")


@pytest.mark.parametrize("name,pairs", [("d2048_h16_n1024_dv128", ((0, 0), (7, 15))),
                                        ("d2048_h4_n16384_dv512", ((5, 2),))])
def test_scan_backward_full_size_sampled(sdm, oracle, cuda_device, name, pairs):
    """A full-size workload (the bench's, and one whose state only fits in
    global memory), in the launch configuration the benchmark times, with a
    seeded synthetic selection; sampled (b, h) pairs compared with the oracle
    over the whole sequence."""
    shape = synth.WORKLOADS[name]
    inp = synth.make_inputs(shape, seed=0, device=cuda_device)
    gen = torch.Generator().manual_seed(3)

    def selection(K):  # distinct slots (a + k s) mod N with s odd (N a power of two), positive weights
        lead = (shape.B, shape.T, shape.H, 1)
        a = torch.randint(0, shape.N, lead, generator=gen)
        st = 2 * torch.randint(0, shape.N // 2, lead, generator=gen) + 1
        idx = ((a + torch.arange(K) * st) % shape.N).to(torch.int32).contiguous()
        w = torch.rand(lead[:3] + (K,), generator=gen) + 0.05
        return idx, (w / w.sum(-1, keepdim=True)).contiguous()

    idx_w, w_w = selection(shape.W)
    idx_r, w_r = selection(shape.R)
    dy = torch.randn((shape.B, shape.T, shape.H, shape.d_v), generator=gen)
    dev = cuda_device
    M0 = inp["M0"].float()
    out = sdm.scan_backward(idx_w.to(dev), w_w.to(dev), idx_r.to(dev), w_r.to(dev), inp["v"], inp["alpha"],
                            inp["beta"], M0, dy.to(dev))
    sdm.stream_check()
    for b, h in pairs:
        s = lambda t: t[b:b + 1, :, h:h + 1].contiguous()
        want = oracle.scan_backward(s(idx_w).numpy(), s(w_w).numpy().astype(np.float64), s(idx_r).numpy(),
                                    s(w_r).numpy().astype(np.float64), f32(s(inp["v"])), f32(s(inp["alpha"])),
                                    f32(s(inp["beta"])), f32(M0[h:h + 1].unsqueeze(0)), f32(s(dy)),
                                    np.zeros((1, 1, shape.N, shape.d_v)))
        for k in ("dv", "dalpha", "dbeta", "dw_w", "dw_r"):
            assert_rel_close(s(out[k]).cpu().numpy(), want[k], TOL_BWD, f"{k} (b={b}, h={h})")
        assert_rel_close(out["dM0"][b:b + 1, h:h + 1].cpu().numpy(), want["dM0"], TOL_BWD, f"dM0 (b={b}, h={h})")


@pytest.mark.parametrize("gdtype", [torch.float32, torch.bfloat16])
def test_rmsnorm_gate_and_backward_match_oracle(sdm, oracle, cuda_device, gdtype):
    gen = torch.Generator().manual_seed(4)
    x = torch.randn((3, 7, 2, 96), generator=gen)
    g = torch.randn(x.shape, generator=gen).to(gdtype)
    dout = torch.randn(x.shape, generator=gen)
    y = sdm.rmsnorm_gate(x.to(cuda_device).clone(), g.to(cuda_device), eps=1e-6)
    dx, dg = sdm.rmsnorm_gate_backward(x.to(cuda_device), g.to(cuda_device), dout.to(cuda_device), eps=1e-6)
    sdm.stream_check()
    assert_rel_close(y.cpu().numpy(), oracle.rmsnorm_gate(f32(x), f32(g), eps=1e-6), 1e-5, "epilogue")
    wdx, wdg = oracle.rmsnorm_gate_backward(f32(x), f32(g), f32(dout), eps=1e-6)
    assert_rel_close(dx.cpu().numpy(), wdx, 1e-5, "dL/dy_pre")
    assert_rel_close(dg.cpu().numpy(), wdg, 1e-5, "dL/dg")


@pytest.mark.parametrize("name,W,R,gate", [("d2048_h16_n1024_dv128", 64, 64, True), ("d2048_h16_n1024_dv128", 16, 8, False),
                                          ("d2048_h4_n16384_dv512", 64, 64, True)])
def test_layer_backward_matches_oracle(sdm, oracle, cuda_device, name, W, R, gate):
    """sdm_layer_backward (selection, epilogue, recurrence and selection-weight
    backwards in one call) against the oracle's pieces composed by hand."""
    shape = synth.WORKLOADS[name].replace(B=2, T=37, H=2, W=W, R=R)
    inp = synth.make_inputs(shape, seed=13, device="cpu", with_gate=gate)
    gen = torch.Generator().manual_seed(14)
    dy = torch.randn((shape.B, shape.T, shape.H, shape.d_v), generator=gen)
    idx_w, w_w = oracle.pkm_topk(f32(inp["kp"]), W)
    idx_r, w_r = oracle.pkm_topk(f32(inp["qp"]), R)
    M0 = f32(inp["M0"])
    M0b = np.broadcast_to(M0[None], (shape.B,) + M0.shape)
    y_pre, _ = oracle.scan_f64(idx_w, w_w, idx_r, w_r, f32(inp["v"]), f32(inp["alpha"]), f32(inp["beta"]), M0b)
    dy_scan = f32(dy).astype(np.float64)
    if gate:
        dy_scan, want_dg = oracle.rmsnorm_gate_backward(y_pre, f32(inp["g"]), f32(dy), eps=1e-6)
    want = oracle.scan_backward(idx_w, w_w, idx_r, w_r, f32(inp["v"]), f32(inp["alpha"]), f32(inp["beta"]), M0b,
                                dy_scan)
    want_dkp = oracle.pkm_topk_backward(idx_w, w_w, want["dw_w"], shape.sqrt_n)
    want_dqp = oracle.pkm_topk_backward(idx_r, w_r, want["dw_r"], shape.sqrt_n)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    got = sdm.layer_backward(d["kp"], d["qp"], d["v"], d["alpha"], d["beta"], d["M0"].float().contiguous(),
                             dy.to(cuda_device), W, R, g=d.get("g"),
                             y_pre=torch.from_numpy(y_pre.astype(np.float32)).to(cuda_device) if gate else None)
    sdm.stream_check()
    pairs = [("dkp", want_dkp), ("dqp", want_dqp), ("dv", want["dv"]), ("dalpha", want["dalpha"]),
             ("dbeta", want["dbeta"]), ("dM0", want["dM0"])]
    if gate:
        pairs.append(("dg", want_dg))
    for k, w_ in pairs:
        assert_rel_close(got[k].cpu().numpy(), w_, TOL_BWD, k)


@pytest.mark.parametrize("T,sqrt_n,d_v,W,R", [(300, 32, 128, 64, 64), (257, 16, 64, 16, 8), (128, 32, 128, 64, 64)])
def test_forward_checkpoints_replace_the_backward_recompute(sdm, cuda_device, T, sqrt_n, d_v, W, R):
    """sdm_layer_forward_ckpt gives the forward's results bit for bit, each
    stored checkpoint is the state after the tokens before it (a forward over
    that prefix), and the backward given them returns every derivative bit for
    bit as the backward that recomputes them."""
    shape = synth.WORKLOADS["d2048_h16_n1024_dv128"].replace(B=2, T=T, H=2, sqrt_n=sqrt_n, d_v=d_v, W=W, R=R)
    inp = synth.make_inputs(shape, seed=T, device=cuda_device, with_gate=True)
    args = (inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], inp["M0"], W, R)
    y0, M0_out = sdm.layer_forward(*args)
    y1, M1_out, ck = sdm.layer_forward_ckpt(*args)
    sdm.stream_check()
    assert torch.equal(y0, y1) and torch.equal(M0_out, M1_out)
    sh = sdm.make_shape(shape.B, T, shape.H, sqrt_n, W, R, d_v, torch.bfloat16, torch.float32)
    C, nbytes = sdm.layer_checkpoint_size(sh)
    n = (T + C - 1) // C
    assert nbytes == (n - 1) * shape.B * shape.H * shape.N * d_v * 4 and ck.numel() * 4 == nbytes
    ck = ck.view(max(n - 1, 0), shape.B, shape.H, shape.N, d_v)
    for k in range(1, n):
        pre = [t[:, :k * C].contiguous() for t in args[:5]]
        _, Mk = sdm.layer_forward(*pre, inp["M0"], W, R)
        assert torch.equal(ck[k - 1], Mk), f"checkpoint {k}"
    # the backward with the gate, from the pre-epilogue output, with and without the checkpoints
    gen = torch.Generator(device="cpu").manual_seed(T + 1)
    dy = torch.randn((shape.B, T, shape.H, d_v), generator=gen).to(cuda_device)
    y_pre = y0
    ref = sdm.layer_backward(*args[:6], dy, W, R, g=inp["g"], y_pre=y_pre)
    got = sdm.layer_backward(*args[:6], dy, W, R, g=inp["g"], y_pre=y_pre, checkpoints=ck.reshape(-1))
    sdm.stream_check()
    for k in ref:
        assert torch.equal(ref[k], got[k]), k


def test_forward_checkpoints_only_where_the_forward_stores_them(sdm, cuda_device):
    long = synth.WORKLOADS["long_t1m_n262144_dv2048"]
    sh = sdm.make_shape(1, 64, long.H, long.sqrt_n, long.W, long.R, long.d_v, torch.bfloat16, torch.bfloat16)
    with pytest.raises(sdm.SdmError, match="resident recurrence"):
        sdm.layer_checkpoint_size(sh)
