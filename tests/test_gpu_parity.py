"""CUDA path against the oracle, element by element, through the C ABI.

Selected indices must be bit-exact; weights within 1e-6; y and the final
state within 1e-4 * max|ref| (fp32 state) or 2e-2 * max|ref| (bf16 state).
"""

import numpy as np
import pytest
import torch

from parity_helpers import (TOL_WEIGHTS, assert_rel_close, f32, oracle_on_compact_state, scan_inputs, tol_for)
from sparse_memory_linear_pkm_b200 import synth

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------- selection --

def _scores(kind, B, T, H, sqrt_n, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    shape = (B, T, H, 2 * sqrt_n)
    if kind == "normal":
        x = torch.randn(shape, generator=g)
    elif kind == "ties":
        x = torch.randint(-1, 2, shape, generator=g).float()
    elif kind == "zeros":
        x = torch.zeros(shape)
        x[torch.rand(shape, generator=g) < 0.5] = -0.0
    elif kind == "close":  # sums that differ below fp32 resolution
        x = torch.randn(shape, generator=g)
        x[..., sqrt_n:] = 1.0
        x[..., :sqrt_n] = torch.randint(0, 4, (B, T, H, sqrt_n), generator=g).float() * 2.0 ** -30
    else:
        raise ValueError(kind)
    return x.to(dtype)


SELECT = [(32, 8), (32, 64), (128, 64), (512, 64), (1, 1), (2, 4), (3, 5), (4, 16), (8, 40), (16, 256),
          (1024, 64), (64, 128)]


@pytest.mark.parametrize("sqrt_n,K", SELECT)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("kind", ["normal", "ties", "zeros", "close"])
def test_pkm_topk_matches_oracle(sdm, oracle, cuda_device, sqrt_n, K, dtype, kind):
    if kind == "close" and dtype == torch.bfloat16:
        pytest.skip("bf16 cannot hold the sub-resolution offsets")
    B, T, H = 2, 37, 3
    x = _scores(kind, B, T, H, sqrt_n, dtype, seed=sqrt_n * 1000 + K)
    idx, w = sdm.pkm_topk(x.to(cuda_device), K)
    sdm.stream_check()
    oi, ow = oracle.pkm_topk(f32(x), K)
    got = idx.cpu().numpy()
    bad = np.argwhere(got != oi)
    assert bad.size == 0, f"index mismatch at {bad[:5].tolist()}: gpu {got[tuple(bad[0][:3])]} oracle {oi[tuple(bad[0][:3])]}"
    assert np.abs(w.cpu().numpy() - ow).max() <= TOL_WEIGHTS


def test_pkm_topk_nan_stays_in_range(sdm, cuda_device):
    x = torch.randn(1, 9, 2, 64)
    x[0, ::2, :, 5] = float("nan")
    idx, _ = sdm.pkm_topk(x.to(cuda_device), 16)
    sdm.stream_check()
    i = idx.cpu()
    assert int(i.min()) >= 0 and int(i.max()) < 32 * 32


# -------------------------------------------------------- slot utilisation --

def _bincount(idx: np.ndarray, N: int) -> np.ndarray:
    """counts[b,h,i] = #{(t,k): idx[b,t,h,k] == i}, by definition."""
    B, _, H, _ = idx.shape
    out = np.zeros((B, H, N), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            out[b, h] = np.bincount(idx[b, :, h, :].ravel(), minlength=N)
    return out


# sqrt_n, K, T: N below and above the shared-memory bin limit; T spanning
# several 256-token blocks with a ragged tail
SLOTS = [(32, 64, 37), (8, 40, 300), (16, 6, 301), (128, 16, 513), (256, 64, 70), (1, 1, 5)]


@pytest.mark.parametrize("sqrt_n,K,T", SLOTS)
def test_slot_counts_match_bincount(sdm, oracle, cuda_device, sqrt_n, K, T):
    B, H, N = 2, 3, sqrt_n * sqrt_n
    x = _scores("ties", B, T, H, sqrt_n, torch.float32, seed=T * 7 + K)
    oi, _ = oracle.pkm_topk(f32(x), K)
    counts = sdm.slot_counts(torch.from_numpy(oi).to(cuda_device), N)
    sdm.stream_check()
    got = counts.cpu().numpy()
    want = _bincount(oi, N)
    assert np.array_equal(got, want)
    assert (got.sum(axis=-1) == T * K).all()


def test_slot_counts_accumulate_over_token_ranges(sdm, cuda_device):
    g = torch.Generator().manual_seed(5)
    N = 4096
    idx = torch.randint(0, N, (1, 600, 2, 8), generator=g, dtype=torch.int32)
    d = idx.to(cuda_device)
    counts = sdm.slot_counts(d[:, :257].contiguous(), N)
    sdm.slot_counts(d[:, 257:].contiguous(), N, counts)
    sdm.stream_check()
    assert np.array_equal(counts.cpu().numpy(), _bincount(idx.numpy(), N))


@pytest.mark.parametrize("K", [2, 4])  # scalar and 16-byte index loads
def test_slot_counts_out_of_range_flagged(sdm, cuda_device, K):
    idx = torch.zeros((1, 4, 1, K), dtype=torch.int32)
    idx[0, 1, 0, 0] = 64
    idx[0, 2, 0, 1] = -1
    for N in (64, 20000):  # shared-memory and global bins
        counts = sdm.slot_counts(idx.clone().masked_fill_(idx >= 64, N).to(cuda_device), N)
        with pytest.raises(sdm.SdmError, match="DEVICE_FAULT"):
            sdm.stream_check()
        assert int(counts.sum()) == 4 * K - 2 and int(counts[0, 0, 0]) == 4 * K - 2


# ------------------------------------------------------------ recurrence --

SCAN = [
    # sqrt_n, d_v, W, R, in, state, variant, T, B, H
    (32, 16, 8, 8, "f32", "f32", "resident", 37, 1, 2),
    (32, 128, 64, 64, "bf16", "f32", "resident", 29, 2, 2),
    (32, 128, 64, 64, "bf16", "f32", "streaming", 29, 2, 2),
    (128, 512, 64, 64, "bf16", "f32", "streaming", 23, 1, 2),
    (64, 64, 64, 64, "bf16", "bf16", "streaming", 31, 1, 1),
    (8, 32, 5, 3, "f32", "bf16", "streaming", 41, 2, 1),
    (8, 32, 5, 3, "f32", "bf16", "resident", 41, 2, 1),
    (4, 16, 16, 16, "f32", "f32", "streaming", 50, 1, 2),
    (4, 16, 16, 16, "f32", "f32", "resident", 50, 1, 2),
    (16, 64, 7, 9, "bf16", "bf16", "resident", 33, 1, 3),
    (16, 48, 12, 4, "f32", "f32", "streaming", 19, 1, 1),
    (256, 2048, 64, 64, "bf16", "bf16", "streaming", 17, 1, 1),
    # the pipelined kernel: slots split over two CTAs per column tile (parts = 2), except in the
    # last case, whose 96 column tiles leave room for one CTA each (parts = 1)
    (32, 128, 64, 64, "bf16", "f32", "pipelined", 29, 2, 2),
    (128, 512, 64, 64, "bf16", "f32", "pipelined", 23, 1, 2),
    (64, 64, 64, 64, "bf16", "bf16", "pipelined", 31, 1, 1),
    (16, 64, 7, 9, "bf16", "bf16", "pipelined", 33, 1, 3),
    (32, 128, 100, 30, "f32", "f32", "pipelined", 25, 1, 2),
    (4, 32, 16, 16, "f32", "f32", "pipelined", 50, 1, 2),
    (256, 2048, 64, 64, "bf16", "bf16", "pipelined", 17, 1, 1),
    (64, 2048, 64, 64, "bf16", "bf16", "pipelined", 20, 1, 3),
]


def _run_scan(sdm, dev, shape, inp, variant, g=None, tile=0):
    d = {k: v.to(dev) for k, v in inp.items()}
    M = d["M"].clone()
    y = sdm.scan(d["idx_w"], d["w_w"], d["idx_r"], d["w_r"], d["v"], d["alpha"], d["beta"], M,
                 g=None if g is None else g.to(dev), variant=variant, tile=tile)
    sdm.stream_check()
    return y, M


@pytest.mark.parametrize("case", SCAN, ids=lambda c: "-".join(map(str, c)))
def test_scan_matches_oracle(sdm, oracle, cuda_device, case):
    sqrt_n, d_v, W, R, tin, tst, variant, T, B, H = case
    shape = synth.Shape("t", B=B, T=T, H=H, sqrt_n=sqrt_n, d_v=d_v, W=W, R=R, in_dtype=tin, state_dtype=tst)
    inp = scan_inputs(shape, seed=sum(case[:4]) + T)
    y, M = _run_scan(sdm, cuda_device, shape, inp, variant)
    oy, oM, _ = oracle.scan(inp["idx_w"].numpy(), inp["w_w"].numpy().astype(np.float64), inp["idx_r"].numpy(),
                            inp["w_r"].numpy().astype(np.float64), f32(inp["v"]), f32(inp["alpha"]),
                            f32(inp["beta"]), f32(inp["M"]), state_bf16=(tst == "bf16"))
    tol = tol_for(tst)
    assert_rel_close(y.cpu().numpy(), oy, tol, "y")
    assert_rel_close(f32(M), oM, tol, "M_T")


@pytest.mark.parametrize("tst,tile", [("bf16", k) for k in range(1, 6)] + [("f32", k) for k in range(1, 4)])
def test_pipelined_tiles_match_oracle(sdm, oracle, cuda_device, tst, tile):
    """Every entry of the pipelined kernel's tile table (warp counts, stage
    depth) against the oracle, on a case with many slot collisions."""
    shape = synth.Shape("t", B=1, T=150, H=2, sqrt_n=12, d_v=256 if tst == "bf16" else 128, W=24, R=20,
                        in_dtype="bf16", state_dtype=tst)
    inp = scan_inputs(shape, seed=70 + tile)
    y, M = _run_scan(sdm, cuda_device, shape, inp, "pipelined", tile=tile)
    oy, oM, _ = oracle.scan(inp["idx_w"].numpy(), inp["w_w"].numpy().astype(np.float64), inp["idx_r"].numpy(),
                            inp["w_r"].numpy().astype(np.float64), f32(inp["v"]), f32(inp["alpha"]),
                            f32(inp["beta"]), f32(inp["M"]), state_bf16=(tst == "bf16"))
    assert_rel_close(y.cpu().numpy(), oy, tol_for(tst), "y")
    assert_rel_close(f32(M), oM, tol_for(tst), "M_T")


@pytest.mark.parametrize("tst,tiles", [("bf16", (1, 2, 3)), ("f32", (1, 3))])
@pytest.mark.parametrize("T", [1, 2, 7, 64, 151])
def test_pipelined_two_token_steps_bit_identical(sdm, cuda_device, tst, tiles, T):
    """Tokens taken two per barrier step (the second recomputing the first's
    writes of shared slots) give the same y and state bit for bit as one
    token per step: every value and every sum is formed in the same order."""
    shape = synth.Shape("t", B=2, T=T, H=1, sqrt_n=8, d_v=256 if tst == "bf16" else 128, W=16, R=12,
                        in_dtype="bf16", state_dtype=tst)
    inp = scan_inputs(shape, seed=90 + T)
    outs = [_run_scan(sdm, cuda_device, shape, inp, "pipelined", tile=k) for k in tiles]
    for y, M in outs[1:]:
        assert torch.equal(y, outs[0][0]) and torch.equal(M, outs[0][1])


@pytest.mark.parametrize("variant", ["resident", "streaming", "pipelined"])
def test_scan_deterministic_and_chunkable(sdm, cuda_device, variant):
    """Two runs are bit-identical, and scanning [0, T1) then [T1, T) equals one
    scan over [0, T) bit for bit (the state is the checkpoint)."""
    shape = synth.Shape("t", B=2, T=45, H=2, sqrt_n=16, d_v=64, W=16, R=16, in_dtype="bf16", state_dtype="f32")
    inp = scan_inputs(shape, seed=5)
    y1, M1 = _run_scan(sdm, cuda_device, shape, inp, variant)
    y2, M2 = _run_scan(sdm, cuda_device, shape, inp, variant)
    assert torch.equal(y1, y2) and torch.equal(M1, M2)
    T1 = 19
    first = {k: (v[:, :T1].contiguous() if k != "M" else v) for k, v in inp.items()}
    ya, Ma = _run_scan(sdm, cuda_device, shape, first, variant)
    second = {k: (v[:, T1:].contiguous() if k != "M" else Ma.cpu()) for k, v in inp.items()}
    yb, Mb = _run_scan(sdm, cuda_device, shape, second, variant)
    assert torch.equal(torch.cat([ya, yb], dim=1), y1)
    assert torch.equal(Mb, M1)


def test_variants_agree(sdm, cuda_device):
    shape = synth.Shape("t", B=1, T=40, H=2, sqrt_n=32, d_v=128, W=64, R=64, in_dtype="bf16", state_dtype="f32")
    inp = scan_inputs(shape, seed=9)
    ya, Ma = _run_scan(sdm, cuda_device, shape, inp, "resident")
    for variant in ("streaming", "pipelined"):
        yb, Mb = _run_scan(sdm, cuda_device, shape, inp, variant)
        assert_rel_close(yb.cpu().numpy(), ya.cpu().numpy(), 1e-5, f"y ({variant})")
        assert_rel_close(f32(Mb), f32(Ma), 1e-5, f"M_T ({variant})")


def test_scan_out_of_range_index_flagged(sdm, cuda_device):
    shape = synth.Shape("t", B=1, T=8, H=1, sqrt_n=8, d_v=32, W=4, R=4, in_dtype="f32", state_dtype="f32")
    inp = scan_inputs(shape, seed=3)
    inp["idx_w"][0, 3, 0, 1] = 64  # N = 64
    inp["idx_r"][0, 5, 0, 2] = -7
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    for variant in ("resident", "streaming", "pipelined"):
        M = d["M"].clone()
        sdm.scan(d["idx_w"], d["w_w"], d["idx_r"], d["w_r"], d["v"], d["alpha"], d["beta"], M, variant=variant)
        with pytest.raises(sdm.SdmError, match="DEVICE_FAULT"):
            sdm.stream_check()
        sdm.stream_check()  # the word was cleared
        assert torch.isfinite(M).all()


# ----------------------------------------------------------- whole layer --

def _layer_case(sdm, oracle, dev, shape, seed, with_gate=False, variant="auto"):
    inp = synth.make_inputs(shape, seed=seed, device="cpu", with_gate=with_gate)
    d = {k: v.to(dev) for k, v in inp.items()}
    y, M_T = sdm.layer_forward(d["kp"], d["qp"], d["v"], d["alpha"], d["beta"], d["M0"], shape.W, shape.R,
                               g=d.get("g"), variant=variant)
    sdm.stream_check()
    idx_w, w_w = oracle.pkm_topk(f32(inp["kp"]), shape.W)
    idx_r, w_r = oracle.pkm_topk(f32(inp["qp"]), shape.R)
    M0 = f32(inp["M0"])
    oy, rows = oracle_on_compact_state(oracle, idx_w, w_w, idx_r, w_r, f32(inp["v"]), f32(inp["alpha"]),
                                       f32(inp["beta"]), lambda b, h, s: M0[h, s],
                                       shape.state_dtype == "bf16", g=None if not with_gate else f32(inp["g"]))
    tol = tol_for(shape.state_dtype)
    assert_rel_close(y.cpu().numpy(), oy, tol, "y")
    M_T_host = f32(M_T)
    for (b, h), (s, want) in rows.items():
        assert_rel_close(M_T_host[b, h, s], want, tol, f"M_T rows of (b={b}, h={h})")
        untouched = np.setdiff1d(np.arange(shape.N), s)
        assert np.array_equal(M_T_host[b, h, untouched], M0[h, untouched])


@pytest.mark.parametrize("name,steps", [("tiny_n1024_dv16", (1,) * 9), ("d2048_h16_n1024_dv128", (1, 1, 3, 1, 7)),
                                        ("d2048_h4_n16384_dv512", (1,) * 6), ("long_t1m_n262144_dv2048", (1, 2, 1))])
def test_layer_step_chain(sdm, oracle, cuda_device, name, steps):
    """Decode-style calls carrying the state (T = 1 or a few tokens each) equal
    the whole-sequence layer and the oracle."""
    T = sum(steps)
    shape = synth.WORKLOADS[name].replace(B=2, T=T, H=2)
    if name == "long_t1m_n262144_dv2048":
        shape = shape.replace(B=1)
    inp = synth.make_inputs(shape, seed=23, device="cpu")
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    y_ref, M_ref = sdm.layer_forward(d["kp"], d["qp"], d["v"], d["alpha"], d["beta"], d["M0"], shape.W, shape.R)
    M = d["M0"].unsqueeze(0).repeat(shape.B, 1, 1, 1).contiguous()
    ys, t0 = [], 0
    for n in steps:
        sl = lambda x: x[:, t0:t0 + n].contiguous()
        ys.append(sdm.layer_step(sl(d["kp"]), sl(d["qp"]), sl(d["v"]), sl(d["alpha"]), sl(d["beta"]), M,
                                 shape.W, shape.R))
        t0 += n
    sdm.stream_check()
    y = torch.cat(ys, dim=1)
    tol = tol_for(shape.state_dtype)
    assert_rel_close(y.cpu().numpy(), y_ref.cpu().numpy(), tol, "y (steps vs whole sequence)")
    assert_rel_close(f32(M), f32(M_ref), tol, "M_T (steps vs whole sequence)")
    idx_w, w_w = oracle.pkm_topk(f32(inp["kp"]), shape.W)
    idx_r, w_r = oracle.pkm_topk(f32(inp["qp"]), shape.R)
    M0 = f32(inp["M0"])
    oy, _ = oracle_on_compact_state(oracle, idx_w, w_w, idx_r, w_r, f32(inp["v"]), f32(inp["alpha"]),
                                    f32(inp["beta"]), lambda b, h, s: M0[h, s], shape.state_dtype == "bf16")
    assert_rel_close(y.cpu().numpy(), oy, tol, "y (steps vs oracle)")


@pytest.mark.parametrize("name,W,R,gate", [("d2048_h16_n1024_dv128", 64, 64, True), ("tiny_n1024_dv16", 8, 8, False),
                                          ("d2048_h4_n16384_dv512", 64, 64, True),
                                          ("long_t1m_n262144_dv2048", 64, 64, False),
                                          ("d2048_h16_n1024_dv128", 16, 16, False)])
def test_decode_step_single_launch_matches_general_path(sdm, cuda_device, name, W, R, gate):
    """T = 1 calls with the automatic variant run the single-launch decode
    kernel; they give the same state bit for bit as the general path (forced
    streaming variant) and y up to summation order, with and without the
    RMS-norm x gate."""
    shape = synth.WORKLOADS[name].replace(B=2, T=5, H=3, W=W, R=R)
    if name == "long_t1m_n262144_dv2048":
        shape = shape.replace(B=1, H=1)
    inp = synth.make_inputs(shape, seed=31, device="cpu", with_gate=gate)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    M_a = d["M0"].unsqueeze(0).repeat(shape.B, 1, 1, 1).contiguous()
    M_b = M_a.clone()
    for t in range(shape.T):
        sl = {k: d[k][:, t:t + 1].contiguous() for k in ("kp", "qp", "v", "alpha", "beta")}
        g = d["g"][:, t:t + 1].contiguous() if gate else None
        ya = sdm.layer_step(sl["kp"], sl["qp"], sl["v"], sl["alpha"], sl["beta"], M_a, W, R, g=g)
        yb = sdm.layer_step(sl["kp"], sl["qp"], sl["v"], sl["alpha"], sl["beta"], M_b, W, R, g=g,
                            variant="streaming")
        sdm.stream_check()
        assert torch.equal(M_a, M_b), f"state differs after token {t}"
        assert_rel_close(ya.cpu().numpy(), yb.cpu().numpy(), 1e-5, f"y of token {t}")


def test_layer_forward_tiny_workload_full(sdm, oracle, cuda_device):
    _layer_case(sdm, oracle, cuda_device, synth.WORKLOADS["tiny_n1024_dv16"], seed=0)


@pytest.mark.parametrize("name", synth.WORKLOAD_ORDER[1:])
def test_layer_forward_reduced_workloads(sdm, oracle, cuda_device, name):
    """Each workload's sqrt_n, d_v, W, R and dtypes with a short, ragged T."""
    s = synth.WORKLOADS[name]
    _layer_case(sdm, oracle, cuda_device, s.replace(B=min(s.B, 2), T=37, H=min(s.H, 3)), seed=1)


@pytest.mark.parametrize("variant", ["resident", "streaming", "pipelined"])
def test_layer_forward_epilogue(sdm, oracle, cuda_device, variant):
    s = synth.WORKLOADS["d2048_h16_n1024_dv128"].replace(B=1, T=21, H=2)
    _layer_case(sdm, oracle, cuda_device, s, seed=2, with_gate=True, variant=variant)


@pytest.mark.parametrize("sqrt_n,W,R,T", [(1, 1, 1, 5), (4, 16, 16, 9), (8, 40, 3, 1), (2, 3, 4, 0)])
def test_layer_forward_edge_shapes(sdm, oracle, cuda_device, sqrt_n, W, R, T):
    s = synth.Shape("edge", B=2, T=T, H=2, sqrt_n=sqrt_n, d_v=32, W=W, R=R, in_dtype="f32", state_dtype="f32")
    if T == 0:
        inp = synth.make_inputs(s, seed=0, device=cuda_device)
        y, M_T = sdm.layer_forward(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], inp["M0"], W, R)
        sdm.stream_check()
        assert y.numel() == 0 and torch.equal(M_T, torch.stack([inp["M0"]] * 2))
        return
    _layer_case(sdm, oracle, cuda_device, s, seed=4)


# ---------------------------------------------- full-size, sampled checks --

@pytest.mark.parametrize("name", synth.WORKLOAD_ORDER[1:])
def test_full_size_workload_sampled(sdm, oracle, cuda_device, name):
    """The full workload in the launch configuration the benchmark times:
    selection bit-exact on sampled token-heads, y of the first tokens of every
    (b, h) against the oracle, the final state's never-written rows equal to
    M0, and the convex-combination bound on y and M_T everywhere."""
    shape = synth.WORKLOADS[name]
    inp = synth.make_inputs(shape, seed=0, device=cuda_device)
    y, M_T = sdm.layer_forward(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], inp["M0"], shape.W,
                               shape.R)
    sdm.stream_check()
    tol = tol_for(shape.state_dtype)
    # (1) selection on sampled token-heads
    idx_w, w_w = sdm.pkm_topk(inp["kp"], shape.W)
    sdm.stream_check()
    gen = torch.Generator().manual_seed(7)
    n_units = shape.B * shape.T * shape.H
    units = torch.randint(0, n_units, (192,), generator=gen)
    kp_s = inp["kp"].reshape(n_units, -1)[units.to(cuda_device)]
    oi, ow = oracle.pkm_topk(f32(kp_s), shape.W)
    assert np.array_equal(idx_w.reshape(n_units, -1)[units.to(cuda_device)].cpu().numpy(), oi)
    assert np.abs(w_w.reshape(n_units, -1)[units.to(cuda_device)].cpu().numpy() - ow).max() <= TOL_WEIGHTS
    # (2) the first T' tokens of every (b, h)
    Tp = 24
    sl = lambda t: f32(t[:, :Tp])
    oiw, oww = oracle.pkm_topk(sl(inp["kp"]), shape.W)
    oir, owr = oracle.pkm_topk(sl(inp["qp"]), shape.R)
    M0 = inp["M0"]
    rows_fn = lambda b, h, s: f32(M0[h][torch.as_tensor(s, device=cuda_device).long()])
    oy, _ = oracle_on_compact_state(oracle, oiw, oww, oir, owr, sl(inp["v"]), sl(inp["alpha"]), sl(inp["beta"]),
                                    rows_fn, shape.state_dtype == "bf16")
    assert_rel_close(y[:, :Tp].cpu().numpy(), oy, tol, "y prefix")
    # (3) rows no token writes keep M0 exactly; (4) convex bound
    bound = max(float(inp["M0"].abs().max()), float(inp["v"].abs().max()))
    assert float(y.abs().max()) <= bound * (1 + 1e-3)
    assert float(M_T.float().abs().max()) <= bound * (1 + 1e-2)
    for b in range(shape.B):
        for h in range(shape.H):
            written = torch.zeros(shape.N, dtype=torch.bool, device=cuda_device)
            written[idx_w[b, :, h].reshape(-1).long()] = True
            assert torch.equal(M_T[b, h][~written], M0[h][~written])


# ------------------------------------------------- block-scaled fp8 state --

def test_quantize_fp8blk_matches_oracle(sdm, oracle, cuda_device):
    gen = torch.Generator().manual_seed(21)
    x = torch.randn((64, 48), generator=gen) * torch.pow(2.0, torch.randint(-30, 30, (64, 1), generator=gen).float())
    x[3] = 0.0
    x[4, :16] = -0.0
    x[5, 5] = 1e30
    x[6, :] = 2.0 ** -130
    buf = sdm.quantize_fp8blk(x.to(cuda_device))
    sdm.stream_check()
    codes, exps = sdm.fp8blk_parts(buf, x.numel())
    oc, oe = oracle.quantize_fp8blk(f32(x))
    assert np.array_equal(codes.cpu().numpy(), oc.reshape(-1))
    assert np.array_equal(exps.cpu().numpy(), oe.reshape(-1))


def test_fp8_state_only_in_the_decode_step(sdm, cuda_device):
    shape = synth.WORKLOADS["tiny_n1024_dv16"].replace(B=1, T=2, H=1)
    inp = synth.make_inputs(shape, seed=1, device=cuda_device)
    buf = sdm.quantize_fp8blk(inp["M0"].float().contiguous())
    with pytest.raises(sdm.SdmError, match="fp8"):
        sdm.layer_step(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], buf, shape.W, shape.R)
