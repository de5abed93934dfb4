"""The overlapped layer call: a one-batch-row call on the pipelined recurrence,
long enough for several token chunks, runs the selection and records of each
next chunk beside the current chunk's recurrence (sdm_layer_forward). Its
outputs must be those of the one-pass primitives bit for bit: sdm_pkm_topk of
k' and q' over the whole call, then one sdm_scan over the whole sequence."""

import ctypes

import pytest
import torch

from sparse_memory_linear_pkm_b200 import native, synth

pytestmark = pytest.mark.gpu

CHUNK = 65536  # tokens a chunk (the library's overlap chunk)


@pytest.mark.parametrize("state,d_v", [("bf16", 256), ("f32", 128)])
def test_overlapped_layer_call_equals_one_pass(sdm, cuda_device, state, d_v):
    T = 2 * CHUNK + 1003  # three chunks, the last one ragged
    shape = synth.Shape("overlap", B=1, T=T, H=2, sqrt_n=32, d_v=d_v, W=16, R=12, in_dtype="bf16",
                        state_dtype=state)
    inp = synth.make_inputs(shape, seed=21, device=cuda_device)
    sh = sdm.make_shape(1, T, 2, 32, 16, 12, d_v, torch.bfloat16, shape.torch_state(), variant="pipelined")
    assert sdm.layer_forward_chunks(sh) == 3
    # per chunk two selections, records and the recurrence; the state copy and the parts' sum once
    assert native.load().sdm_layer_forward_launches(ctypes.byref(sh), 0) == 4 * 3 + 1 + 1
    # the traced form with an event pair around each chunk's recurrence launch
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6 + 2 * 3)]
    for e in ev:
        e.record()
    y, M_T = sdm.layer_forward(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], inp["M0"], shape.W,
                               shape.R, variant="pipelined", events=ev)
    torch.cuda.synchronize()
    sdm.stream_check()
    chunk_ms = [ev[6 + 2 * k].elapsed_time(ev[7 + 2 * k]) for k in range(3)]
    assert all(ms > 0 for ms in chunk_ms)
    assert sum(chunk_ms) <= ev[3].elapsed_time(ev[4]) + 1e-3  # the launches lie inside the recurrence stage
    with pytest.raises(native.SdmError):  # per-chunk events of another count
        sdm.layer_forward(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], inp["M0"], shape.W, shape.R,
                          variant="pipelined", events=ev[:10])
    idx_w, w_w = sdm.pkm_topk(inp["kp"], shape.W)
    idx_r, w_r = sdm.pkm_topk(inp["qp"], shape.R)
    M = inp["M0"].unsqueeze(0).clone()
    y1 = sdm.scan(idx_w, w_w, idx_r, w_r, inp["v"], inp["alpha"], inp["beta"], M, variant="pipelined")
    sdm.stream_check()
    assert torch.equal(M_T, M), "state differs from the one-pass recurrence"
    assert torch.equal(y, y1), "y differs from the one-pass recurrence"


def test_overlapped_layer_call_with_epilogue_and_repeat(sdm, cuda_device):
    """The same with the RMS-norm x gate epilogue, and two calls in a row on
    one stream (the library's streams and the caller's stay ordered)."""
    T = 2 * CHUNK + 17
    shape = synth.Shape("overlap_g", B=1, T=T, H=1, sqrt_n=16, d_v=256, W=8, R=8, in_dtype="bf16",
                        state_dtype="bf16")
    inp = synth.make_inputs(shape, seed=22, device=cuda_device, with_gate=True)
    outs = [sdm.layer_forward(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], inp["M0"], shape.W,
                              shape.R, g=inp["g"], variant="pipelined") for _ in range(2)]
    sdm.stream_check()
    idx_w, w_w = sdm.pkm_topk(inp["kp"], shape.W)
    idx_r, w_r = sdm.pkm_topk(inp["qp"], shape.R)
    M = inp["M0"].unsqueeze(0).clone()
    y1 = sdm.scan(idx_w, w_w, idx_r, w_r, inp["v"], inp["alpha"], inp["beta"], M, g=inp["g"], variant="pipelined")
    sdm.stream_check()
    for y, M_T in outs:
        assert torch.equal(M_T, M) and torch.equal(y, y1)


def test_overlapped_layer_call_fp8_state(sdm, cuda_device):
    """The block-scaled fp8 state through the overlapped call equals one
    sdm_layer_step over the whole sequence (one pass from the same state)."""
    T = 2 * CHUNK + 301
    shape = synth.Shape("overlap_fp8", B=1, T=T, H=2, sqrt_n=32, d_v=256, W=16, R=16, in_dtype="bf16",
                        state_dtype="bf16")
    inp = synth.make_inputs(shape, seed=23, device=cuda_device)
    M0 = sdm.quantize_fp8blk(inp["M0"].float().contiguous())
    sh = sdm.make_shape(1, T, 2, 32, 16, 16, 256, torch.bfloat16, torch.uint8, variant="pipelined")
    assert sdm.layer_forward_chunks(sh) == 3
    y, M_T = sdm.layer_forward(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], M0, shape.W, shape.R,
                               variant="pipelined")
    sdm.stream_check()
    M = M0.clone()
    y1 = sdm.layer_step(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], M, shape.W, shape.R,
                        variant="pipelined")
    sdm.stream_check()
    assert torch.equal(M_T.reshape(-1), M), "fp8 state differs from the one-pass call"
    assert torch.equal(y, y1), "y differs from the one-pass call"
