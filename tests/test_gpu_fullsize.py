"""Full-size workloads in the launch configuration the benchmark times, against
the oracle (GPU machine host cores), through the C ABI.

The three fp32-state workloads are compared whole: the selection of every
token-head (indices bit-exact, weights within 1e-6), all of y and every row
of the final state within 1e-4 * max|ref|. The long-context workload
(T = 2^20, N = 262144, bf16 state) is too long for the oracle to finish; its
full-size launch is checked on a prefix of 65,536 tokens: the selection of
those 131,072 token-heads (both halves of the layer's selection: keys and
queries), y of every token of the prefix, and the final state of a call over
the prefix alone (the recurrence is causal, and the kernel's launch
configuration does not depend on T), all within 2e-2 * max|ref|; rows the full
launch never writes keep M0 exactly.
"""

import numpy as np
import pytest
import torch

from parity_helpers import TOL_WEIGHTS, assert_rel_close, f32, tol_for
from sparse_memory_linear_pkm_b200 import synth

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _check_selection(sdm, oracle, scores, K):
    idx, w = sdm.pkm_topk(scores, K)
    sdm.stream_check()
    oi, ow = oracle.pkm_topk(f32(scores), K)
    got = idx.cpu().numpy()
    bad = np.argwhere(got != oi)
    assert bad.size == 0, f"index mismatch at {bad[:3].tolist()} of {got.shape}"
    assert np.abs(w.cpu().numpy() - ow).max() <= TOL_WEIGHTS
    return oi, ow


@pytest.mark.parametrize("name", ["d2048_h16_n1024_dv128", "d2048_h4_n16384_dv512", "d4096_h8_n16384_dv512"])
def test_full_size_layer_matches_oracle(sdm, oracle, cuda_device, name):
    shape = synth.WORKLOADS[name]
    inp = synth.make_inputs(shape, seed=0, device=cuda_device)
    y, M_T = sdm.layer_forward(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], inp["M0"], shape.W,
                               shape.R)
    sdm.stream_check()
    y, M_T = y.cpu().numpy(), M_T.float().cpu().numpy()
    oiw, oww = _check_selection(sdm, oracle, inp["kp"], shape.W)
    oir, owr = _check_selection(sdm, oracle, inp["qp"], shape.R)
    M0 = f32(inp["M0"])
    M = np.ascontiguousarray(np.broadcast_to(M0[None], (shape.B,) + M0.shape))
    del inp["kp"], inp["qp"]
    oy, oM, _ = oracle.scan(oiw, oww, oir, owr, f32(inp["v"]), f32(inp["alpha"]), f32(inp["beta"]), M,
                            state_bf16=shape.state_dtype == synth.BF16)
    tol = tol_for(shape.state_dtype)
    assert_rel_close(y, oy, tol, "y")
    assert_rel_close(M_T, oM, tol, "M_T")


def test_long_context_layer_matches_oracle_on_prefix(sdm, oracle, cuda_device):
    shape = synth.WORKLOADS["long_t1m_n262144_dv2048"]
    Tp = 65536
    inp = synth.make_inputs(shape, seed=0, device=cuda_device)
    y, M_T = sdm.layer_forward(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], inp["M0"], shape.W,
                               shape.R)
    sdm.stream_check()
    tol = tol_for(shape.state_dtype)
    # rows no token of the whole sequence writes keep M0 exactly
    idx_w, _ = sdm.pkm_topk(inp["kp"], shape.W)
    for b in range(shape.B):
        for h in range(shape.H):
            written = torch.zeros(shape.N, dtype=torch.bool, device=cuda_device)
            written[idx_w[b, :, h].reshape(-1).long()] = True
            assert torch.equal(M_T[b, h][~written], inp["M0"][h][~written])
    del idx_w, M_T
    y_prefix = y[:, :Tp].cpu().numpy()
    del y
    pre = {k: inp[k][:, :Tp].contiguous() for k in ("kp", "qp", "v", "alpha", "beta")}
    yp, M_Tp = sdm.layer_forward(pre["kp"], pre["qp"], pre["v"], pre["alpha"], pre["beta"], inp["M0"], shape.W,
                                 shape.R)
    sdm.stream_check()
    # the prefix call is the same computation as the full launch's first Tp tokens
    assert np.array_equal(yp.cpu().numpy(), y_prefix)
    del yp
    M_Tp = M_Tp.float().cpu().numpy()
    oiw, oww = _check_selection(sdm, oracle, pre["kp"], shape.W)
    oir, owr = _check_selection(sdm, oracle, pre["qp"], shape.R)
    M0 = f32(inp["M0"])
    del inp
    oy, oM, _ = oracle.scan(oiw, oww, oir, owr, f32(pre["v"]), f32(pre["alpha"]), f32(pre["beta"]), M0[None],
                            state_bf16=True)
    assert_rel_close(y_prefix, oy, tol, "y over the prefix")
    assert_rel_close(M_Tp, oM, tol, "M after the prefix")
