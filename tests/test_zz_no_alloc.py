"""sdm_layer_forward_noalloc: the layer call for hosts that cannot give the
library any device scratch memory (for example a plugin whose host engine owns
the whole device pool, or a loop that must not call an allocator once it
runs). It takes its scratch from a fixed array inside the library instead of a
caller workspace, so its results must match sdm_layer_forward's.

Two calls in a row with different inputs check that what the first call left
in the shared array does not leak into the second. Kept in a file that pytest
collects last; it also passes on its own in a fresh process.
"""

import ctypes

import pytest
import torch

from parity_helpers import assert_rel_close, tol_for
from sparse_memory_linear_pkm_b200 import native, synth

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _shape(s: synth.Shape) -> native.Shape:
    code = {synth.F32: native.F32, synth.BF16: native.BF16}
    return native.Shape(s.B, s.T, s.H, s.sqrt_n, s.W, s.R, s.d_v, code[s.in_dtype], code[s.state_dtype], 1e-6, 0)


def _noalloc(lib, s, d, stream):
    y = torch.empty((s.B, s.T, s.H, s.d_v), dtype=torch.float32, device=d["kp"].device)
    M_T = torch.empty((s.B,) + tuple(d["M0"].shape), dtype=d["M0"].dtype, device=d["kp"].device)
    st = lib.sdm_layer_forward_noalloc(ctypes.byref(_shape(s)), _p(d["kp"]), _p(d["qp"]), _p(d["v"]),
                                       _p(d["alpha"]), _p(d["beta"]), _p(d.get("g")), _p(d["M0"]), _p(M_T),
                                       _p(y), stream)
    native.check(st)
    native.check(lib.sdm_stream_check(stream))
    return y, M_T


@pytest.mark.parametrize("name", ["tiny_n1024_dv16", "d2048_h16_n1024_dv128"])
def test_noalloc_matches_layer_forward_on_two_calls(cuda_device, name):
    import sparse_memory_linear_pkm_b200 as sdm

    lib = native.load()
    s = synth.WORKLOADS[name]
    if name != "tiny_n1024_dv16":
        s = s.replace(B=2, T=16, H=4)  # scratch need well under the fixed size
    assert sdm.layer_forward_workspace_bytes(_shape(s)) <= native.NOALLOC_SCRATCH_BYTES
    stream = ctypes.c_void_p(torch.cuda.current_stream(cuda_device).cuda_stream)
    tol = tol_for(s.state_dtype)
    for seed in (11, 12):
        d = {k: v.to(cuda_device) for k, v in synth.make_inputs(s, seed=seed, device="cpu").items()}
        y_ref, M_ref = sdm.layer_forward(d["kp"], d["qp"], d["v"], d["alpha"], d["beta"], d["M0"], s.W, s.R)
        sdm.stream_check()
        y, M_T = _noalloc(lib, s, d, stream)
        assert_rel_close(y.cpu().numpy(), y_ref.cpu().numpy(), tol, f"y (seed {seed})")
        assert_rel_close(M_T.float().cpu().numpy(), M_ref.float().cpu().numpy(), tol, f"M_T (seed {seed})")


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_device):
    lib = native.load()
    s = synth.WORKLOADS["d2048_h16_n1024_dv128"]  # needs about 1.2 GB of scratch
    fake = ctypes.c_void_p(1 << 20)
    st = lib.sdm_layer_forward_noalloc(ctypes.byref(_shape(s)), *([fake] * 5), None, fake, fake, fake, None)
    assert st == 1
    msg = lib.sdm_last_error().decode()
    assert "scratch" in msg and str(native.NOALLOC_SCRATCH_BYTES) in msg
