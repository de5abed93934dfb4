"""The C ABI library loads on the CPU and exports what include/sdm.h declares;
host-side validation answers without touching a GPU."""

import ctypes
import re
from pathlib import Path

import pytest

from sparse_memory_linear_pkm_b200 import build as build_mod
from sparse_memory_linear_pkm_b200 import native

ROOT = Path(__file__).resolve().parent.parent
HEADER = ROOT / "include" / "sdm.h"


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return native.load()


def declared_functions():
    text = HEADER.read_text()
    return set(re.findall(r"SDM_API\s+[\w\s\*]+?\b(sdm_\w+)\s*\(", text))


def test_header_and_binding_agree():
    assert declared_functions() == set(native.PROTOTYPES)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.sdm_abi_version() == native.ABI_VERSION == 2


def test_only_the_abi_is_exported(lib):
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", str(native.LIBRARY)], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert exported == declared_functions()


def test_status_strings(lib):
    for code in range(5):
        assert lib.sdm_status_string(code)
    assert lib.sdm_status_string(99) == b"unknown status"


def shape(**kw):
    d = dict(B=2, T=5, H=3, sqrt_n=8, W=4, R=4, d_v=32, in_dtype=native.BF16, state_dtype=native.F32,
             rms_eps=1e-6, variant=0)
    d.update(kw)
    return native.Shape(**d)


@pytest.mark.parametrize("bad", [dict(sqrt_n=0), dict(sqrt_n=1025), dict(W=0), dict(R=65), dict(W=257, sqrt_n=32),
                                 dict(d_v=24), dict(d_v=8), dict(B=-1), dict(in_dtype=7), dict(variant=4),
                                 dict(rms_eps=-1.0), dict(tile=-1), dict(tile=65)])
def test_invalid_shapes_rejected_on_host(lib, bad):
    s = shape(**bad)
    assert lib.sdm_scan_workspace_bytes(ctypes.byref(s)) == 0
    assert lib.sdm_layer_forward_workspace_bytes(ctypes.byref(s)) == 0
    st = lib.sdm_scan(ctypes.byref(s), *([None] * 10), None, 0, None)
    assert st == 1 and lib.sdm_last_error()


def test_workspace_sizes(lib):
    """Without a device the records workspace is the largest any recurrence
    kernel needs: the streaming kernel's records, or the pipelined kernel's,
    one per slot part (two parts), followed by the second part's read sums."""
    s = shape()
    rec_words = 4 + 4 + 4 + 4 + 8 // 2 + 4  # Wp, Wp, Rp, Rp, Fp/2, alpha/beta block
    # W, R rounded to 8: uint16 source rows, (a, c) pairs, read weights, slots, counts
    pipe_words = 8 // 2 + 8 // 2 + 2 * 8 + 8 + 8 + 8 + 4
    a256 = lambda x: (x + 255) // 256 * 256
    rec = max(a256(2 * 3 * 5 * rec_words * 4), a256(2 * 2 * 3 * 5 * pipe_words * 4) + a256(2 * 5 * 3 * 32 * 4))
    assert lib.sdm_scan_workspace_bytes(ctypes.byref(s)) == rec
    per = (2 * 5 * 3 * 4 * 4 + 255) // 256 * 256
    assert lib.sdm_layer_forward_workspace_bytes(ctypes.byref(s)) == 4 * per + rec


def test_argument_errors_without_gpu(lib):
    # null pointers and K out of range are caught before any CUDA call
    assert lib.sdm_pkm_topk(None, native.F32, 1, 1, 1, 4, 3, None, None, None) == 1
    assert b"scores" in lib.sdm_last_error()
    assert lib.sdm_pkm_topk(None, native.F32, 1, 1, 1, 4, 17, None, None, None) == 1
    assert b"K" in lib.sdm_last_error()
    # misaligned pointer
    assert lib.sdm_pkm_topk(ctypes.c_void_p(8), native.F32, 1, 1, 1, 4, 3, ctypes.c_void_p(16),
                            ctypes.c_void_p(32), None) == 1
    assert b"aligned" in lib.sdm_last_error()
    # empty problems are no-ops
    assert lib.sdm_pkm_topk(None, native.F32, 0, 7, 3, 4, 3, None, None, None) == 0
    s = shape(T=0)
    assert lib.sdm_scan(ctypes.byref(s), *([None] * 10), None, 0, None) == 0
    # too little workspace
    s = shape()
    fake = ctypes.c_void_p(1 << 20)
    st = lib.sdm_scan(ctypes.byref(s), *([fake] * 7), None, fake, fake, fake, 16, None)
    assert st == 1 and b"workspace" in lib.sdm_last_error()


def test_build_flags_target_sm100a():
    assert build_mod.ARCH_FLAGS == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_slot_count_arguments_without_gpu(lib):
    assert lib.sdm_slot_counts(None, 1, 4, 1, 2, 64, None, None) == 1
    assert b"idx" in lib.sdm_last_error()
    assert lib.sdm_slot_counts(ctypes.c_void_p(64), 1, 4, 1, 0, 64, ctypes.c_void_p(64), None) == 1
    assert b"K and N" in lib.sdm_last_error()
    assert lib.sdm_slot_counts(None, 1, 0, 1, 2, 64, ctypes.c_void_p(64), None) == 0


def test_backward_workspace_and_support_without_gpu(lib):
    # B=1, T=300, H=2, N=1024, W=R=64, d_v=128: 32 tiles of 4 columns per (b, h), 128-token chunks
    s = shape(B=1, T=300, H=2, sqrt_n=32, W=64, R=64, d_v=128)
    tiles = 1 * 2 * 32
    ckpt = tiles * (3 - 1) * 1024 * 4 * 4
    log = tiles * 128 * 64 * 4 * 4
    part = (1 * 300 * 2 * 32 * (64 + 64 + 2) * 4 + 255) // 256 * 256
    rec = (1 * 2 * 300 * (4 * 64 + 4) * 4 + 255) // 256 * 256  # slots, weights, alpha/beta per token
    assert lib.sdm_scan_backward_workspace_bytes(ctypes.byref(s)) == ckpt + log + part + rec
    s = shape(B=1, T=300, H=2, sqrt_n=32, W=64, R=64, d_v=128, state_dtype=native.BF16)
    assert lib.sdm_scan_backward_workspace_bytes(ctypes.byref(s)) == 0
    assert b"fp32 state" in lib.sdm_last_error()
    # N = 16384: tiles of 32 columns in global memory; one chunk; a working copy of the state
    s = shape(B=1, T=4, H=1, sqrt_n=128, W=8, R=8, d_v=64)
    log = 2 * 4 * 8 * 32 * 4
    part = (1 * 4 * 1 * 2 * (8 + 8 + 2) * 4 + 255) // 256 * 256
    rec = (1 * 1 * 4 * (4 * 8 + 4) * 4 + 255) // 256 * 256
    work = 1 * 1 * 16384 * 64 * 4
    assert lib.sdm_scan_backward_workspace_bytes(ctypes.byref(s)) == log + part + rec + work
    assert lib.sdm_pkm_topk_backward(None, None, None, 1, 2, 1, 4, 3, None, None) == 1
    assert lib.sdm_pkm_topk_backward(None, None, None, 0, 2, 1, 4, 3, None, None) == 0


def test_layer_step_launch_count(lib):
    assert lib.sdm_layer_step_launches(ctypes.byref(shape(T=1, W=8, R=8))) == 1  # single-launch decode
    assert lib.sdm_layer_step_launches(ctypes.byref(shape(T=2, W=8, R=8))) == 4
    assert lib.sdm_layer_step_launches(ctypes.byref(shape(T=1, W=8, R=4))) == 4
    assert lib.sdm_layer_step_launches(ctypes.byref(shape(T=1, W=8, R=8, variant=2))) == 4
    assert lib.sdm_layer_step_launches(ctypes.byref(shape(sqrt_n=0))) == -1


def test_layer_backward_arguments_without_gpu(lib):
    s = shape(B=1, T=3, H=1, sqrt_n=8, W=4, R=4, d_v=32)
    n = lib.sdm_layer_backward_workspace_bytes(ctypes.byref(s))
    assert n > lib.sdm_scan_backward_workspace_bytes(ctypes.byref(s)) > 0
    fake = ctypes.c_void_p(1 << 20)
    # g given without y_pre
    st = lib.sdm_layer_backward(ctypes.byref(s), *([fake] * 6), fake, None, *([fake] * 8), fake, n, None)
    assert st == 1 and b"y_pre" in lib.sdm_last_error()
    # too little workspace
    st = lib.sdm_layer_backward(ctypes.byref(s), *([fake] * 16), fake, 16, None)
    assert st == 1 and b"workspace" in lib.sdm_last_error()
    assert lib.sdm_rmsnorm_gate(None, None, native.F32, 2, 0, ctypes.c_float(1e-6), None) == 1
    assert lib.sdm_rmsnorm_gate_backward(None, None, native.F32, None, 0, 8, ctypes.c_float(1e-6), None, None,
                                         None) == 0


def test_layer_forward_launch_count_needs_device_or_fails(lib):
    # The count depends on the recurrence variant chosen for the device (resident 4, streaming 5,
    # pipelined 5 or 6 with the slot parts' sum); without a GPU it reports -1.
    n = lib.sdm_layer_forward_launches(ctypes.byref(shape()), 0)
    assert n in (-1, 4, 5, 6)
    assert lib.sdm_layer_forward_launches(ctypes.byref(shape(sqrt_n=0)), 0) == -1


def test_fp8_state_arguments_without_gpu(lib):
    assert lib.sdm_quantize_fp8blk(None, -1, None, None, None) == 1
    assert lib.sdm_quantize_fp8blk(None, 2, None, None, None) == 1 and b"x" in lib.sdm_last_error()
    fake = ctypes.c_void_p(1 << 20)
    assert lib.sdm_quantize_fp8blk(fake, 2, fake, None, None) == 1 and b"exps" in lib.sdm_last_error()
    assert lib.sdm_quantize_fp8blk(None, 0, None, None, None) == 0
    # the fp8 state is a valid state dtype for shapes; as an input dtype it is not
    assert lib.sdm_layer_step_launches(ctypes.byref(shape(T=1, W=8, R=8, state_dtype=native.FP8_B16))) == 1
    assert lib.sdm_layer_step_launches(ctypes.byref(shape(in_dtype=native.FP8_B16))) == -1


def test_backward_workspace_of_the_large_state_workload(lib):
    # d2048_h4_n16384_dv512: 32-column tiles in global memory, chunks of 2048 tokens
    # (the power of two at or above sqrt(T N / W) = 1448), a working copy of the state.
    s = shape(B=8, T=8192, H=4, sqrt_n=128, W=64, R=64, d_v=512)
    tiles = 8 * 4 * (512 // 32)
    N, C = 16384, 2048
    ckpt = tiles * (8192 // C - 1) * N * 32 * 4
    log = tiles * C * 64 * 32 * 4
    part = 8 * 8192 * 4 * (512 // 32) * (64 + 64 + 2) * 4
    rec = 8 * 4 * 8192 * (4 * 64 + 4) * 4
    work = 8 * 4 * N * 512 * 4
    assert lib.sdm_scan_backward_workspace_bytes(ctypes.byref(s)) == ckpt + log + part + rec + work
