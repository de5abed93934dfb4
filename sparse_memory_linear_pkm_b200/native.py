"""ctypes binding of libsdm_b200.so (the C ABI declared in include/sdm.h).

Argument marshalling only: every step of the computation runs in the CUDA
library. Loading fails loudly when the library has not been built.
"""

from __future__ import annotations

import ctypes
from pathlib import Path

PKG = Path(__file__).resolve().parent
LIBRARY = PKG / "libsdm_b200.so"

SDM_OK = 0
STATUS_NAMES = {0: "SDM_OK", 1: "SDM_ERR_INVALID_ARGUMENT", 2: "SDM_ERR_UNSUPPORTED", 3: "SDM_ERR_CUDA",
                4: "SDM_ERR_DEVICE_FAULT"}
F32, BF16, FP8_B16 = 0, 1, 2  # FP8_B16: state only (E4M3 codes + a power-of-two scale per 16 values)
VARIANTS = {"auto": 0, "resident": 1, "streaming": 2, "pipelined": 3}
NOALLOC_SCRATCH_BYTES = 16 << 20  # SDM_NOALLOC_SCRATCH_BYTES in include/sdm.h
ABI_VERSION = 2  # SDM_ABI_VERSION in include/sdm.h


class Shape(ctypes.Structure):
    """sdm_shape_t."""

    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32),
                ("sqrt_n", ctypes.c_int32), ("W", ctypes.c_int32), ("R", ctypes.c_int32),
                ("d_v", ctypes.c_int32), ("in_dtype", ctypes.c_int32), ("state_dtype", ctypes.c_int32),
                ("rms_eps", ctypes.c_float), ("variant", ctypes.c_int32), ("tile", ctypes.c_int32)]


_p = ctypes.c_void_p
_i32 = ctypes.c_int32
_sz = ctypes.c_size_t
_shape_p = ctypes.POINTER(Shape)

# name -> (restype, argtypes); one entry per function declared in include/sdm.h.
PROTOTYPES = {
    "sdm_abi_version": (_i32, []),
    "sdm_row_sumsq": (_i32, [_p, ctypes.c_int64, _i32, _p, _p]),
    "sdm_rmsnorm_gate_rows": (_i32, [_p, _p, _i32, _p, ctypes.c_int64, _i32, _i32, ctypes.c_float, _p]),
    "sdm_status_string": (ctypes.c_char_p, [_i32]),
    "sdm_last_error": (ctypes.c_char_p, []),
    "sdm_pkm_topk": (_i32, [_p, _i32, _i32, _i32, _i32, _i32, _i32, _p, _p, _p]),
    "sdm_scan_workspace_bytes": (_sz, [_shape_p]),
    "sdm_scan_variant": (_i32, [_shape_p]),
    "sdm_scan": (_i32, [_shape_p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "sdm_state_init": (_i32, [_shape_p, _p, _p, _p]),
    "sdm_layer_forward_workspace_bytes": (_sz, [_shape_p]),
    "sdm_layer_forward": (_i32, [_shape_p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "sdm_layer_step_workspace_bytes": (_sz, [_shape_p]),
    "sdm_layer_step_launches": (_i32, [_shape_p]),
    "sdm_layer_forward_launches": (_i32, [_shape_p, _i32]),
    "sdm_layer_forward_chunks": (_i32, [_shape_p]),
    "sdm_scan_describe": (_i32, [_shape_p, ctypes.c_char_p, _sz]),
    "sdm_scan_backward_workspace_bytes": (_sz, [_shape_p]),
    "sdm_scan_backward": (_i32, [_shape_p] + [_p] * 8 + [_i32] + [_p] * 8 + [_sz, _p]),
    "sdm_pkm_topk_backward": (_i32, [_p, _p, _p, _i32, _i32, _i32, _i32, _i32, _p, _p]),
    "sdm_rmsnorm_gate": (_i32, [_p, _p, _i32, ctypes.c_int64, _i32, ctypes.c_float, _p]),
    "sdm_rmsnorm_gate_backward": (_i32, [_p, _p, _i32, _p, ctypes.c_int64, _i32, ctypes.c_float, _p, _p, _p]),
    "sdm_layer_backward_workspace_bytes": (_sz, [_shape_p]),
    "sdm_layer_backward": (_i32, [_shape_p] + [_p] * 17 + [_sz, _p]),
    "sdm_layer_checkpoint_size": (_i32, [_shape_p, _p, _p]),
    "sdm_layer_forward_ckpt": (_i32, [_shape_p] + [_p] * 10 + [_sz, _p, _sz, _p]),
    "sdm_layer_backward_ckpt": (_i32, [_shape_p] + [_p] * 17 + [_sz, _p, _sz, _p]),
    "sdm_slot_counts": (_i32, [_p, _i32, _i32, _i32, _i32, _i32, _p, _p]),
    "sdm_quantize_fp8blk": (_i32, [_p, ctypes.c_int64, _p, _p, _p]),
    "sdm_layer_step": (_i32, [_shape_p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "sdm_layer_forward_traced": (_i32, [_shape_p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p,
                                         ctypes.POINTER(_p), _i32]),
    "sdm_layer_forward_noalloc": (_i32, [_shape_p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p]),
    "sdm_stream_check": (_i32, [_p]),
}


class SdmError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")


_LIB = None


def load(path: Path | str | None = None) -> ctypes.CDLL:
    """Loads the CUDA library once; raises if it is missing."""
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    p = Path(path) if path is not None else LIBRARY
    if not p.exists():
        raise RuntimeError(f"{p.name} is not built: run `python -m sparse_memory_linear_pkm_b200.build`")
    lib = ctypes.CDLL(str(p))
    for name, (res, args) in PROTOTYPES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if lib.sdm_abi_version() != ABI_VERSION:
        raise RuntimeError("libsdm_b200.so ABI version mismatch")
    if path is None:
        _LIB = lib
    return lib


def check(status: int) -> None:
    if status != SDM_OK:
        msg = load().sdm_last_error().decode(errors="replace")
        raise SdmError(status, msg)
