"""CPU oracle for the Sparse Delta Memory recurrent core -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library never calls it and shares
no code with it. The arithmetic lives in ``sdm_oracle.cpp`` (plain C++, double
precision); this module only compiles it, loads it with ctypes and marshals
numpy arrays.

Sources: the papers.ananclaw.com explainer of arXiv 2607.07386 (section 3.1,
steps 1-3) and the gist.science "Technical Summary: Sparse Delta Memory (SDM)"
(Core Mechanism 1-4). See ``sdm_oracle.cpp`` for the step-by-step definition.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
SOURCE = _HERE / "sdm_oracle.cpp"
LIBRARY = _HERE / "liboracle_sdm.so"

_c_i32 = ctypes.c_int32
_c_i64 = ctypes.c_int64
_c_ptr = ctypes.c_void_p


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover - non-Linux
        return max(1, os.cpu_count() or 1)


def build(mutant: int = 0, out: Path | None = None, force: bool = False) -> Path:
    """Compiles the oracle with g++ and returns the shared-library path.

    ``mutant`` plants one known mistake (see ``sdm_oracle.cpp``); it is used
    only by the tests that show the pins catch such mistakes.
    """
    out = Path(out) if out is not None else (LIBRARY if mutant == 0 else _HERE / f"liboracle_sdm_m{mutant}.so")
    if not force and out.exists() and out.stat().st_mtime >= SOURCE.stat().st_mtime:
        return out
    tmp = out.with_suffix(f".tmp{os.getpid()}.so")
    cmd = [
        "g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread",
        "-ffp-contract=off", "-fno-fast-math",
        f"-DORACLE_MUTANT={int(mutant)}", str(SOURCE), "-o", str(tmp),
    ]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(_c_ptr)


class Oracle:
    """ctypes front end of one compiled oracle library."""

    def __init__(self, path: Path | str | None = None):
        path = Path(path) if path is not None else build()
        self.path = path
        lib = ctypes.CDLL(str(path))
        lib.oracle_pkm_topk.restype = ctypes.c_int
        lib.oracle_pkm_topk.argtypes = [_c_ptr, _c_i64, _c_i32, _c_i32, _c_ptr, _c_ptr, _c_i32]
        lib.oracle_scan.restype = ctypes.c_int
        lib.oracle_scan.argtypes = [
            _c_i32, _c_i32, _c_i32, _c_i64, _c_i32, _c_i32, _c_i32,
            _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr,
            ctypes.c_double, _c_i32, _c_ptr, _c_ptr, _c_i32, ctypes.POINTER(_c_i64),
        ]
        lib.oracle_scan_f64.restype = ctypes.c_int
        lib.oracle_scan_f64.argtypes = [
            _c_i32, _c_i32, _c_i32, _c_i64, _c_i32, _c_i32, _c_i32,
            _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_i32,
        ]
        lib.oracle_scan_backward.restype = ctypes.c_int
        lib.oracle_scan_backward.argtypes = [
            _c_i32, _c_i32, _c_i32, _c_i64, _c_i32, _c_i32, _c_i32,
            _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr,
            _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_i32,
        ]
        lib.oracle_pkm_topk_backward.restype = ctypes.c_int
        lib.oracle_pkm_topk_backward.argtypes = [_c_i64, _c_i32, _c_i32, _c_ptr, _c_ptr, _c_ptr, _c_ptr]
        lib.oracle_rmsnorm_gate.restype = ctypes.c_int
        lib.oracle_rmsnorm_gate.argtypes = [_c_i64, _c_i32, _c_ptr, _c_ptr, ctypes.c_double]
        lib.oracle_rmsnorm_gate_backward.restype = ctypes.c_int
        lib.oracle_rmsnorm_gate_backward.argtypes = [_c_i64, _c_i32, _c_ptr, _c_ptr, _c_ptr, ctypes.c_double,
                                                     _c_ptr, _c_ptr]
        lib.oracle_round_e4m3.restype = ctypes.c_uint8
        lib.oracle_round_e4m3.argtypes = [ctypes.c_double]
        lib.oracle_decode_e4m3.restype = ctypes.c_double
        lib.oracle_decode_e4m3.argtypes = [ctypes.c_uint8]
        lib.oracle_quantize_fp8blk.restype = ctypes.c_int
        lib.oracle_quantize_fp8blk.argtypes = [_c_ptr, _c_i64, _c_ptr, _c_ptr]
        lib.oracle_scan_fp8blk.restype = ctypes.c_int
        lib.oracle_scan_fp8blk.argtypes = [
            _c_i32, _c_i32, _c_i32, _c_i64, _c_i32, _c_i32, _c_i32,
            _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_i32,
        ]
        lib.oracle_round_to_bf16.restype = ctypes.c_float
        lib.oracle_round_to_bf16.argtypes = [ctypes.c_double]
        self.lib = lib

    # -- selection ---------------------------------------------------------
    def pkm_topk(self, scores, K: int, n_threads: int | None = None):
        """Top-K slots of s1 (+) s2 for every leading index of ``scores``.

        scores: [..., 2*sqrt_n] float32.  Returns (idx int32 [..., K],
        w float64 [..., K]) in selection order.
        """
        s = _f32(scores)
        two_sqrt_n = s.shape[-1]
        if two_sqrt_n % 2:
            raise ValueError("last dimension must be 2*sqrt_n")
        sqrt_n = two_sqrt_n // 2
        lead = s.shape[:-1]
        n_units = int(np.prod(lead)) if lead else 1
        idx = np.empty(lead + (K,), dtype=np.int32)
        w = np.empty(lead + (K,), dtype=np.float64)
        rc = self.lib.oracle_pkm_topk(_p(s), n_units, sqrt_n, int(K), _p(idx), _p(w),
                                      n_threads or default_threads())
        if rc != 0:
            raise ValueError(f"oracle_pkm_topk rejected sqrt_n={sqrt_n} K={K}")
        return idx, w

    # -- recurrence ----------------------------------------------------------
    def scan(self, idx_w, w_w, idx_r, w_r, v, alpha, beta, M, g=None, eps: float = 1e-6,
             state_bf16: bool = False, n_threads: int | None = None):
        """Runs the write/read recurrence; returns (y float64, M_T float32, op_count).

        Shapes: idx_w, w_w [B,T,H,W]; idx_r, w_r [B,T,H,R]; v [B,T,H,d_v];
        alpha, beta [B,T,H]; M [B,H,N,d_v] (not modified; a copy is returned).
        """
        idx_w, idx_r = _i32(idx_w), _i32(idx_r)
        w_w, w_r = _f64(w_w), _f64(w_r)
        v, alpha, beta = _f32(v), _f32(alpha), _f32(beta)
        M_T = _f32(M).copy()
        B, T, H, W = idx_w.shape
        R = idx_r.shape[-1]
        d_v = v.shape[-1]
        N = M_T.shape[2]
        gg = None if g is None else _f32(g)
        y = np.zeros((B, T, H, d_v), dtype=np.float64)
        ops = _c_i64(0)
        rc = self.lib.oracle_scan(B, T, H, N, d_v, W, R, _p(idx_w), _p(w_w), _p(idx_r), _p(w_r),
                                  _p(v), _p(alpha), _p(beta), _p(gg), float(eps), int(bool(state_bf16)),
                                  _p(M_T), _p(y), n_threads or default_threads(), ctypes.byref(ops))
        if rc != 0:
            raise ValueError(f"oracle_scan failed with code {rc}")
        return y, M_T, int(ops.value)

    def scan_f64(self, idx_w, w_w, idx_r, w_r, v, alpha, beta, M, n_threads: int | None = None):
        """The recurrence with inputs and state in double, never rounded (no
        epilogue). Returns (y float64, M_T float64)."""
        idx_w, idx_r = _i32(idx_w), _i32(idx_r)
        w_w, w_r = _f64(w_w), _f64(w_r)
        v, alpha, beta = _f64(v), _f64(alpha), _f64(beta)
        M_T = _f64(M).copy()
        B, T, H, W = idx_w.shape
        R = idx_r.shape[-1]
        d_v = v.shape[-1]
        N = M_T.shape[2]
        y = np.zeros((B, T, H, d_v), dtype=np.float64)
        rc = self.lib.oracle_scan_f64(B, T, H, N, d_v, W, R, _p(idx_w), _p(w_w), _p(idx_r), _p(w_r),
                                      _p(v), _p(alpha), _p(beta), _p(M_T), _p(y), n_threads or default_threads())
        if rc != 0:
            raise ValueError(f"oracle_scan_f64 failed with code {rc}")
        return y, M_T

    def scan_backward(self, idx_w, w_w, idx_r, w_r, v, alpha, beta, M0, dy, dM_T=None,
                      n_threads: int | None = None):
        """Derivatives of L = sum <dy, y> + <dM_T, M_T> through the recurrence
        (scan_f64's function). Returns a dict with dv, dalpha, dbeta, dw_w,
        dw_r and dM0 (all float64)."""
        idx_w, idx_r = _i32(idx_w), _i32(idx_r)
        w_w, w_r = _f64(w_w), _f64(w_r)
        v, alpha, beta, M0, dy = _f64(v), _f64(alpha), _f64(beta), _f64(M0), _f64(dy)
        B, T, H, W = idx_w.shape
        R = idx_r.shape[-1]
        d_v = v.shape[-1]
        N = M0.shape[2]
        dM = np.zeros_like(M0) if dM_T is None else _f64(dM_T).copy()
        out = {"dv": np.zeros_like(v), "dalpha": np.zeros_like(alpha), "dbeta": np.zeros_like(beta),
               "dw_w": np.zeros_like(w_w), "dw_r": np.zeros_like(w_r)}
        rc = self.lib.oracle_scan_backward(B, T, H, N, d_v, W, R, _p(idx_w), _p(w_w), _p(idx_r), _p(w_r),
                                           _p(v), _p(alpha), _p(beta), _p(M0), _p(dy), _p(dM), _p(out["dv"]),
                                           _p(out["dalpha"]), _p(out["dbeta"]), _p(out["dw_w"]),
                                           _p(out["dw_r"]), n_threads or default_threads())
        if rc != 0:
            raise ValueError(f"oracle_scan_backward failed with code {rc}")
        out["dM0"] = dM
        return out

    def pkm_topk_backward(self, idx, w, dw, sqrt_n: int):
        """dL/dscores [..., 2*sqrt_n] of the selection weights for a fixed
        selection, given dL/dw."""
        idx, w, dw = _i32(idx), _f64(w), _f64(dw)
        lead = idx.shape[:-1]
        K = idx.shape[-1]
        n_units = int(np.prod(lead)) if lead else 1
        ds = np.zeros(lead + (2 * sqrt_n,), dtype=np.float64)
        rc = self.lib.oracle_pkm_topk_backward(n_units, int(sqrt_n), int(K), _p(idx), _p(w), _p(dw), _p(ds))
        if rc != 0:
            raise ValueError(f"oracle_pkm_topk_backward failed with code {rc}")
        return ds

    def rmsnorm_gate(self, x, g, eps: float = 1e-6):
        """The epilogue alone: g * x / sqrt(mean(x^2) + eps) over the last axis (double)."""
        y = _f64(x).copy()
        gg = _f64(g)
        d_v = y.shape[-1]
        rc = self.lib.oracle_rmsnorm_gate(y.size // d_v, d_v, _p(y), _p(gg), float(eps))
        if rc != 0:
            raise ValueError("oracle_rmsnorm_gate failed")
        return y

    def rmsnorm_gate_backward(self, x, g, dout, eps: float = 1e-6):
        """(dL/dx, dL/dg) of the epilogue for dL/dout; x is the row before it."""
        x, g, dout = _f64(x), _f64(g), _f64(dout)
        d_v = x.shape[-1]
        dx, dg = np.zeros_like(x), np.zeros_like(x)
        rc = self.lib.oracle_rmsnorm_gate_backward(x.size // d_v, d_v, _p(x), _p(g), _p(dout), float(eps), _p(dx),
                                                   _p(dg))
        if rc != 0:
            raise ValueError("oracle_rmsnorm_gate_backward failed")
        return dx, dg

    # -- block-scaled fp8 state ---------------------------------------------------
    def round_e4m3(self, x: float) -> int:
        return int(self.lib.oracle_round_e4m3(float(x)))

    def decode_e4m3(self, code: int) -> float:
        return float(self.lib.oracle_decode_e4m3(int(code)))

    def quantize_fp8blk(self, x):
        """Blocks of 16 fp32 values -> (codes uint8 [..., 16k], exps int8 [..., k])."""
        x = _f32(x)
        nb = x.size // 16
        codes = np.empty(x.shape, dtype=np.uint8)
        exps = np.empty(x.shape[:-1] + (x.shape[-1] // 16,), dtype=np.int8)
        self.lib.oracle_quantize_fp8blk(_p(x), nb, _p(codes), _p(exps))
        return codes, exps

    def dequantize_fp8blk(self, codes, exps):
        table = np.array([self.decode_e4m3(c) for c in range(256)])
        vals = table[np.asarray(codes)]
        return vals * np.ldexp(1.0, np.repeat(np.asarray(exps, dtype=np.int64), 16, axis=-1))

    def scan_fp8blk(self, idx_w, w_w, idx_r, w_r, v, alpha, beta, codes, exps, n_threads: int | None = None):
        """The recurrence on the block-scaled fp8 state (codes [B,H,N,d_v],
        exps [B,H,N,d_v/16], not modified). Returns (y float64, codes_T, exps_T)."""
        idx_w, idx_r = _i32(idx_w), _i32(idx_r)
        w_w, w_r = _f64(w_w), _f64(w_r)
        v, alpha, beta = _f32(v), _f32(alpha), _f32(beta)
        C = np.ascontiguousarray(codes, dtype=np.uint8).copy()
        X = np.ascontiguousarray(exps, dtype=np.int8).copy()
        B, T, H, W = idx_w.shape
        R = idx_r.shape[-1]
        d_v = v.shape[-1]
        N = C.shape[2]
        y = np.zeros((B, T, H, d_v), dtype=np.float64)
        rc = self.lib.oracle_scan_fp8blk(B, T, H, N, d_v, W, R, _p(idx_w), _p(w_w), _p(idx_r), _p(w_r), _p(v),
                                         _p(alpha), _p(beta), _p(C), _p(X), _p(y), n_threads or default_threads())
        if rc != 0:
            raise ValueError(f"oracle_scan_fp8blk failed with code {rc}")
        return y, C, X

    # -- whole layer ---------------------------------------------------------
    def layer_forward(self, kp, qp, v, alpha, beta, M0, W: int, R: int, g=None,
                      eps: float = 1e-6, state_bf16: bool = False, n_threads: int | None = None):
        """Selection on k' (top-W) and q' (top-R), M <- M0 for every batch row,
        then the recurrence. Returns a dict with idx_w, w_w, idx_r, w_r, y, M_T."""
        idx_w, w_w = self.pkm_topk(kp, W, n_threads)
        idx_r, w_r = self.pkm_topk(qp, R, n_threads)
        M0 = _f32(M0)
        B = np.asarray(kp).shape[0]
        M = np.ascontiguousarray(np.broadcast_to(M0[None], (B,) + M0.shape))
        y, M_T, ops = self.scan(idx_w, w_w, idx_r, w_r, v, alpha, beta, M, g=g, eps=eps,
                                state_bf16=state_bf16, n_threads=n_threads)
        return {"idx_w": idx_w, "w_w": w_w, "idx_r": idx_r, "w_r": w_r, "y": y, "M_T": M_T,
                "ops": ops}

    def round_to_bf16(self, x: float) -> float:
        return float(self.lib.oracle_round_to_bf16(float(x)))


_DEFAULT: Oracle | None = None


def get() -> Oracle:
    """Returns the (lazily built) unmodified oracle."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle(build())
    return _DEFAULT
