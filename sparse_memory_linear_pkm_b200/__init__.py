"""B200-native (sm_100a) Sparse Delta Memory recurrent core.

Python front end of the C ABI in include/sdm.h. Tensors are torch CUDA tensors
(torch provides device memory and the current stream); every step of the
computation runs in libsdm_b200.so, which must be built
(``python -m sparse_memory_linear_pkm_b200.build``). There is no CPU path.

    y, M_T = layer_forward(kp, qp, v, alpha, beta, M0, W=64, R=64)

Layouts: kp, qp [B,T,H,2*sqrt_n]; v, g [B,T,H,d_v]; alpha, beta [B,T,H];
M0 [H,N,d_v]; M [B,H,N,d_v]; y [B,T,H,d_v] fp32; idx, w [B,T,H,K].
"""

from __future__ import annotations

import ctypes

import torch

from . import native, synth
from .native import SdmError

__all__ = ["pkm_topk", "scan", "state_init", "layer_forward", "layer_step", "slot_counts", "scan_describe",
           "scan_backward", "pkm_topk_backward", "rmsnorm_gate", "rmsnorm_gate_backward", "layer_backward",
           "quantize_fp8blk", "fp8blk_parts", "stream_check", "make_shape", "layer_checkpoint_size", "layer_forward_ckpt",
           "scan_workspace_bytes", "layer_forward_workspace_bytes", "scan_variant", "SdmError", "synth", "native"]

_DTYPE = {torch.float32: native.F32, torch.bfloat16: native.BF16,
          torch.uint8: native.FP8_B16}  # a uint8 state buffer holds the block-scaled fp8 state


def _code(t: torch.Tensor, what: str) -> int:
    try:
        return _DTYPE[t.dtype]
    except KeyError:
        raise TypeError(f"{what} must be float32 or bfloat16, got {t.dtype}") from None


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def make_shape(B, T, H, sqrt_n, W, R, d_v, in_dtype=torch.bfloat16, state_dtype=torch.float32,
               rms_eps: float = 1e-6, variant: str = "auto", tile: int = 0) -> native.Shape:
    return native.Shape(B, T, H, sqrt_n, W, R, d_v, _DTYPE[in_dtype], _DTYPE[state_dtype], rms_eps,
                        native.VARIANTS[variant], tile)


def scan_variant(shape: native.Shape) -> str:
    """'resident', 'streaming' or 'pipelined': the recurrence kernel this shape runs on the current device."""
    v = int(native.load().sdm_scan_variant(ctypes.byref(shape)))
    if v < 0:
        native.check(1)
    return {1: "resident", 2: "streaming", 3: "pipelined"}[v]


def scan_describe(shape: native.Shape) -> str:
    """The recurrence kernel's launch configuration for this shape, as text."""
    buf = ctypes.create_string_buffer(128)
    native.check(native.load().sdm_scan_describe(ctypes.byref(shape), buf, len(buf)))
    return buf.value.decode()


def scan_workspace_bytes(shape: native.Shape) -> int:
    return int(native.load().sdm_scan_workspace_bytes(ctypes.byref(shape)))


def layer_forward_workspace_bytes(shape: native.Shape) -> int:
    return int(native.load().sdm_layer_forward_workspace_bytes(ctypes.byref(shape)))


def layer_forward_chunks(shape: native.Shape) -> int:
    """Token chunks a layer_forward call of this shape runs as (1: one pass; more: overlapped)."""
    n = int(native.load().sdm_layer_forward_chunks(ctypes.byref(shape)))
    if n < 0:
        native.check(1)
    return n


def _workspace(nbytes: int, device, workspace: torch.Tensor | None) -> torch.Tensor:
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace needs {nbytes} bytes")
        return workspace
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def pkm_topk(scores: torch.Tensor, K: int):
    """Product-key top-K of s1 (+) s2 per token-head; returns (idx int32, w fp32)."""
    B, T, H, two_n = scores.shape
    lib = native.load()
    idx = torch.empty((B, T, H, K), dtype=torch.int32, device=scores.device)
    w = torch.empty((B, T, H, K), dtype=torch.float32, device=scores.device)
    native.check(lib.sdm_pkm_topk(_ptr(scores), _code(scores, "scores"), B, T, H, two_n // 2, K, _ptr(idx),
                                  _ptr(w), _stream(scores.device)))
    return idx, w


def scan(idx_w, w_w, idx_r, w_r, v, alpha, beta, M, g=None, eps: float = 1e-6, variant: str = "auto",
         y: torch.Tensor | None = None, workspace: torch.Tensor | None = None, tile: int = 0) -> torch.Tensor:
    """The write/read recurrence over a given selection. M [B,H,N,d_v] is
    updated in place (M_0 -> M_T); returns y [B,T,H,d_v] fp32."""
    B, T, H, W = idx_w.shape
    R = idx_r.shape[-1]
    d_v = v.shape[-1]
    N = M.shape[2]
    sqrt_n = int(round(N ** 0.5))
    shape = native.Shape(B, T, H, sqrt_n, W, R, d_v, _code(v, "v"), _code(M, "M"), eps, native.VARIANTS[variant],
                         tile)
    lib = native.load()
    if y is None:
        y = torch.empty((B, T, H, d_v), dtype=torch.float32, device=v.device)
    ws = _workspace(scan_workspace_bytes(shape), v.device, workspace)
    native.check(lib.sdm_scan(ctypes.byref(shape), _ptr(idx_w), _ptr(w_w), _ptr(idx_r), _ptr(w_r), _ptr(v),
                              _ptr(alpha), _ptr(beta), _ptr(g), _ptr(M), _ptr(y), _ptr(ws),
                              ws.numel() * ws.element_size(), _stream(v.device)))
    return y


def scan_backward_workspace_bytes(shape: native.Shape) -> int:
    lib = native.load()
    n = int(lib.sdm_scan_backward_workspace_bytes(ctypes.byref(shape)))
    msg = lib.sdm_last_error().decode(errors="replace")
    if n == 0 and msg:
        raise native.SdmError(2, msg)
    return n


def scan_backward(idx_w, w_w, idx_r, w_r, v, alpha, beta, M_in, dy, dM: torch.Tensor | None = None,
                  workspace: torch.Tensor | None = None) -> dict:
    """Derivatives of the recurrence (no epilogue) for dy = dL/dy and
    dM = dL/dM_T (zeros when None). M_in is the fp32 state the forward started
    from, [B,H,N,d_v] or [H,N,d_v] shared by the batch. Returns a dict with
    dv, dalpha, dbeta, dw_w, dw_r (fp32) and dM0 = dL/dM_0 per batch row
    [B,H,N,d_v] (``dM`` itself when given, updated in place)."""
    B, T, H, W = idx_w.shape
    R = idx_r.shape[-1]
    d_v = v.shape[-1]
    N = M_in.shape[-2]
    sqrt_n = int(round(N ** 0.5))
    shared = M_in.dim() == 3
    dev = v.device
    shape = native.Shape(B, T, H, sqrt_n, W, R, d_v, _code(v, "v"), _code(M_in, "M_in"), 1e-6, 0)
    lib = native.load()
    if dM is None:
        dM = torch.zeros((B, H, N, d_v), dtype=torch.float32, device=dev)
    out = {"dv": torch.empty((B, T, H, d_v), dtype=torch.float32, device=dev),
           "dalpha": torch.empty((B, T, H), dtype=torch.float32, device=dev),
           "dbeta": torch.empty((B, T, H), dtype=torch.float32, device=dev),
           "dw_w": torch.empty((B, T, H, W), dtype=torch.float32, device=dev),
           "dw_r": torch.empty((B, T, H, R), dtype=torch.float32, device=dev)}
    ws = _workspace(scan_backward_workspace_bytes(shape), dev, workspace)
    native.check(lib.sdm_scan_backward(ctypes.byref(shape), _ptr(idx_w), _ptr(w_w), _ptr(idx_r), _ptr(w_r), _ptr(v),
                                       _ptr(alpha), _ptr(beta), _ptr(M_in), int(shared), _ptr(dy), _ptr(dM),
                                       _ptr(out["dv"]), _ptr(out["dalpha"]), _ptr(out["dbeta"]), _ptr(out["dw_w"]),
                                       _ptr(out["dw_r"]), _ptr(ws), ws.numel() * ws.element_size(), _stream(dev)))
    out["dM0"] = dM
    return out


def pkm_topk_backward(idx: torch.Tensor, w: torch.Tensor, dw: torch.Tensor, sqrt_n: int,
                      dscores: torch.Tensor | None = None) -> torch.Tensor:
    """dL/dscores [B,T,H,2*sqrt_n] fp32 of the selection weights (fixed selection)."""
    B, T, H, K = idx.shape
    if dscores is None:
        dscores = torch.empty((B, T, H, 2 * sqrt_n), dtype=torch.float32, device=idx.device)
    native.check(native.load().sdm_pkm_topk_backward(_ptr(idx), _ptr(w), _ptr(dw), B, T, H, sqrt_n, K,
                                                      _ptr(dscores), _stream(idx.device)))
    return dscores


def rmsnorm_gate(y: torch.Tensor, g: torch.Tensor, eps: float = 1e-6) -> torch.Tensor:
    """The RMS-norm x gate epilogue in place on y [..., d_v] fp32; returns y."""
    d_v = y.shape[-1]
    native.check(native.load().sdm_rmsnorm_gate(_ptr(y), _ptr(g), _code(g, "g"), y.numel() // d_v, d_v,
                                                float(eps), _stream(y.device)))
    return y


def row_sumsq(y: torch.Tensor) -> torch.Tensor:
    """Sum of squares over the last axis of y [..., d] fp32 (fixed order); shape y.shape[:-1]."""
    d = y.shape[-1]
    ss = torch.empty(y.shape[:-1], dtype=torch.float32, device=y.device)
    native.check(native.load().sdm_row_sumsq(_ptr(y), y.numel() // d, d, _ptr(ss), _stream(y.device)))
    return ss


def rmsnorm_gate_rows(y: torch.Tensor, g: torch.Tensor, ss: torch.Tensor, d_total: int,
                      eps: float = 1e-6) -> torch.Tensor:
    """The epilogue in place on a column slice y [..., d] of rows of d_total
    values, given the full rows' sums of squares ss [...]; returns y."""
    d = y.shape[-1]
    native.check(native.load().sdm_rmsnorm_gate_rows(_ptr(y), _ptr(g), _code(g, "g"), _ptr(ss), y.numel() // d, d,
                                                     int(d_total), float(eps), _stream(y.device)))
    return y


def rmsnorm_gate_backward(y_pre: torch.Tensor, g: torch.Tensor, dout: torch.Tensor, eps: float = 1e-6):
    """(dL/dy_pre, dL/dg) of the epilogue for dL/dout; y_pre is the row before it."""
    d_v = y_pre.shape[-1]
    dy_pre = torch.empty_like(y_pre)
    dg = torch.empty(y_pre.shape, dtype=torch.float32, device=y_pre.device)
    native.check(native.load().sdm_rmsnorm_gate_backward(_ptr(y_pre), _ptr(g), _code(g, "g"), _ptr(dout),
                                                         y_pre.numel() // d_v, d_v, float(eps), _ptr(dy_pre),
                                                         _ptr(dg), _stream(y_pre.device)))
    return dy_pre, dg


def layer_checkpoint_size(shape: native.Shape) -> tuple[int, int]:
    """(chunk tokens C, bytes) of the checkpoints sdm_layer_forward_ckpt stores
    for a later backward of this shape; raises SdmError where the forward does
    not store them."""
    chunk, nbytes = ctypes.c_int32(0), ctypes.c_size_t(0)
    native.check(native.load().sdm_layer_checkpoint_size(ctypes.byref(shape), ctypes.byref(chunk), ctypes.byref(nbytes)))
    return int(chunk.value), int(nbytes.value)


def layer_forward_ckpt(kp, qp, v, alpha, beta, M0, W: int, R: int, g=None, eps: float = 1e-6,
                       workspace: torch.Tensor | None = None):
    """layer_forward that also stores the backward's checkpoints (the state
    before every chunk of C tokens after the first, [n-1,B,H,N,d_v] fp32).
    Returns (y, M_out, checkpoints)."""
    B, T, H, two_n = kp.shape
    d_v = v.shape[-1]
    shape = native.Shape(B, T, H, two_n // 2, W, R, d_v, _code(kp, "kp"), _code(M0, "M0"), eps, 0, 0)
    lib = native.load()
    chunk, nbytes = layer_checkpoint_size(shape)
    y = torch.empty((B, T, H, d_v), dtype=torch.float32, device=kp.device)
    M_out = torch.empty((B,) + tuple(M0.shape), dtype=M0.dtype, device=kp.device)
    ckpt = torch.empty((max(nbytes, 16) // 4,), dtype=torch.float32, device=kp.device)
    ws = _workspace(layer_forward_workspace_bytes(shape), kp.device, workspace)
    native.check(lib.sdm_layer_forward_ckpt(ctypes.byref(shape), _ptr(kp), _ptr(qp), _ptr(v), _ptr(alpha), _ptr(beta),
                                            _ptr(g), _ptr(M0), _ptr(M_out), _ptr(y), _ptr(ckpt), nbytes, _ptr(ws),
                                            ws.numel() * ws.element_size(), _stream(kp.device)))
    return y, M_out, ckpt[:nbytes // 4]


def layer_backward(kp, qp, v, alpha, beta, M0, dy, W: int, R: int, g=None, y_pre=None, dM=None, eps: float = 1e-6,
                   workspace: torch.Tensor | None = None, checkpoints: torch.Tensor | None = None) -> dict:
    """Derivatives of the layer (selection, recurrence, optional epilogue)
    for dy = dL/d(output) and dM = dL/dM_T (zeros when None); M0 [H,N,d_v]
    fp32 is the shared initial state; y_pre (the output before the epilogue)
    is needed with g. Returns dkp, dqp, dv, dalpha, dbeta, dM0 (per batch row)
    and, with g, dg (all fp32). ``checkpoints``: the ones layer_forward_ckpt
    stored for the same inputs (the backward then skips recomputing them)."""
    B, T, H, two_n = kp.shape
    d_v = v.shape[-1]
    N = M0.shape[-2]
    dev = kp.device
    shape = native.Shape(B, T, H, two_n // 2, W, R, d_v, _code(kp, "kp"), _code(M0, "M0"), eps, 0)
    lib = native.load()
    if dM is None:
        dM = torch.zeros((B, H, N, d_v), dtype=torch.float32, device=dev)
    f = lambda *sh: torch.empty(sh, dtype=torch.float32, device=dev)
    out = {"dkp": f(B, T, H, two_n), "dqp": f(B, T, H, two_n), "dv": f(B, T, H, d_v), "dalpha": f(B, T, H),
           "dbeta": f(B, T, H)}
    if g is not None:
        out["dg"] = f(B, T, H, d_v)
    need = int(lib.sdm_layer_backward_workspace_bytes(ctypes.byref(shape)))
    if need == 0:
        raise native.SdmError(2, lib.sdm_last_error().decode(errors="replace"))
    ws = _workspace(need, dev, workspace)
    ck_bytes = 0 if checkpoints is None else checkpoints.numel() * checkpoints.element_size()
    native.check(lib.sdm_layer_backward_ckpt(ctypes.byref(shape), _ptr(kp), _ptr(qp), _ptr(v), _ptr(alpha),
                                             _ptr(beta), _ptr(g), _ptr(M0), _ptr(y_pre), _ptr(dy), _ptr(dM),
                                             _ptr(out["dkp"]), _ptr(out["dqp"]), _ptr(out["dv"]), _ptr(out["dalpha"]),
                                             _ptr(out["dbeta"]), _ptr(out.get("dg")), _ptr(checkpoints), ck_bytes,
                                             _ptr(ws), ws.numel() * ws.element_size(), _stream(dev)))
    out["dM0"] = dM
    return out


def quantize_fp8blk(x: torch.Tensor) -> torch.Tensor:
    """A block-scaled fp8 state buffer (uint8: the E4M3 codes of x, then one
    int8 exponent per 16 values) from fp32 x [..., d_v] with d_v a multiple of
    16; pass it as the state M of layer_step (T = 1)."""
    n = x.numel()
    if n % 16:
        raise ValueError("the number of values must be a multiple of 16")
    buf = torch.empty(n + n // 16, dtype=torch.uint8, device=x.device)
    native.check(native.load().sdm_quantize_fp8blk(_ptr(x), n // 16, _ptr(buf), ctypes.c_void_p(buf.data_ptr() + n),
                                                   _stream(x.device)))
    return buf


def fp8blk_parts(buf: torch.Tensor, n_values: int):
    """(codes uint8 [n_values], exps int8 [n_values // 16]) views of a fp8 state buffer."""
    return buf[:n_values], buf[n_values:].view(torch.int8)


def state_init(M0: torch.Tensor, B: int, out: torch.Tensor | None = None) -> torch.Tensor:
    """M[b] <- M0 for b in [0, B)."""
    H, N, d_v = M0.shape
    sqrt_n = int(round(N ** 0.5))
    M = out if out is not None else torch.empty((B, H, N, d_v), dtype=M0.dtype, device=M0.device)
    shape = native.Shape(B, 1, H, sqrt_n, 1, 1, d_v, native.F32, _code(M0, "M0"), 1e-6, 0)
    native.check(native.load().sdm_state_init(ctypes.byref(shape), _ptr(M0), _ptr(M), _stream(M0.device)))
    return M


def slot_counts(idx: torch.Tensor, N: int, counts: torch.Tensor | None = None) -> torch.Tensor:
    """Per-slot selection counts: counts[b,h,i] += #{(t,k): idx[b,t,h,k] == i};
    idx [B,T,H,K] int32. Returns counts [B,H,N] int32 (accumulated into
    `counts` when given)."""
    B, T, H, K = idx.shape
    if counts is None:
        counts = torch.zeros((B, H, N), dtype=torch.int32, device=idx.device)
    native.check(native.load().sdm_slot_counts(_ptr(idx), B, T, H, K, N, _ptr(counts), _stream(idx.device)))
    return counts


def layer_step(kp, qp, v, alpha, beta, M, W: int, R: int, g=None, eps: float = 1e-6, variant: str = "auto",
               y: torch.Tensor | None = None, workspace: torch.Tensor | None = None, tile: int = 0) -> torch.Tensor:
    """Selection and recurrence over T tokens continuing from the state in M
    [B,H,N,d_v], which is updated in place (decode: T = 1 per call). Returns y."""
    B, T, H, two_n = kp.shape
    d_v = v.shape[-1]
    shape = native.Shape(B, T, H, two_n // 2, W, R, d_v, _code(kp, "kp"), _code(M, "M"), eps,
                         native.VARIANTS[variant], tile)
    lib = native.load()
    if y is None:
        y = torch.empty((B, T, H, d_v), dtype=torch.float32, device=kp.device)
    ws = _workspace(int(lib.sdm_layer_step_workspace_bytes(ctypes.byref(shape))), kp.device, workspace)
    native.check(lib.sdm_layer_step(ctypes.byref(shape), _ptr(kp), _ptr(qp), _ptr(v), _ptr(alpha), _ptr(beta),
                                    _ptr(g), _ptr(M), _ptr(y), _ptr(ws), ws.numel() * ws.element_size(),
                                    _stream(kp.device)))
    return y


def layer_forward(kp, qp, v, alpha, beta, M0, W: int, R: int, g=None, eps: float = 1e-6,
                  variant: str = "auto", y: torch.Tensor | None = None, M_out: torch.Tensor | None = None,
                  workspace: torch.Tensor | None = None, events=None, tile: int = 0):
    """Selection (top-W of k', top-R of q'), M_out <- M0 per batch row, the
    recurrence and the optional RMS-norm x g epilogue. Returns (y, M_out).

    ``events``: optional list of 6 already-created torch.cuda.Event objects
    recorded between the stages, or 6 + 2 per chunk of an overlapped call
    (see sdm_layer_forward_traced in sdm.h)."""
    B, T, H, two_n = kp.shape
    d_v = v.shape[-1]
    shape = native.Shape(B, T, H, two_n // 2, W, R, d_v, _code(kp, "kp"), _code(M0, "M0"), eps,
                         native.VARIANTS[variant], tile)
    lib = native.load()
    if y is None:
        y = torch.empty((B, T, H, d_v), dtype=torch.float32, device=kp.device)
    if M_out is None:
        M_out = torch.empty((B,) + tuple(M0.shape), dtype=M0.dtype, device=kp.device)
    ws = _workspace(layer_forward_workspace_bytes(shape), kp.device, workspace)
    if events is None:
        ev, n_ev = None, 0
    else:
        if len(events) < 6 or len(events) % 2:
            raise ValueError("events must hold 6 (+ 2 a chunk) torch.cuda.Event objects")
        ev, n_ev = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events]), len(events)
    native.check(lib.sdm_layer_forward_traced(ctypes.byref(shape), _ptr(kp), _ptr(qp), _ptr(v), _ptr(alpha),
                                              _ptr(beta), _ptr(g), _ptr(M0), _ptr(M_out), _ptr(y), _ptr(ws),
                                              ws.numel() * ws.element_size(), _stream(kp.device), ev, n_ev))
    return y, M_out


def stream_check(device: torch.device | None = None) -> None:
    """Synchronises the current stream and raises SdmError if a kernel set the
    device error word (an index outside [0, N), an expired bounded wait)."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    native.check(native.load().sdm_stream_check(_stream(device)))
