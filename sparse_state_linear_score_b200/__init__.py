"""Sparse Delta Memory (SDM) hot path on NVIDIA B200 — Python binding of libsdm.so.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels (see include/sdm.h).  PyTorch provides device memory and streams.  There
is no CPU fallback: importing this package without a loadable libsdm.so raises.

Typical use::

    import sparse_state_linear_score_b200 as sdm
    d = sdm.Dims(B, H, T, d_k, n_sub, d_v, k_half, W, R, x_dtype="bf16", v_dtype="bf16")
    st = sdm.State(d, M0)                      # M0: [H, N, d_v] fp32 on the GPU
    sdm.state_reset(d, st)
    out, sel = sdm.prefill(d, q, k, v, alpha, beta, skw, skr, st)
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

__all__ = ["Dims", "State", "SdmError", "state_reset", "state_materialize", "score_topk", "score_qk",
           "forward_workspace_bytes", "forward", "forward_noalloc", "forward_plan", "forward_run",
           "forward_run_gated", "prefill",
           "decode_step", "device_error", "weight_stats", "gemm_bf16", "layer_in", "layer_out", "lib_path",
           "DEVERR_SLOT_RANGE",
           "DEVERR_DUP_WRITE", "DEVERR_ALPHA"]

F32, BF16 = 0, 1
_DT = {"f32": F32, "bf16": BF16, torch.float32: F32, torch.bfloat16: BF16}
DEVERR_SLOT_RANGE, DEVERR_DUP_WRITE, DEVERR_ALPHA = 1, 2, 4


class SdmError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_lib.sdm_status_str(status).decode()}")


DECAY_ALL, DECAY_TOUCHED = 0, 1
_DECAY = {"all": DECAY_ALL, "touched": DECAY_TOUCHED}


class Dims(ctypes.Structure):
    """sdm_dims.  decay: "all" (alpha scales every slot at every token) or "touched"
    (only the token's write slots); see sdm_decay in include/sdm.h."""
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "H", "T", "d_k", "n_sub", "d_v", "k_half", "W", "R", "x_dtype", "v_dtype",
                 "decay")]

    def __init__(self, B, H, T, d_k, n_sub, d_v, k_half, W, R, x_dtype="f32", v_dtype="f32",
                 decay="all"):
        super().__init__(B, H, T, d_k, n_sub, d_v, k_half, W, R, _DT[x_dtype], _DT[v_dtype],
                         _DECAY[decay])

    @property
    def N(self) -> int:
        return self.n_sub * self.n_sub

    def with_T(self, T: int) -> "Dims":
        x = Dims(self.B, self.H, T, self.d_k, self.n_sub, self.d_v, self.k_half, self.W, self.R)
        x.x_dtype, x.v_dtype, x.decay = self.x_dtype, self.v_dtype, self.decay
        return x


class _CState(ctypes.Structure):
    _fields_ = [("M", ctypes.c_void_p), ("stamp", ctypes.c_void_p), ("Lambda", ctypes.c_void_p),
                ("M0", ctypes.c_void_p)]


def _load():
    path = _build.LIB
    if not os.path.exists(path) or not _build.up_to_date():
        _build.build()  # raises if nvcc fails: no fallback path exists
    lib = ctypes.CDLL(path)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    D = ctypes.POINTER(Dims)
    S = ctypes.POINTER(_CState)
    sig = {
        "sdm_status_str": ([I32], ctypes.c_char_p),
        "sdm_abi_version": ([], I32),
        "sdm_state_bytes": ([D, P, P, P], I32),
        "sdm_state_reset": ([D, S, P], I32),
        "sdm_state_materialize": ([D, S, P, P], I32),
        "sdm_score_topk": ([D, P, P, I32, P, P, P], I32),
        "sdm_score_qk": ([D, P, P, P, P, P, P, P, P, P], I32),
        "sdm_score_path": ([D, I32], I32),
        "sdm_decode_path": ([D], I32),
        "sdm_forward_workspace_bytes": ([D], SZ),
        "sdm_forward": ([D, P, P, P, P, P, P, P, S, P, P, SZ, P], I32),
        "sdm_forward_plan": ([D, P, P, P, P, P, P, S, P, SZ, P], I32),
        "sdm_forward_run": ([D, P, P, P, P, P, P, S, P, P, SZ, P], I32),
        "sdm_forward_run_gated": ([D, P, P, P, P, P, P, S, P, P, P, ctypes.c_float, P, P, SZ, P],
                                  I32),
        "sdm_prefill": ([D, P, P, P, P, P, P, P, S, P, P, P, P, P, P, SZ, P], I32),
        "sdm_decode_step": ([D, P, P, P, P, P, P, P, S, P, P, P, P, P, P], I32),
        "sdm_device_error": ([ctypes.POINTER(ctypes.c_uint32), I32, P], I32),
        "sdm_forward_noalloc": ([D, P, P, P, P, P, P, P, S, P, P], I32),
        "sdm_backward_workspace_bytes": ([D], SZ),
        "sdm_call_log_bytes": ([D], SZ),
        "sdm_call_log_save": ([D, P, S, P, SZ, P], I32),
        "sdm_call_log_restore": ([D, P, P, SZ, S, P], I32),
        "sdm_score_backward": ([D, P, P, I32, P, P, P, P, P, P], I32),
        "sdm_backward": ([D, P, P, P, P, P, P, P, S, P, P, P, P, P, P, P, P, P, SZ, P], I32),
        "sdm_gemm_bf16": ([I32, I32, I32, P, P, P, P], I32),
        "sdm_layer_in_workspace_bytes": ([D], SZ),
        "sdm_layer_in": ([D, P, P, P, P, I32, P, P, P, P, P, P, P, SZ, P], I32),
        "sdm_layer_out_workspace_bytes": ([D], SZ),
        "sdm_layer_out": ([D, P, P, P, ctypes.c_float, P, I32, P, P, SZ, P], I32),
        "sdm_weight_stats_workspace_bytes": ([ctypes.c_int64, I32], SZ),
        "sdm_weight_stats": ([ctypes.c_int64, I32, P, P, P, P, I32, P, P, P, SZ, P], I32),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


_lib = _load()


def lib_path() -> str:
    return _build.LIB


def _ptr(t: torch.Tensor | None, what: str, dtype=None):
    """Device address of a contiguous CUDA tensor (an int: the argtypes convert it)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
_cur_device = getattr(torch._C, "_cuda_getDevice", None)


def _stream(stream=None):
    """cudaStream_t of `stream`, else of the current stream (without building a Stream)."""
    if stream is not None:
        return stream.cuda_stream
    if _raw_stream is not None and _cur_device is not None:
        return _raw_stream(_cur_device())
    return torch.cuda.current_stream().cuda_stream


def _ok(status: int, what: str):
    if status != 0:
        raise SdmError(status, what)


def _xdt(d: Dims):
    return torch.float32 if d.x_dtype == F32 else torch.bfloat16


def _vdt(d: Dims):
    return torch.float32 if d.v_dtype == F32 else torch.bfloat16


class State:
    """Lazy-decay memory state of B*H sequences (see include/sdm.h, sdm_state)."""

    def __init__(self, d: Dims, M0: torch.Tensor, device=None):
        device = M0.device if device is None else device
        self.M = torch.empty((d.B, d.H, d.N, d.d_v), dtype=torch.float32, device=device)
        self.stamp = torch.empty((d.B, d.H, d.N), dtype=torch.float64, device=device)
        self.Lambda = torch.zeros((d.B, d.H), dtype=torch.float64, device=device)
        if tuple(M0.shape) != (d.H, d.N, d.d_v):
            raise ValueError(f"M0 must be [H, N, d_v] = {(d.H, d.N, d.d_v)}")
        self.M0 = M0
        self._c = _CState(_ptr(self.M, "M", torch.float32), _ptr(self.stamp, "stamp", torch.float64),
                          _ptr(self.Lambda, "Lambda", torch.float64), _ptr(M0, "M0", torch.float32))

    @property
    def c(self) -> _CState:
        return self._c


def state_reset(d: Dims, st: State, stream=None):
    _ok(_lib.sdm_state_reset(ctypes.byref(d), ctypes.byref(st.c), _stream(stream)), "sdm_state_reset")


def state_materialize(d: Dims, st: State, out: torch.Tensor | None = None, stream=None):
    if out is None:
        out = torch.empty_like(st.M)
    _ok(_lib.sdm_state_materialize(ctypes.byref(d), ctypes.byref(st.c), _ptr(out, "out"),
                                   _stream(stream)), "sdm_state_materialize")
    return out


def call_log_bytes(d: Dims) -> int:
    return int(_lib.sdm_call_log_bytes(ctypes.byref(d)))


def call_log_save(d: Dims, widx, st: State, log=None, stream=None):
    """sdm_call_log_save: before a call with write slots widx [B,H,T,W], record the rows,
    stamps and Lambda it will overwrite.  Returns the log (uint8 device tensor)."""
    if log is None:
        log = torch.empty(max(16, call_log_bytes(d)), dtype=torch.uint8, device=st.M.device)
    _ok(_lib.sdm_call_log_save(ctypes.byref(d), _ptr(widx, "widx", torch.int32),
                               ctypes.byref(st.c), _ptr(log, "log"), log.numel(),
                               _stream(stream)), "sdm_call_log_save")
    return log


def call_log_restore(d: Dims, widx, log, st: State, stream=None):
    """sdm_call_log_restore: after the call, put back the state it started from."""
    _ok(_lib.sdm_call_log_restore(ctypes.byref(d), _ptr(widx, "widx", torch.int32),
                                  _ptr(log, "log"), log.numel(), ctypes.byref(st.c),
                                  _stream(stream)), "sdm_call_log_restore")


def score_topk(d: Dims, x, subkeys, top: int, idx=None, w=None, stream=None):
    shape = (d.B, d.H, d.T, top)
    if idx is None:
        idx = torch.empty(shape, dtype=torch.int32, device=x.device)
    if w is None:
        w = torch.empty(shape, dtype=torch.float32, device=x.device)
    _ok(_lib.sdm_score_topk(ctypes.byref(d), _ptr(x, "x", _xdt(d)), _ptr(subkeys, "subkeys", _xdt(d)),
                            top, _ptr(idx, "idx", torch.int32), _ptr(w, "w", torch.float32),
                            _stream(stream)), "sdm_score_topk")
    return idx, w


SCORE_TC, SCORE_ROWS, SCORE_WARP = 1, 2, 3


def score_path(d: Dims, top: int) -> int:
    """sdm_score_path: the scoring kernel a call of these dims launches (SCORE_TC: the
    tensor-core kernel, SCORE_ROWS: the row scorer, SCORE_WARP: one warp per row)."""
    r = int(_lib.sdm_score_path(ctypes.byref(d), top))
    if r < 0:
        raise SdmError(-r, "sdm_score_path")
    return r


DECODE_FUSED, DECODE_TWO = 1, 2


def decode_path(d: Dims) -> int:
    """sdm_decode_path: DECODE_FUSED when decode_step is one launch (scoring and recurrence
    step in the same CTAs), DECODE_TWO when it is a scoring launch and a recurrence launch."""
    r = int(_lib.sdm_decode_path(ctypes.byref(d)))
    if r < 0:
        raise SdmError(-r, "sdm_decode_path")
    return r


def score_qk(d: Dims, q, k, skw, skr, sel=None, stream=None):
    """sdm_score_qk: both roles of one call.  Returns (widx, ww, ridx, rw)."""
    if sel is None:
        sel = selection_buffers(d, q.device)
    widx, ww, ridx, rw = sel
    xdt = _xdt(d)
    _ok(_lib.sdm_score_qk(ctypes.byref(d), _ptr(q, "q", xdt), _ptr(k, "k", xdt),
                          _ptr(skw, "skw", xdt), _ptr(skr, "skr", xdt),
                          _ptr(widx, "widx", torch.int32), _ptr(ww, "ww", torch.float32),
                          _ptr(ridx, "ridx", torch.int32), _ptr(rw, "rw", torch.float32),
                          _stream(stream)), "sdm_score_qk")
    return sel


def forward_workspace_bytes(d: Dims) -> int:
    return int(_lib.sdm_forward_workspace_bytes(ctypes.byref(d)))


def workspace(d: Dims, device="cuda") -> torch.Tensor:
    return torch.empty(max(16, forward_workspace_bytes(d)), dtype=torch.uint8, device=device)


def _fw_args(d, v, alpha, beta, widx, ww, ridx, rw):
    return (_ptr(v, "v", _vdt(d)), _ptr(alpha, "alpha", torch.float32), _ptr(beta, "beta", torch.float32),
            _ptr(widx, "widx", torch.int32), _ptr(ww, "ww", torch.float32),
            _ptr(ridx, "ridx", torch.int32), _ptr(rw, "rw", torch.float32))


def forward(d: Dims, v, alpha, beta, widx, ww, ridx, rw, st: State, out=None, ws=None, stream=None):
    if out is None:
        out = torch.empty((d.B, d.H, d.T, d.d_v), dtype=torch.float32, device=v.device)
    if ws is None:
        ws = workspace(d, v.device)
    a = _fw_args(d, v, alpha, beta, widx, ww, ridx, rw)
    _ok(_lib.sdm_forward(ctypes.byref(d), *a, ctypes.byref(st.c), _ptr(out, "out", torch.float32),
                         _ptr(ws, "ws"), ws.numel(), _stream(stream)), "sdm_forward")
    return out


def forward_noalloc(d: Dims, v, alpha, beta, widx, ww, ridx, rw, st: State, out=None, stream=None):
    """sdm_forward with the library's fixed 64 MiB device scratch instead of a workspace."""
    if out is None:
        out = torch.empty((d.B, d.H, d.T, d.d_v), dtype=torch.float32, device=v.device)
    a = _fw_args(d, v, alpha, beta, widx, ww, ridx, rw)
    _ok(_lib.sdm_forward_noalloc(ctypes.byref(d), *a, ctypes.byref(st.c),
                                 _ptr(out, "out", torch.float32), _stream(stream)),
        "sdm_forward_noalloc")
    return out


def forward_plan(d: Dims, alpha, beta, widx, ww, ridx, rw, st: State, ws, stream=None):
    _ok(_lib.sdm_forward_plan(ctypes.byref(d), _ptr(alpha, "alpha", torch.float32),
                              _ptr(beta, "beta", torch.float32), _ptr(widx, "widx", torch.int32),
                              _ptr(ww, "ww", torch.float32), _ptr(ridx, "ridx", torch.int32),
                              _ptr(rw, "rw", torch.float32), ctypes.byref(st.c), _ptr(ws, "ws"),
                              ws.numel(), _stream(stream)), "sdm_forward_plan")


def forward_run(d: Dims, v, beta, widx, ww, ridx, rw, st: State, out, ws, stream=None):
    _ok(_lib.sdm_forward_run(ctypes.byref(d), _ptr(v, "v", _vdt(d)), _ptr(beta, "beta", torch.float32),
                             _ptr(widx, "widx", torch.int32), _ptr(ww, "ww", torch.float32),
                             _ptr(ridx, "ridx", torch.int32), _ptr(rw, "rw", torch.float32),
                             ctypes.byref(st.c), _ptr(out, "out", torch.float32), _ptr(ws, "ws"),
                             ws.numel(), _stream(stream)), "sdm_forward_run")
    return out


def selection_buffers(d: Dims, device="cuda"):
    """Caller buffers for the write / read selections of one call: widx, ww, ridx, rw."""
    return (torch.empty((d.B, d.H, d.T, d.W), dtype=torch.int32, device=device),
            torch.empty((d.B, d.H, d.T, d.W), dtype=torch.float32, device=device),
            torch.empty((d.B, d.H, d.T, d.R), dtype=torch.int32, device=device),
            torch.empty((d.B, d.H, d.T, d.R), dtype=torch.float32, device=device))


def prefill(d: Dims, q, k, v, alpha, beta, skw, skr, st: State, sel=None, out=None, ws=None,
            stream=None):
    """Scoring of k and q, then the recurrence.  Returns (out, (widx, ww, ridx, rw))."""
    dev = q.device
    if sel is None:
        sel = selection_buffers(d, dev)
    if out is None:
        out = torch.empty((d.B, d.H, d.T, d.d_v), dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(d, dev)
    widx, ww, ridx, rw = sel
    xdt = _xdt(d)
    _ok(_lib.sdm_prefill(ctypes.byref(d), _ptr(q, "q", xdt), _ptr(k, "k", xdt), _ptr(v, "v", _vdt(d)),
                         _ptr(alpha, "alpha", torch.float32), _ptr(beta, "beta", torch.float32),
                         _ptr(skw, "skw", xdt), _ptr(skr, "skr", xdt), ctypes.byref(st.c),
                         _ptr(widx, "widx", torch.int32), _ptr(ww, "ww", torch.float32),
                         _ptr(ridx, "ridx", torch.int32), _ptr(rw, "rw", torch.float32),
                         _ptr(out, "out", torch.float32), _ptr(ws, "ws"), ws.numel(),
                         _stream(stream)), "sdm_prefill")
    return out, sel


def backward_workspace_bytes(d: Dims) -> int:
    return int(_lib.sdm_backward_workspace_bytes(ctypes.byref(d)))


def backward(d: Dims, v, alpha, beta, widx, ww, ridx, rw, st: State, dout, ws=None, grads=None,
             stream=None, dM_end=None) -> dict:
    """sdm_backward: gradients of the recurrence over one call for the output gradient dout
    [B,H,T,d_v] fp32 and, optionally, the gradient dM_end [B,H,N,d_v] fp32 of the memory
    after the last token.  `st` must hold the state at the start of the call; it is replayed
    and restored in place.  Returns dict dv, dalpha, dbeta, dww, drw, dM_in (fp32)."""
    dev = v.device
    if dM_end is not None:
        # the kernels read B*H*N*d_v floats from it: a smaller tensor would be read past its end
        if tuple(dM_end.shape) != (d.B, d.H, d.N, d.d_v):
            raise ValueError(f"dM_end must have shape {(d.B, d.H, d.N, d.d_v)}, "
                             f"got {tuple(dM_end.shape)}")
        if dM_end.device != dev:
            raise ValueError(f"dM_end is on {dM_end.device}, the other inputs on {dev}")
    if ws is None:
        ws = torch.empty(max(16, backward_workspace_bytes(d)), dtype=torch.uint8, device=dev)
    if grads is None:
        f = dict(dtype=torch.float32, device=dev)
        grads = {"dv": torch.empty((d.B, d.H, d.T, d.d_v), **f),
                 "dalpha": torch.empty((d.B, d.H, d.T), **f),
                 "dbeta": torch.empty((d.B, d.H, d.T), **f),
                 "dww": torch.empty((d.B, d.H, d.T, d.W), **f),
                 "drw": torch.empty((d.B, d.H, d.T, d.R), **f),
                 "dM_in": torch.empty((d.B, d.H, d.N, d.d_v), **f)}
    a = _fw_args(d, v, alpha, beta, widx, ww, ridx, rw)
    g = grads
    _ok(_lib.sdm_backward(ctypes.byref(d), *a, ctypes.byref(st.c),
                          _ptr(dout, "dout", torch.float32),
                          None if dM_end is None else _ptr(dM_end, "dM_end", torch.float32),
                          _ptr(g["dv"], "dv", torch.float32),
                          _ptr(g["dalpha"], "dalpha", torch.float32),
                          _ptr(g["dbeta"], "dbeta", torch.float32),
                          _ptr(g["dww"], "dww", torch.float32), _ptr(g["drw"], "drw", torch.float32),
                          _ptr(g["dM_in"], "dM_in", torch.float32), _ptr(ws, "ws"), ws.numel(),
                          _stream(stream)), "sdm_backward")
    return grads


def score_backward(d: Dims, x, subkeys, top: int, idx, w, dw, dx=None, dsubkeys=None,
                   stream=None):
    """sdm_score_backward: (dx [B,H,T,d_k], dsubkeys [H,2,n,d_k/2]) fp32 for the selection
    weights' gradient dw, the selections idx / w held fixed.  dsubkeys is added to (a new
    zero tensor when not given)."""
    dev = x.device
    if dx is None:
        dx = torch.empty((d.B, d.H, d.T, d.d_k), dtype=torch.float32, device=dev)
    if dsubkeys is None:
        dsubkeys = torch.zeros((d.H, 2, d.n_sub, d.d_k // 2), dtype=torch.float32, device=dev)
    xdt = _xdt(d)
    _ok(_lib.sdm_score_backward(ctypes.byref(d), _ptr(x, "x", xdt), _ptr(subkeys, "subkeys", xdt),
                                top, _ptr(idx, "idx", torch.int32), _ptr(w, "w", torch.float32),
                                _ptr(dw, "dw", torch.float32), _ptr(dx, "dx", torch.float32),
                                _ptr(dsubkeys, "dsubkeys", torch.float32), _stream(stream)),
        "sdm_score_backward")
    return dx, dsubkeys


def decode_step(d: Dims, q, k, v, alpha, beta, skw, skr, st: State, sel=None, out=None,
                stream=None):
    """One token per sequence (d.T must be 1).  q, k: [B,H,d_k]; v: [B,H,d_v]; gates [B,H]."""
    dev = q.device
    if sel is None:
        sel = selection_buffers(d, dev)
    if out is None:
        out = torch.empty((d.B, d.H, d.d_v), dtype=torch.float32, device=dev)
    widx, ww, ridx, rw = sel
    xdt = _xdt(d)
    _ok(_lib.sdm_decode_step(ctypes.byref(d), _ptr(q, "q", xdt), _ptr(k, "k", xdt),
                             _ptr(v, "v", _vdt(d)), _ptr(alpha, "alpha", torch.float32),
                             _ptr(beta, "beta", torch.float32), _ptr(skw, "skw", xdt),
                             _ptr(skr, "skr", xdt), ctypes.byref(st.c),
                             _ptr(widx, "widx", torch.int32), _ptr(ww, "ww", torch.float32),
                             _ptr(ridx, "ridx", torch.int32), _ptr(rw, "rw", torch.float32),
                             _ptr(out, "out", torch.float32), _stream(stream)), "sdm_decode_step")
    return out, sel


def device_error(clear: bool = True, stream=None) -> int:
    """The device error word (DEVERR_* bits); synchronises the stream."""
    bits = ctypes.c_uint32(0)
    st = _lib.sdm_device_error(ctypes.byref(bits), 1 if clear else 0, _stream(stream))
    if st not in (0, 6):
        raise SdmError(st, "sdm_device_error")
    return int(bits.value)


def weight_stats(w: torch.Tensor, probs=(0.1, 0.5, 0.9), cum: bool = True, stream=None) -> dict:
    """Memory-utilisation diagnostics (sdm_weight_stats) of weight rows w [..., K] fp32 given
    best first: per-row cumulative mass (if cum) and exp(entropy)/K, their means, and the
    order statistics of exp(entropy)/K at floor(p * (rows - 1))."""
    K = int(w.shape[-1])
    rows = int(w.numel() // K) if K else 0
    dev = w.device
    eff = torch.empty(w.shape[:-1], dtype=torch.float32, device=dev)
    cum_t = torch.empty(w.shape, dtype=torch.float32, device=dev) if cum else None
    mean = torch.empty(K + 1, dtype=torch.float32, device=dev)
    pr = (ctypes.c_double * max(1, len(probs)))(*probs)
    quant = torch.empty(max(1, len(probs)), dtype=torch.float32, device=dev)
    nbytes = _lib.sdm_weight_stats_workspace_bytes(rows, K)
    ws = torch.empty(max(1, nbytes), dtype=torch.uint8, device=dev)
    _ok(_lib.sdm_weight_stats(rows, K, _ptr(w, "w", torch.float32), _ptr(cum_t, "cum"),
                              _ptr(eff, "eff"), _ptr(mean, "mean"), len(probs), pr,
                              _ptr(quant, "quant"), _ptr(ws, "ws"), nbytes, _stream(stream)),
        "sdm_weight_stats")
    return {"cum": cum_t, "eff": eff, "mean_cum": mean[:K], "mean_eff": mean[K],
            "quant": quant[:len(probs)]}


def gemm_bf16(A: torch.Tensor, Bt: torch.Tensor, C: torch.Tensor | None = None, stream=None):
    """C = A @ Bt.T on the tensor cores: A [M, K] bf16, Bt [N, K] bf16 -> C [M, N] fp32."""
    M, K = A.shape
    N = Bt.shape[0]
    if Bt.shape[1] != K:
        raise ValueError("A and Bt must share K")
    if C is None:
        C = torch.empty((M, N), dtype=torch.float32, device=A.device)
    _ok(_lib.sdm_gemm_bf16(M, N, K, _ptr(A, "A", torch.bfloat16), _ptr(Bt, "Bt", torch.bfloat16),
                           _ptr(C, "C", torch.float32), _stream(stream)), "sdm_gemm_bf16")
    return C


def layer_out(d: Dims, o: torch.Tensor, g: torch.Tensor, wn: torch.Tensor, Wo_t: torch.Tensor,
              eps: float = 1e-6, y: torch.Tensor | None = None, ws: torch.Tensor | None = None,
              stream=None):
    """SDM layer output: RMS-norm of each head's read, swish gate, output projection.
    o [B,H,T,d_v] fp32, g [B,T,H*d_v] bf16, wn [d_v] fp32, Wo_t [d_model, H*d_v] bf16
    -> y [B,T,d_model] fp32."""
    d_model = int(Wo_t.shape[0])
    if y is None:
        y = torch.empty((d.B, d.T, d_model), dtype=torch.float32, device=o.device)
    nbytes = _lib.sdm_layer_out_workspace_bytes(ctypes.byref(d))
    if ws is None:
        ws = torch.empty(max(16, nbytes), dtype=torch.uint8, device=o.device)
    _ok(_lib.sdm_layer_out(ctypes.byref(d), _ptr(o, "o", torch.float32), _ptr(g, "g", torch.bfloat16),
                           _ptr(wn, "wn", torch.float32), float(eps),
                           _ptr(Wo_t, "Wo_t", torch.bfloat16), d_model,
                           _ptr(y, "y", torch.float32), _ptr(ws, "ws"), ws.numel(),
                           _stream(stream)), "sdm_layer_out")
    return y


def forward_run_gated(d: Dims, v, beta, widx, ww, ridx, rw, st: State, g, wn, eps: float = 1e-6,
                      out=None, a=None, ws=None, stream=None):
    """sdm_forward_run_gated: the row pass (after forward_plan on the same ws) with the layer
    output side's RMS-norm and swish gate fused into the read.  g [B,T,H*d_v] bf16, wn [d_v]
    fp32.  Returns (out [B,H,T,d_v] fp32, a [B,T,H*d_v] bf16); y = gemm_bf16(a, Wo_t)."""
    dev = v.device
    if out is None:
        out = torch.empty((d.B, d.H, d.T, d.d_v), dtype=torch.float32, device=dev)
    if a is None:
        a = torch.empty((d.B, d.T, d.H * d.d_v), dtype=torch.bfloat16, device=dev)
    if ws is None:
        raise ValueError("forward_run_gated needs the workspace forward_plan filled")
    _ok(_lib.sdm_forward_run_gated(ctypes.byref(d), _ptr(v, "v", _vdt(d)),
                                   _ptr(beta, "beta", torch.float32),
                                   _ptr(widx, "widx", torch.int32), _ptr(ww, "ww", torch.float32),
                                   _ptr(ridx, "ridx", torch.int32), _ptr(rw, "rw", torch.float32),
                                   ctypes.byref(st.c),
                                   _ptr(out, "out", torch.float32), _ptr(g, "g", torch.bfloat16),
                                   _ptr(wn, "wn", torch.float32), float(eps),
                                   _ptr(a, "a", torch.bfloat16), _ptr(ws, "ws"), ws.numel(),
                                   _stream(stream)), "sdm_forward_run_gated")
    return out, a


def layer_in(d: Dims, x: torch.Tensor, Win_t: torch.Tensor, A_log: torch.Tensor,
             dt_bias: torch.Tensor, out: dict | None = None, ws: torch.Tensor | None = None,
             stream=None) -> dict:
    """SDM layer input side: x [B,T,d_model] bf16, Win_t [H*(2dk+2dv+2), d_model] bf16,
    A_log / dt_bias [H] fp32 -> q, k [B,H,T,d_k] bf16, v [B,H,T,d_v], g [B,T,H*d_v] bf16,
    alpha, beta [B,H,T] fp32 (the inputs of prefill and layer_out)."""
    dev = x.device
    d_model = int(x.shape[-1])
    vdt = torch.bfloat16 if d.v_dtype == BF16 else torch.float32
    if out is None:
        out = {"q": torch.empty((d.B, d.H, d.T, d.d_k), dtype=torch.bfloat16, device=dev),
               "k": torch.empty((d.B, d.H, d.T, d.d_k), dtype=torch.bfloat16, device=dev),
               "v": torch.empty((d.B, d.H, d.T, d.d_v), dtype=vdt, device=dev),
               "g": torch.empty((d.B, d.T, d.H * d.d_v), dtype=torch.bfloat16, device=dev),
               "alpha": torch.empty((d.B, d.H, d.T), dtype=torch.float32, device=dev),
               "beta": torch.empty((d.B, d.H, d.T), dtype=torch.float32, device=dev)}
    nbytes = _lib.sdm_layer_in_workspace_bytes(ctypes.byref(d))
    if ws is None:
        ws = torch.empty(max(16, nbytes), dtype=torch.uint8, device=dev)
    _ok(_lib.sdm_layer_in(ctypes.byref(d), _ptr(x, "x", torch.bfloat16),
                          _ptr(Win_t, "Win_t", torch.bfloat16), _ptr(A_log, "A_log", torch.float32),
                          _ptr(dt_bias, "dt_bias", torch.float32), d_model,
                          _ptr(out["q"], "q", torch.bfloat16), _ptr(out["k"], "k", torch.bfloat16),
                          _ptr(out["v"], "v", vdt), _ptr(out["g"], "g", torch.bfloat16),
                          _ptr(out["alpha"], "alpha", torch.float32),
                          _ptr(out["beta"], "beta", torch.float32), _ptr(ws, "ws"), ws.numel(),
                          _stream(stream)), "sdm_layer_in")
    return out
