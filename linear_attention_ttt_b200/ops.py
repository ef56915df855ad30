"""Python binding of libttt_b200.so (argument marshalling only).

Every function here builds ``ttt_tensor`` descriptors from torch tensors
(pointer, element type, shape, strides), passes the current CUDA stream, and
calls the C ABI of ``include/ttt.h``. All computation happens in the CUDA
library; if it is missing, loading fails with an error (there is no fallback).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# TTT_B200_LIB selects another build of the library, e.g. the debug-bounds one
# (libttt_b200_dbg.so, from `python -m linear_attention_ttt_b200.build --debug-bounds`).
LIB_PATH = os.environ.get("TTT_B200_LIB") or os.path.join(_PKG, "libttt_b200.so")
DEBUG_LIB_PATH = os.path.join(_PKG, "libttt_b200_dbg.so")

TTT_F32, TTT_BF16 = 0, 1
TTT_LOSS_MSE, TTT_LOSS_NEG_DOT = 0, 1
LACT_UPDATE_GD, LACT_UPDATE_MUON = 0, 1

STATUS = {
    0: "TTT_OK", -1: "TTT_ERR_NULL", -2: "TTT_ERR_SHAPE", -3: "TTT_ERR_DTYPE",
    -4: "TTT_ERR_LAYOUT", -5: "TTT_ERR_UNSUPPORTED", -6: "TTT_ERR_CUDA",
    -7: "TTT_ERR_TIMEOUT", -8: "TTT_ERR_ALLOC", -9: "TTT_ERR_ARG", -10: "TTT_ERR_SCRATCH",
    -11: "TTT_ERR_BOUNDS",
}
ERR_CODES = {name: code for code, name in STATUS.items()}


class TTTError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({_lib_or_none_msg(code)})")


def _lib_or_none_msg(code):
    try:
        return load().ttt_status_string(code).decode()
    except Exception:  # pragma: no cover
        return "?"


class TTTTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


_LIB = None
P = ctypes.POINTER(TTTTensor)
# lact_grad_reduce_fn of include/ttt.h
REDUCE_FN = ctypes.CFUNCTYPE(ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                             ctypes.c_void_p)

SIGNATURES = {
    "ttt_linear_fwd": ([P, P, P, P, P, ctypes.c_int32, ctypes.c_int32, P, P, ctypes.c_void_p],
                       ctypes.c_int32),
    "lact_swiglu_fwd": ([P, P, P, P, P, P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P,
                         ctypes.c_void_p], ctypes.c_int32),
    "lact_swiglu_fwd_ex": ([P, P, P, P, P, P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                            P, P, P, P, ctypes.c_void_p], ctypes.c_int32),
    "lact_swiglu_fwd_noalloc": ([P, P, P, P, P, P, P, ctypes.c_int32, ctypes.c_int32,
                                 ctypes.c_int32, P, P, P, P, ctypes.c_void_p], ctypes.c_int32),
    "lact_swiglu_fwd_momentum": ([P, P, P, P, P, P, P, ctypes.c_int32, ctypes.c_float,
                                  ctypes.c_int32, P, P, P, P, P, P, P, P, P, P,
                                  ctypes.c_void_p], ctypes.c_int32),
    "ttt_linear_bwd": ([P, P, P, P, P, ctypes.c_int32, ctypes.c_int32, P, P, P, P, P, P, P,
                        ctypes.c_void_p], ctypes.c_int32),
    "ttt_mlp_fwd": ([P, P, P, P, P, P, P, P, ctypes.c_int32, P, P, P, P, P, ctypes.c_void_p],
                    ctypes.c_int32),
    "window_attention_fwd": ([P, P, P, ctypes.c_int32, ctypes.c_int32, P, ctypes.c_void_p],
                             ctypes.c_int32),
    "lact_swiglu_window_fwd": ([P, P, P, P, P, P, P, ctypes.c_int32, ctypes.c_int32,
                               ctypes.c_int32, P, ctypes.c_void_p], ctypes.c_int32),
    "lact_swiglu_fwd_cp": ([P, P, P, P, P, P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                            P, P, P, P, REDUCE_FN, ctypes.c_void_p, ctypes.c_void_p],
                           ctypes.c_int32),
    "lact_swiglu_bwd": ([P, P, P, P, P, P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                         P, P, P, P, P, P, P, P, P, P, P, ctypes.c_void_p], ctypes.c_int32),
    "ttt_status_string": ([ctypes.c_int32], ctypes.c_char_p),
    "ttt_get_device_status": ([ctypes.c_void_p], ctypes.c_int32),
    "ttt_version": ([], ctypes.c_int32),
    "ttt_test_fail_allocations": ([ctypes.c_int32], None),
    "ttt_selftest_wait_timeout": ([ctypes.c_void_p], ctypes.c_int32),
    "ttt_selftest_bounds": ([ctypes.c_void_p], ctypes.c_int32),
}


def load(path: str = LIB_PATH):
    """Load the CUDA library (raises OSError if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(path):
            raise OSError(f"{path} is missing: run `python -m linear_attention_ttt_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _LIB = lib
    return _LIB


def describe(t: Optional[torch.Tensor]):
    """ttt_tensor descriptor of a torch tensor (None -> NULL pointer)."""
    if t is None:
        return None
    if t.dtype == torch.float32:
        dt = TTT_F32
    elif t.dtype == torch.bfloat16:
        dt = TTT_BF16
    else:
        raise TypeError(f"unsupported dtype {t.dtype}")
    if t.dim() > 4:
        raise ValueError("at most 4 dims")
    d = TTTTensor()
    d.data = t.data_ptr() if t.numel() > 0 else 0
    d.dtype = dt
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _ref(d):
    return ctypes.byref(d) if d is not None else None


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(code, what):
    if code != 0:
        raise TTTError(code, what)


def ttt_linear_fwd(q, k, v, eta, W0, chunk: int, loss: int, out=None, W_final=None,
                   stream=None, want_final: bool = True):
    """TTT-Linear (loss=TTT_LOSS_MSE) or inner-product / linear attention
    (loss=TTT_LOSS_NEG_DOT) forward. Returns (out, W_final or None)."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    if W_final is None and want_final:
        W_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    ds = [describe(x) for x in (q, k, v, eta, W0, out, W_final)]
    code = load().ttt_linear_fwd(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]), _ref(ds[3]), _ref(ds[4]),
                                 int(chunk), int(loss), _ref(ds[5]), _ref(ds[6]), _stream(stream))
    _check(code, "ttt_linear_fwd")
    return out, W_final


def ttt_linear_bwd(q, k, v, eta, W0, chunk: int, loss: int, dy, dW_final=None, stream=None):
    """Backward of ttt_linear_fwd: given dL/dy (and optionally dL/dW_final),
    returns (dq, dk, dv, deta, dW0); dW0 has W0's shape (summed over the
    batch when W0 is shared by it)."""
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    deta = torch.empty(eta.shape, dtype=torch.float32, device=q.device)
    dW0 = torch.empty(W0.shape, dtype=torch.float32, device=q.device)
    ds = [describe(x) for x in (q, k, v, eta, W0, dy, dW_final, dq, dk, dv, deta, dW0)]
    r = [_ref(d) for d in ds]
    code = load().ttt_linear_bwd(*r[:5], int(chunk), int(loss), *r[5:], _stream(stream))
    _check(code, "ttt_linear_bwd")
    return dq, dk, dv, deta, dW0


def ttt_mlp_fwd(q, k, v, eta, W1, b1, W2, b2, chunk: int, out=None, finals=False, stream=None):
    """TTT-MLP forward (two-layer ReLU MLP fast weight, mini-batch rule). With
    finals=True also returns the final (W1, b1, W2, b2) as [B,H,...] tensors."""
    B, H, T, dk = q.shape
    dv, dh = v.shape[-1], W1.shape[-2]
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    F = [None] * 4
    if finals:
        F = [torch.empty(s, dtype=torch.float32, device=q.device)
             for s in ((B, H, dh, dk), (B, H, dh), (B, H, dv, dh), (B, H, dv))]
    ds = [describe(x) for x in (q, k, v, eta, W1, b1, W2, b2, out, *F)]
    r = [_ref(d) for d in ds]
    code = load().ttt_mlp_fwd(*r[:8], int(chunk), *r[8:], _stream(stream))
    _check(code, "ttt_mlp_fwd")
    return (out, *F) if finals else out


def lact_swiglu_fwd(q, k, v, eta, W1, W2, W3, chunk: int, update_rule: int = LACT_UPDATE_GD,
                    causal: int = 1, out=None, finals=False, stream=None):
    """LaCT SwiGLU fast-weight layer forward. With finals=True also returns
    the final (W1, W2, W3) as [B,H,...] fp32 tensors."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dh = W1.shape[-2]
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    F = [None, None, None]
    if finals:
        F = [torch.empty((B, H, dh, dk), dtype=torch.float32, device=q.device),
             torch.empty((B, H, dv, dh), dtype=torch.float32, device=q.device),
             torch.empty((B, H, dh, dk), dtype=torch.float32, device=q.device)]
    ds = [describe(x) for x in (q, k, v, eta, W1, W2, W3, out, *F)]
    r = [_ref(d) for d in ds]
    code = load().lact_swiglu_fwd_ex(*r[:7], int(chunk), int(update_rule), int(causal), r[7],
                                     r[8], r[9], r[10], _stream(stream))
    _check(code, "lact_swiglu_fwd")
    return (out, *F) if finals else out


def lact_swiglu_bwd(q, k, v, eta, W1, W2, W3, chunk: int, update_rule: int, causal: int, dy,
                    dW_final=(None, None, None), stream=None):
    """Backward of lact_swiglu_fwd: returns (dq, dk, dv, deta, dW1, dW2, dW3),
    the weight gradients in the shapes of W1, W2, W3."""
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    deta = torch.empty(eta.shape, dtype=torch.float32, device=q.device)
    dW = [torch.empty(W.shape, dtype=torch.float32, device=q.device) for W in (W1, W2, W3)]
    ds = [describe(x) for x in (q, k, v, eta, W1, W2, W3, dy, *dW_final, dq, dk, dv, deta, *dW)]
    r = [_ref(d) for d in ds]
    code = load().lact_swiglu_bwd(*r[:7], int(chunk), int(update_rule), int(causal), *r[7:],
                                  _stream(stream))
    _check(code, "lact_swiglu_bwd")
    return (dq, dk, dv, deta, *dW)


def lact_swiglu_fwd_noalloc(q, k, v, eta, W1, W2, W3, chunk: int,
                            update_rule: int = LACT_UPDATE_GD, causal: int = 1, out=None,
                            finals=False, stream=None):
    """lact_swiglu_fwd on the library's fixed device scratch pool: the C call
    allocates no device memory (for callers that cannot allocate; see
    include/ttt.h). Output tensors passed in are written in place; tensors
    created here (when `out` or the finals are omitted) are the caller's
    convenience, made before the call."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dh = W1.shape[-2]
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    F = [None, None, None]
    if finals:
        F = [torch.empty((B, H, dh, dk), dtype=torch.float32, device=q.device),
             torch.empty((B, H, dv, dh), dtype=torch.float32, device=q.device),
             torch.empty((B, H, dh, dk), dtype=torch.float32, device=q.device)]
    ds = [describe(x) for x in (q, k, v, eta, W1, W2, W3, out, *F)]
    r = [_ref(d) for d in ds]
    code = load().lact_swiglu_fwd_noalloc(*r[:7], int(chunk), int(update_rule), int(causal), r[7],
                                          r[8], r[9], r[10], _stream(stream))
    _check(code, "lact_swiglu_fwd_noalloc")
    return (out, *F) if finals else out


def lact_swiglu_fwd_momentum(q, k, v, eta, W1, W2, W3, chunk: int, beta: float,
                             causal: int = 1, M0=(None, None, None), out=None, finals=False,
                             stream=None):
    """LaCT forward with heavy-ball momentum on the chunk gradients
    (M <- beta M + G, W <- W - M, then the row renorm). M0 = (M1, M2, M3)
    initial momentum (None: zero). With finals=True also returns the final
    (W1, W2, W3) and (M1, M2, M3) as [B,H,...] fp32 tensors."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dh = W1.shape[-2]
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    F = [None] * 6
    if finals:
        shapes = [(B, H, dh, dk), (B, H, dv, dh), (B, H, dh, dk)] * 2
        F = [torch.empty(s, dtype=torch.float32, device=q.device) for s in shapes]
    ds = [describe(x) for x in (q, k, v, eta, W1, W2, W3, *M0, out, *F)]
    r = [_ref(d) for d in ds]
    code = load().lact_swiglu_fwd_momentum(*r[:7], int(chunk), float(beta), int(causal),
                                           r[7], r[8], r[9], r[10], *r[11:17], _stream(stream))
    _check(code, "lact_swiglu_fwd_momentum")
    return (out, tuple(F[:3]), tuple(F[3:])) if finals else out


def window_attention_fwd(q, k, v, window: int, out=None, accumulate: bool = False, stream=None):
    """Sliding-window causal softmax attention (scale 1/sqrt(d)); with
    accumulate=True the result is added into `out`."""
    if out is None:
        out = torch.zeros_like(v) if accumulate else torch.empty_like(v)
    ds = [describe(x) for x in (q, k, v, out)]
    r = [_ref(d) for d in ds]
    code = load().window_attention_fwd(r[0], r[1], r[2], int(window), int(bool(accumulate)), r[3],
                                       _stream(stream))
    _check(code, "window_attention_fwd")
    return out


def lact_swiglu_window_fwd(q, k, v, eta, W1, W2, W3, chunk: int, update_rule: int, window: int,
                           out=None, stream=None):
    """LaCT layer (causal) plus window attention on the same q, k, v, summed."""
    if out is None:
        out = torch.empty_like(v)
    ds = [describe(x) for x in (q, k, v, eta, W1, W2, W3, out)]
    r = [_ref(d) for d in ds]
    code = load().lact_swiglu_window_fwd(*r[:7], int(chunk), int(update_rule), int(window), r[7],
                                         _stream(stream))
    _check(code, "lact_swiglu_window_fwd")
    return out


def selftest_wait_timeout(stream=None) -> None:
    """Enqueue the failure-detection self-test (a bounded wait that runs out);
    device_status() afterwards returns TTT_ERR_TIMEOUT."""
    _check(load().ttt_selftest_wait_timeout(_stream(stream)), "ttt_selftest_wait_timeout")


def device_status(stream=None) -> int:
    """Synchronise and return (then clear) the device-side status code."""
    return int(load().ttt_get_device_status(_stream(stream)))
