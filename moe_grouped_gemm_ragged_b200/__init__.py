"""Ragged MoE grouped GEMM for B200 (sm_100a): a thin Python binding over ``libgg.so``.

Every function here only checks and marshals arguments (device pointers, sizes, the current
CUDA stream) into the C ABI declared in ``include/gg.h``; all arithmetic runs in the
library's sm_100a kernels. There is no fallback: if the library is missing or cannot load,
the import of the kernels fails with an error.

Groups are cumulative END offsets (int32, on the device, no leading zero): group e covers
rows [offs[e-1], offs[e]) with offs[-1] = 0, as in ``torch._grouped_mm(x, w, offs)``
(PyTorch issue 152668, "Easy repro scenario").
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# GG_LIBRARY may name another build of the same library (e.g. with other tuning macros)
LIB_PATH = os.environ.get("GG_LIBRARY") or os.path.join(_PKG, "libgg.so")

GG_OK, GG_ERR_INVALID_ARG, GG_ERR_UNSUPPORTED, GG_ERR_CUDA = 0, 1, 2, 3
DEV_BAD_OFFSETS = 0x1
DEV_BAD_MASKED_M = 0x2
DEV_TIMEOUT = 0x4
DEV_BAD_ROUTE = 0x8
DEV_ERROR_MASK = 0xFF
DEV_LAUNCHED = 0x100
MAX_EXPERTS = 1024

_lib = None

ACT_NONE, ACT_SILU_MUL = 0, 1
FLAG_ZERO_TAIL, FLAG_W_NK, FLAG_GATE_UP_CONCAT = 0x1, 0x2, 0x4


class _Epilogue(ctypes.Structure):
    _fields_ = [("bias", ctypes.c_void_p), ("bias_scale", ctypes.c_void_p),
                ("act", ctypes.c_int32), ("flags", ctypes.c_int32)]


class GGError(RuntimeError):
    """A non-OK status returned by the C ABI."""

    def __init__(self, code: int, where: str):
        self.code = code
        detail = ""
        if code == GG_ERR_CUDA:
            detail = " (" + lib().gg_last_error().decode() + ")"
        super().__init__(f"{where}: {status_string(code)}{detail}")


def lib() -> ctypes.CDLL:
    """The loaded C library (``libgg.so``). Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m moe_grouped_gemm_ragged_b200._build`"
            " (there is no non-CUDA implementation)")
    L = ctypes.CDLL(LIB_PATH)
    P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    sig = [P, P, P, P, i64, i64, i64, i32, P, P]
    for name in ("gg_forward", "gg_dgrad", "gg_wgrad", "gg_masked_forward"):
        fn = getattr(L, name)
        fn.argtypes = sig
        fn.restype = ctypes.c_int
    L.gg_wgrad_f32.argtypes = [P, P, P, P, ctypes.c_float, ctypes.c_float, i64, i64, i64, i32,
                               P, P]
    L.gg_wgrad_f32.restype = ctypes.c_int
    for name in ("gg_dgrad_ex", "gg_wgrad_ex"):
        fn = getattr(L, name)
        fn.argtypes = [P, P, P, P, i64, i64, i64, i32, i32, P, P]
        fn.restype = ctypes.c_int
    L.gg_forward_ex.argtypes = [P, P, P, P, i64, i64, i64, i32, ctypes.POINTER(_Epilogue), P, P]
    L.gg_forward_ex.restype = ctypes.c_int
    L.gg_masked_forward_ex.argtypes = [P, P, P, P, i64, i64, i64, i32,
                                       ctypes.POINTER(_Epilogue), P, P]
    L.gg_masked_forward_ex.restype = ctypes.c_int
    L.gg_route_workspace_bytes.argtypes = [i64, i32]
    L.gg_route_workspace_bytes.restype = ctypes.c_size_t
    L.gg_route.argtypes = [P, i64, i32, i32, P, i64, P, P, P, P, ctypes.c_size_t, P, P]
    L.gg_route.restype = ctypes.c_int
    L.gg_layer_step_host.argtypes = [P] * 14 + [i64, i64, i64, i32, i32, P, P]
    L.gg_layer_step_host.restype = ctypes.c_int
    L.gg_status_string.argtypes = [ctypes.c_int]
    L.gg_status_string.restype = ctypes.c_char_p
    L.gg_set_watchdog_ns.argtypes = [ctypes.c_uint64]
    L.gg_set_watchdog_ns.restype = ctypes.c_uint64
    L.gg_testing_skip_first_load.argtypes = [ctypes.c_int]
    L.gg_testing_skip_first_load.restype = ctypes.c_int
    L.gg_testing_force_variant.argtypes = [ctypes.c_int]
    L.gg_testing_force_variant.restype = ctypes.c_int
    L.gg_version.restype = ctypes.c_int
    L.gg_last_error.restype = ctypes.c_char_p
    _lib = L
    return L


def status_string(code: int) -> str:
    return lib().gg_status_string(int(code)).decode()


def version() -> int:
    return lib().gg_version()


def set_watchdog_ns(ns: int) -> int:
    """Bound of every in-kernel wait (ns) for later calls; returns the previous value."""
    return int(lib().gg_set_watchdog_ns(int(ns)))


def testing_skip_first_load(enable: bool) -> bool:
    """Test hook: make later calls' first load go missing so the watchdog fires."""
    return bool(lib().gg_testing_skip_first_load(1 if enable else 0))


def testing_force_variant(variant: int) -> int:
    """Test hook: 0 automatic, 1 single-CTA tiles, 2 CTA-pair tiles, 3 wide CTA pairs
    (256 x 512 tiles, the automatic forward/dgrad shape of CTA pairs, and of the SiLU-and-mul
    forward when K >= 4096), each for every pass."""
    return int(lib().gg_testing_force_variant(int(variant)))


def _stream_handle(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(t: torch.Tensor, name: str, dtype, ndim: int):
    # fast path: one combined test; the message below names the first failing property
    if (isinstance(t, torch.Tensor) and t.dtype is dtype and t.dim() == ndim and t.is_cuda
            and t.is_contiguous() and t.get_device() == torch.cuda.current_device()):
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        # the library launches on the current device; another device's pointers would be
        # dereferenced there
        raise ValueError(f"{name} is on {t.device}, the current device is "
                         f"cuda:{torch.cuda.current_device()} (use torch.cuda.device(...))")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _status_ptr(status: Optional[torch.Tensor]):
    if status is None:
        return None
    _check(status, "status", torch.int32, 1)
    return status.data_ptr()


def _raise(rc: int, where: str):
    if rc != GG_OK:
        raise GGError(rc, where)


def forward(A: torch.Tensor, W: torch.Tensor, offs: torch.Tensor, out: torch.Tensor, *,
            status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out[r,:] = A[r,:] @ W[e] for every row r of group e; other rows of ``out`` untouched.

    A bf16 [rows, K], W bf16 [E, K, N], offs int32 [E] (device), out bf16 [rows, N]."""
    _check(A, "A", torch.bfloat16, 2)
    _check(W, "W", torch.bfloat16, 3)
    _check(offs, "offs", torch.int32, 1)
    _check(out, "out", torch.bfloat16, 2)
    rows, K = A.shape
    E, K2, N = W.shape
    if K2 != K or offs.numel() != E or tuple(out.shape) != (rows, N):
        raise ValueError("shape mismatch: A[rows,K], W[E,K,N], offs[E], out[rows,N]")
    rc = lib().gg_forward(_ptr(A), _ptr(W), _ptr(offs), _ptr(out), rows, K, N, E,
                          _status_ptr(status), _stream_handle(stream))
    _raise(rc, "gg_forward")
    return out


def _flags(zero_tail: bool, w_nk: bool) -> int:
    return (FLAG_ZERO_TAIL if zero_tail else 0) | (FLAG_W_NK if w_nk else 0)


def _epilogue(bias, bias_scale, act, E, N, flags=0):
    if bias is not None:
        _check(bias, "bias", torch.bfloat16, 2)
        if tuple(bias.shape) != (E, N):
            raise ValueError("bias must be [E, N]")
    if bias_scale is not None:
        _check(bias_scale, "bias_scale", torch.float32, 1)
    if act not in (ACT_NONE, ACT_SILU_MUL):
        raise ValueError("act must be ACT_NONE or ACT_SILU_MUL")
    return _Epilogue(_ptr(bias), _ptr(bias_scale), act, flags)


def forward_ex(A: torch.Tensor, W: torch.Tensor, offs: torch.Tensor, out: torch.Tensor, *,
               bias: Optional[torch.Tensor] = None, bias_scale: Optional[torch.Tensor] = None,
               act: int = ACT_NONE, zero_tail: bool = False, w_nk: bool = False,
               gate_up_concat: bool = False, status: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """Forward with a fused epilogue: h = A @ W[e] + bias_scale[r] * bias[e]; with
    act=ACT_SILU_MUL out = silu(gate) * up over gate/up column blocks of 128 (N % 256 == 0),
    or, with gate_up_concat, over the two halves [gate | up] of W's columns; out has N/2
    columns. bias_scale is read only for rows inside a group. zero_tail writes zeros to the
    rows past the last offset; w_nk takes W as [E, N, K]."""
    _check(A, "A", torch.bfloat16, 2)
    _check(W, "W", torch.bfloat16, 3)
    _check(offs, "offs", torch.int32, 1)
    _check(out, "out", torch.bfloat16, 2)
    rows, K = A.shape
    if w_nk:
        E, N, K2 = W.shape
    else:
        E, K2, N = W.shape
    ncols = N // 2 if act == ACT_SILU_MUL else N
    if K2 != K or offs.numel() != E or tuple(out.shape) != (rows, ncols):
        raise ValueError("shape mismatch: A[rows,K], W[E,K,N], offs[E], out[rows,N or N/2]")
    flags = _flags(zero_tail, w_nk) | (FLAG_GATE_UP_CONCAT if gate_up_concat else 0)
    epi = _epilogue(bias, bias_scale, act, E, N, flags)
    rc = lib().gg_forward_ex(_ptr(A), _ptr(W), _ptr(offs), _ptr(out), rows, K, N, E,
                             ctypes.byref(epi), _status_ptr(status), _stream_handle(stream))
    _raise(rc, "gg_forward_ex")
    return out


def dgrad_ex(dY: torch.Tensor, W: torch.Tensor, offs: torch.Tensor, dX: torch.Tensor, *,
             zero_tail: bool = False, w_nk: bool = False, status: Optional[torch.Tensor] = None,
             stream=None) -> torch.Tensor:
    """dgrad with flags: zero_tail writes zeros to the rows past the last offset; w_nk takes
    W as [E, N, K]."""
    _check(dY, "dY", torch.bfloat16, 2)
    _check(W, "W", torch.bfloat16, 3)
    _check(offs, "offs", torch.int32, 1)
    _check(dX, "dX", torch.bfloat16, 2)
    rows, N = dY.shape
    if w_nk:
        E, N2, K = W.shape
    else:
        E, K, N2 = W.shape
    if N2 != N or offs.numel() != E or tuple(dX.shape) != (rows, K):
        raise ValueError("shape mismatch: dY[rows,N], W, offs[E], dX[rows,K]")
    rc = lib().gg_dgrad_ex(_ptr(dY), _ptr(W), _ptr(offs), _ptr(dX), rows, K, N, E,
                           _flags(zero_tail, w_nk), _status_ptr(status), _stream_handle(stream))
    _raise(rc, "gg_dgrad_ex")
    return dX


def wgrad_ex(A: torch.Tensor, dY: torch.Tensor, offs: torch.Tensor, dW: torch.Tensor, *,
             w_nk: bool = False, status: Optional[torch.Tensor] = None,
             stream=None) -> torch.Tensor:
    """wgrad with flags: w_nk writes dW as [E, N, K] (dW[e] = dY_e^T @ A_e)."""
    _check(A, "A", torch.bfloat16, 2)
    _check(dY, "dY", torch.bfloat16, 2)
    _check(offs, "offs", torch.int32, 1)
    _check(dW, "dW", torch.bfloat16, 3)
    rows, K = A.shape
    rows2, N = dY.shape
    E = offs.numel()
    want = (E, N, K) if w_nk else (E, K, N)
    if rows2 != rows or tuple(dW.shape) != want:
        raise ValueError(f"shape mismatch: dW must be {want}")
    rc = lib().gg_wgrad_ex(_ptr(A), _ptr(dY), _ptr(offs), _ptr(dW), rows, K, N, E,
                           _flags(False, w_nk), _status_ptr(status), _stream_handle(stream))
    _raise(rc, "gg_wgrad_ex")
    return dW


def masked_forward_ex(A: torch.Tensor, W: torch.Tensor, masked_m: torch.Tensor,
                      out: torch.Tensor, *, bias: Optional[torch.Tensor] = None,
                      bias_scale: Optional[torch.Tensor] = None, act: int = ACT_NONE,
                      gate_up_concat: bool = False, status: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """Masked forward with the fused epilogue of forward_ex; bias_scale is indexed by the
    flat row e*mmax + r; out is [E, mmax, N] or [E, mmax, N/2]."""
    _check(A, "A", torch.bfloat16, 3)
    _check(W, "W", torch.bfloat16, 3)
    _check(masked_m, "masked_m", torch.int32, 1)
    _check(out, "out", torch.bfloat16, 3)
    E, mmax, K = A.shape
    E2, K2, N = W.shape
    ncols = N // 2 if act == ACT_SILU_MUL else N
    if E2 != E or K2 != K or masked_m.numel() != E or tuple(out.shape) != (E, mmax, ncols):
        raise ValueError("shape mismatch: A[E,mmax,K], W[E,K,N], masked_m[E], out")
    epi = _epilogue(bias, bias_scale, act, E, N,
                    FLAG_GATE_UP_CONCAT if gate_up_concat else 0)
    rc = lib().gg_masked_forward_ex(_ptr(A), _ptr(W), _ptr(masked_m), _ptr(out), mmax, K, N, E,
                                    ctypes.byref(epi), _status_ptr(status),
                                    _stream_handle(stream))
    _raise(rc, "gg_masked_forward_ex")
    return out


def dgrad(dY: torch.Tensor, W: torch.Tensor, offs: torch.Tensor, dX: torch.Tensor, *,
          status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """dX[r,:] = dY[r,:] @ W[e]^T for every row r of group e; other rows untouched.

    dY bf16 [rows, N], W bf16 [E, K, N], offs int32 [E], dX bf16 [rows, K]."""
    _check(dY, "dY", torch.bfloat16, 2)
    _check(W, "W", torch.bfloat16, 3)
    _check(offs, "offs", torch.int32, 1)
    _check(dX, "dX", torch.bfloat16, 2)
    rows, N = dY.shape
    E, K, N2 = W.shape
    if N2 != N or offs.numel() != E or tuple(dX.shape) != (rows, K):
        raise ValueError("shape mismatch: dY[rows,N], W[E,K,N], offs[E], dX[rows,K]")
    rc = lib().gg_dgrad(_ptr(dY), _ptr(W), _ptr(offs), _ptr(dX), rows, K, N, E,
                        _status_ptr(status), _stream_handle(stream))
    _raise(rc, "gg_dgrad")
    return dX


def wgrad(A: torch.Tensor, dY: torch.Tensor, offs: torch.Tensor, dW: torch.Tensor, *,
          status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """dW[e] = A[rows of e]^T @ dY[rows of e], all of dW overwritten (zeros if e is empty).

    A bf16 [rows, K], dY bf16 [rows, N], offs int32 [E], dW bf16 [E, K, N]."""
    _check(A, "A", torch.bfloat16, 2)
    _check(dY, "dY", torch.bfloat16, 2)
    _check(offs, "offs", torch.int32, 1)
    _check(dW, "dW", torch.bfloat16, 3)
    rows, K = A.shape
    rows2, N = dY.shape
    E = offs.numel()
    if rows2 != rows or tuple(dW.shape) != (E, K, N):
        raise ValueError("shape mismatch: A[rows,K], dY[rows,N], offs[E], dW[E,K,N]")
    rc = lib().gg_wgrad(_ptr(A), _ptr(dY), _ptr(offs), _ptr(dW), rows, K, N, E,
                        _status_ptr(status), _stream_handle(stream))
    _raise(rc, "gg_wgrad")
    return dW


def wgrad_f32(A: torch.Tensor, dY: torch.Tensor, offs: torch.Tensor, dW: torch.Tensor, *,
              alpha: float = 1.0, beta: float = 1.0, status: Optional[torch.Tensor] = None,
              stream=None) -> torch.Tensor:
    """dW[e] = alpha * A[rows of e]^T @ dY[rows of e] + beta * dW[e], fp32 dW updated in place
    (beta=1 accumulates into a main-grad buffer; beta=0 overwrites without reading dW).

    A bf16 [rows, K], dY bf16 [rows, N], offs int32 [E], dW float32 [E, K, N]."""
    _check(A, "A", torch.bfloat16, 2)
    _check(dY, "dY", torch.bfloat16, 2)
    _check(offs, "offs", torch.int32, 1)
    _check(dW, "dW", torch.float32, 3)
    rows, K = A.shape
    rows2, N = dY.shape
    E = offs.numel()
    if rows2 != rows or tuple(dW.shape) != (E, K, N):
        raise ValueError("shape mismatch: A[rows,K], dY[rows,N], offs[E], dW[E,K,N]")
    rc = lib().gg_wgrad_f32(_ptr(A), _ptr(dY), _ptr(offs), _ptr(dW), float(alpha), float(beta),
                            rows, K, N, E, _status_ptr(status), _stream_handle(stream))
    _raise(rc, "gg_wgrad_f32")
    return dW


def masked_forward(A: torch.Tensor, W: torch.Tensor, masked_m: torch.Tensor,
                   out: torch.Tensor, *, status: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """out[e,r,:] = A[e,r,:] @ W[e] for r < masked_m[e]; other rows of ``out`` untouched.

    A bf16 [E, mmax, K], W bf16 [E, K, N], masked_m int32 [E], out bf16 [E, mmax, N]."""
    _check(A, "A", torch.bfloat16, 3)
    _check(W, "W", torch.bfloat16, 3)
    _check(masked_m, "masked_m", torch.int32, 1)
    _check(out, "out", torch.bfloat16, 3)
    E, mmax, K = A.shape
    E2, K2, N = W.shape
    if E2 != E or K2 != K or masked_m.numel() != E or tuple(out.shape) != (E, mmax, N):
        raise ValueError("shape mismatch: A[E,mmax,K], W[E,K,N], masked_m[E], out[E,mmax,N]")
    rc = lib().gg_masked_forward(_ptr(A), _ptr(W), _ptr(masked_m), _ptr(out), mmax, K, N, E,
                                 _status_ptr(status), _stream_handle(stream))
    _raise(rc, "gg_masked_forward")
    return out


def _check_host(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be a host tensor")
    if t.dtype != dtype or t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d {dtype} tensor")


def layer_step_host(A_h: torch.Tensor, W_h: torch.Tensor, dY_h: torch.Tensor,
                    offs_h: torch.Tensor, out_h: torch.Tensor, dX_h: torch.Tensor,
                    dW_h: torch.Tensor, staging: dict, *, chunks: int = 0,
                    status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Forward + backward of the grouped GEMM layer on host tensors (``gg_layer_step_host``):
    out_h = forward(A_h, W_h), dX_h = dgrad(dY_h, W_h), dW_h = wgrad(A_h, dY_h), streamed
    through the GPU by expert chunks with the copies overlapped with the GEMMs.

    Host tensors (pin them for overlap): A_h bf16 [rows, K], W_h bf16 [E, K, N], dY_h bf16
    [rows, N], offs_h int32 [E]; results out_h [rows, N], dX_h [rows, K], dW_h [E, K, N].
    ``staging`` holds caller-owned CUDA tensors of the same shapes under the keys
    ``A, W, dY, offs, out, dX, dW``. Returns once enqueued on ``stream`` (default: the
    current stream); synchronise it before reading the host results."""
    for t, n, d, k in ((A_h, "A_h", torch.bfloat16, 2), (W_h, "W_h", torch.bfloat16, 3),
                       (dY_h, "dY_h", torch.bfloat16, 2), (offs_h, "offs_h", torch.int32, 1),
                       (out_h, "out_h", torch.bfloat16, 2), (dX_h, "dX_h", torch.bfloat16, 2),
                       (dW_h, "dW_h", torch.bfloat16, 3)):
        _check_host(t, n, d, k)
    host = {"A": A_h, "W": W_h, "dY": dY_h, "offs": offs_h, "out": out_h, "dX": dX_h,
            "dW": dW_h}
    for k, h in host.items():
        if k not in staging:
            raise ValueError(f"staging['{k}'] is missing")
        _check(staging[k], f"staging['{k}']", h.dtype, h.dim())
        if staging[k].shape != h.shape:
            raise ValueError(f"staging['{k}'] must have the shape {tuple(h.shape)}")
    rows, K = A_h.shape
    E, K2, N = W_h.shape
    if (K2 != K or tuple(dY_h.shape) != (rows, N) or offs_h.numel() != E
            or tuple(out_h.shape) != (rows, N) or tuple(dX_h.shape) != (rows, K)
            or tuple(dW_h.shape) != (E, K, N)):
        raise ValueError("shape mismatch: A[rows,K], W[E,K,N], dY[rows,N], offs[E], "
                         "out[rows,N], dX[rows,K], dW[E,K,N]")
    st = staging
    rc = lib().gg_layer_step_host(
        _ptr(A_h), _ptr(W_h), _ptr(dY_h), _ptr(offs_h), _ptr(out_h), _ptr(dX_h), _ptr(dW_h),
        _ptr(st["A"]), _ptr(st["W"]), _ptr(st["dY"]), _ptr(st["offs"]), _ptr(st["out"]),
        _ptr(st["dX"]), _ptr(st["dW"]), rows, K, N, E, int(chunks), _status_ptr(status),
        _stream_handle(stream))
    _raise(rc, "gg_layer_step_host")


def route_workspace_bytes(n_assign: int, E: int) -> int:
    return int(lib().gg_route_workspace_bytes(int(n_assign), int(E)))


def route(topk_ids: torch.Tensor, X: torch.Tensor, E: int, *,
          A_packed: Optional[torch.Tensor] = None, row_of: Optional[torch.Tensor] = None,
          offs: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
          status: Optional[torch.Tensor] = None, stream=None):
    """Token routing into the packed grouped-GEMM layout. Returns (A_packed [T*k, K],
    row_of [T*k], offs [E]); buffers left as None are allocated (uninitialised)."""
    _check(topk_ids, "topk_ids", torch.int32, 2)
    _check(X, "X", torch.bfloat16, 2)
    T, k = topk_ids.shape
    T2, K = X.shape
    if T2 != T:
        raise ValueError("topk_ids[T, k] and X[T, K] disagree on T")
    n = T * k
    dev = X.device
    A_packed = torch.empty((n, K), dtype=X.dtype, device=dev) if A_packed is None else A_packed
    row_of = torch.empty(n, dtype=torch.int32, device=dev) if row_of is None else row_of
    offs = torch.empty(E, dtype=torch.int32, device=dev) if offs is None else offs
    wb = route_workspace_bytes(n, E)
    if workspace is None:
        workspace = torch.empty(max(wb, 4), dtype=torch.uint8, device=dev)
    _check(A_packed, "A_packed", torch.bfloat16, 2)
    _check(row_of, "row_of", torch.int32, 1)
    _check(offs, "offs", torch.int32, 1)
    if tuple(A_packed.shape) != (n, K) or row_of.numel() != n or offs.numel() != E:
        raise ValueError("shape mismatch: A_packed[T*k, K], row_of[T*k], offs[E]")
    rc = lib().gg_route(_ptr(topk_ids), T, k, E, _ptr(X), K, _ptr(A_packed), _ptr(row_of),
                        _ptr(offs), _ptr(workspace), workspace.numel() * workspace.element_size(),
                        _status_ptr(status), _stream_handle(stream))
    _raise(rc, "gg_route")
    return A_packed, row_of, offs


class _GroupedMM(torch.autograd.Function):
    """out = grouped A @ W over the offsets; backward runs dgrad and wgrad on the same
    groups. Output and input gradient are complete tensors (zero past the last offset)."""

    @staticmethod
    def forward(ctx, A, W, offs, w_nk):
        N = W.shape[1] if w_nk else W.shape[2]
        out = torch.empty((A.shape[0], N), dtype=A.dtype, device=A.device)
        forward_ex(A, W, offs, out, zero_tail=True, w_nk=w_nk)
        ctx.save_for_backward(A, W, offs)
        ctx.w_nk = w_nk
        return out

    @staticmethod
    def backward(ctx, dout):
        A, W, offs = ctx.saved_tensors
        dout = dout.contiguous()
        dA = dW = None
        if ctx.needs_input_grad[0]:
            dA = torch.empty_like(A)
            dgrad_ex(dout, W, offs, dA, zero_tail=True, w_nk=ctx.w_nk)
        if ctx.needs_input_grad[1]:
            dW = torch.empty_like(W)
            wgrad_ex(A, dout, offs, dW, w_nk=ctx.w_nk)
        return dA, dW, None, None


def grouped_mm(A: torch.Tensor, W: torch.Tensor, offs: torch.Tensor,
               out: Optional[torch.Tensor] = None, *, w_nk: bool = False) -> torch.Tensor:
    """``torch._grouped_mm(x, w, offs)``-style call (PyTorch issue 152668). With autograd
    (A or W requiring grad) the backward runs gg_dgrad / gg_wgrad and rows past the last
    offset are zero in the output and in dA. Without autograd, ``out`` may be given (rows
    past the last offset are then left as they are)."""
    if torch.is_grad_enabled() and (A.requires_grad or W.requires_grad):
        if out is not None:
            raise ValueError("out= cannot be used with autograd")
        return _GroupedMM.apply(A, W, offs, w_nk)
    if out is None:
        N = W.shape[1] if w_nk else W.shape[2]
        out = torch.empty((A.shape[0], N), dtype=A.dtype, device=A.device)
    return forward_ex(A, W, offs, out, w_nk=w_nk)


__all__ = [
    "forward", "forward_ex", "dgrad", "dgrad_ex", "wgrad", "wgrad_ex", "wgrad_f32",
    "masked_forward", "FLAG_ZERO_TAIL", "FLAG_W_NK", "FLAG_GATE_UP_CONCAT",
    "masked_forward_ex", "ACT_NONE", "ACT_SILU_MUL", "route", "route_workspace_bytes",
    "grouped_mm", "layer_step_host", "status_string", "version",
    "set_watchdog_ns", "testing_skip_first_load", "testing_force_variant", "lib", "GGError",
    "LIB_PATH",
    "DEV_BAD_OFFSETS", "DEV_BAD_MASKED_M", "DEV_TIMEOUT", "DEV_ERROR_MASK", "DEV_LAUNCHED",
    "MAX_EXPERTS",
]
