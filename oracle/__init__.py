"""CPU oracle for the ragged MoE grouped GEMM (fp64 over bf16 inputs).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package; the product library never does. It shares no code
with the CUDA library. The arithmetic lives in ``gg_oracle.c`` (plain loops, OpenMP over
rows); this module marshals numpy arrays into it.

Definitions (see ``gg_oracle.c`` for the passages they follow):
  forward  out[r,:] = A[r,:] @ W[e]            rows r of group e
  dgrad    dX[r,:]  = dY[r,:] @ W[e]^T
  wgrad    dW[e]    = A[group e]^T @ dY[group e]   (exact zeros for an empty group)
  masked   out[e,r,:] = A[e,r,:] @ W[e]       r < clamp(masked_m[e], 0, mmax)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gg_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgg_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2 -fopenmp); returns the shared-library path."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int32
        lib.gg_oracle_group_bounds.argtypes = [P, i32, i64, P, P]
        lib.gg_oracle_group_bounds.restype = ctypes.c_int
        for fn in (lib.gg_oracle_forward_rows, lib.gg_oracle_dgrad_rows):
            fn.argtypes = [P, P, P, i32, i64, i64, i64, P, i64, P, P, ctypes.c_int]
            fn.restype = None
        lib.gg_oracle_wgrad_krows.argtypes = [P, P, P, i32, i64, i64, i64, P, i64, P,
                                              ctypes.c_int]
        lib.gg_oracle_wgrad_krows.restype = None
        lib.gg_oracle_masked_forward_rows.argtypes = [P, P, P, i32, i64, i64, i64, P, i64,
                                                      P, P, ctypes.c_int]
        lib.gg_oracle_masked_forward_rows.restype = ctypes.c_int
        lib.gg_oracle_round_bf16_array.argtypes = [P, i64, P]
        lib.gg_oracle_round_bf16_array.restype = None
        lib.gg_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
        return lib


def default_threads() -> int:
    """Host cores available to this process."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def as_u16(x) -> np.ndarray:
    """bf16 data as a C-contiguous uint16 numpy array (torch bf16 tensors or uint16)."""
    if hasattr(x, "detach"):  # a torch tensor
        import torch
        t = x.detach()
        if t.device.type != "cpu":
            t = t.cpu()
        return np.ascontiguousarray(t.contiguous().view(torch.int16).numpy().view(np.uint16))
    a = np.asarray(x)
    if a.dtype != np.uint16:
        raise TypeError("bf16 data must be a torch.bfloat16 tensor or a uint16 array")
    return np.ascontiguousarray(a)


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def group_bounds(offs, rows_alloc: int):
    """(starts, ends, bad): effective group bounds under the clamp rule."""
    o = np.ascontiguousarray(np.asarray(offs, dtype=np.int32))
    E = len(o)
    s = np.zeros(E, np.int64)
    e = np.zeros(E, np.int64)
    bad = _load().gg_oracle_group_bounds(_ptr(o), E, rows_alloc, _ptr(s), _ptr(e))
    return s, e, bool(bad)


def _rows(rows, n):
    if rows is None:
        return np.arange(n, dtype=np.int64)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    if r.size and (r.min() < 0 or r.max() >= n):
        raise IndexError("row index out of range")
    return r


def forward(A, W, offs, rows=None, threads=None):
    """fp64 forward on ``rows`` (default: all). Returns (out[nrows,N], group_of[nrows]);
    rows in no group come back NaN with group -1."""
    A, W = as_u16(A), as_u16(W)
    o = np.ascontiguousarray(np.asarray(offs, dtype=np.int32))
    rows_alloc, K = A.shape
    E, K2, N = W.shape
    assert K2 == K and len(o) == E
    r = _rows(rows, rows_alloc)
    out = np.empty((len(r), N), np.float64)
    g = np.empty(len(r), np.int32)
    _load().gg_oracle_forward_rows(_ptr(A), _ptr(W), _ptr(o), E, rows_alloc, K, N, _ptr(r),
                                   len(r), _ptr(out), _ptr(g), threads or default_threads())
    return out, g


def dgrad(dY, W, offs, rows=None, threads=None):
    """fp64 dgrad on ``rows``. Returns (dX[nrows,K], group_of[nrows])."""
    dY, W = as_u16(dY), as_u16(W)
    o = np.ascontiguousarray(np.asarray(offs, dtype=np.int32))
    rows_alloc, N = dY.shape
    E, K, N2 = W.shape
    assert N2 == N and len(o) == E
    r = _rows(rows, rows_alloc)
    out = np.empty((len(r), K), np.float64)
    g = np.empty(len(r), np.int32)
    _load().gg_oracle_dgrad_rows(_ptr(dY), _ptr(W), _ptr(o), E, rows_alloc, K, N, _ptr(r),
                                 len(r), _ptr(out), _ptr(g), threads or default_threads())
    return out, g


def wgrad(A, dY, offs, E=None, ks=None, threads=None):
    """fp64 wgrad for the K-rows ``ks`` (default: all). Returns dW[E, len(ks), N]."""
    A, dY = as_u16(A), as_u16(dY)
    o = np.ascontiguousarray(np.asarray(offs, dtype=np.int32))
    rows_alloc, K = A.shape
    rows2, N = dY.shape
    assert rows2 == rows_alloc
    E = len(o) if E is None else E
    assert len(o) == E
    k = _rows(ks, K)
    out = np.empty((E, len(k), N), np.float64)
    _load().gg_oracle_wgrad_krows(_ptr(A), _ptr(dY), _ptr(o), E, rows_alloc, K, N, _ptr(k),
                                  len(k), _ptr(out), threads or default_threads())
    return out


def wgrad_accumulate(A, dY, offs, old, alpha: float, beta: float, ks=None, threads=None):
    """fp64 reference of the fp32 wgrad with scaling and accumulation:
    dW[e, k, n] = alpha * sum_{r in group e} A[r,k] dY[r,n] + beta * old[e, k, n]
    (TransformerEngine PR 3542, "Changes": FP32 outputs, fused accumulation, explicit
    alpha/beta). ``old`` is the fp32 buffer before the call ([E, K, N]); with beta == 0 it
    is not read (so NaN there does not matter). Returns dW[E, len(ks), N]."""
    prod = wgrad(A, dY, offs, ks=ks, threads=threads)
    out = float(alpha) * prod
    if beta != 0.0:
        o = np.asarray(old, dtype=np.float32).astype(np.float64)
        kk = np.arange(o.shape[1]) if ks is None else np.asarray(ks, dtype=np.int64)
        out = out + float(beta) * o[:, kk, :]
    return out


def epilogue(h, groups, rows, bias=None, bias_scale=None, act: int = 0, concat: bool = False):
    """The forward epilogue on fp64 products h[nrows, N] of rows ``rows`` whose groups are
    ``groups`` (rows in no group stay NaN):
      h'[r, n] = h[r, n] + s[r] * bias[e(r), n]      (s = bias_scale, 1 when absent)
    act 0: h'; act 1 (SiLU-and-mul), gate/up interleaved in blocks of 128 columns:
      out[r, 128 b + i] = silu(h'[r, 256 b + i]) * h'[r, 256 b + 128 + i],
    or, with concat, gate and up as the two halves of the N columns:
      out[r, j] = silu(h'[r, j]) * h'[r, N/2 + j],
    silu(x) = x / (1 + exp(-x))
    (TransformerEngine PR 3542 review: per-group bias and a per-token bias scale over the
    logical rows; sglang PR 32385, "Cause": SiLU-and-mul between the gate-up and down GEMMs)."""
    h = np.array(h, dtype=np.float64, copy=True)
    g = np.asarray(groups)
    live = g >= 0
    if bias is not None:
        b = bf16_to_f64(as_u16(bias))
        s = np.ones(len(h)) if bias_scale is None else np.asarray(bias_scale, np.float64)[rows]
        h[live] += s[live, None] * b[g[live]]
    if act == 0:
        return h
    N = h.shape[1]
    assert N % 256 == 0
    if concat:
        gate, up = h[:, : N // 2], h[:, N // 2:]
        return gate / (1.0 + np.exp(-gate)) * up
    nb = N // 256
    hv = h.reshape(len(h), nb, 2, 128)
    gate, up = hv[:, :, 0, :], hv[:, :, 1, :]
    out = gate / (1.0 + np.exp(-gate)) * up
    return out.reshape(len(h), N // 2)


def forward_ex(A, W, offs, bias=None, bias_scale=None, act: int = 0, rows=None, threads=None,
               concat: bool = False):
    """Forward with the epilogue above. Returns (out[nrows, N or N/2], group_of[nrows])."""
    h, g = forward(A, W, offs, rows=rows, threads=threads)
    r = np.arange(h.shape[0]) if rows is None else np.asarray(rows, np.int64)
    return epilogue(h, g, r, bias, bias_scale, act, concat), g


def masked_forward_ex(A, W, masked_m, bias=None, bias_scale=None, act: int = 0, rows=None,
                      threads=None, concat: bool = False):
    """Masked forward with the epilogue above; bias_scale is indexed by flat row e*mmax+r.
    Returns (out, active, bad)."""
    h, act_rows, bad = masked_forward(A, W, masked_m, rows=rows, threads=threads)
    E, mmax, _ = as_u16(A).shape
    r = np.arange(E * mmax) if rows is None else np.asarray(rows, np.int64)
    g = np.where(act_rows, r // mmax, -1)
    return epilogue(h, g, r, bias, bias_scale, act, concat), act_rows, bad


def route(topk_ids, X, E: int):
    """Token routing into the packed grouped-GEMM layout (the step before the path:
    torchtitan's generate_permute_indices in PyTorch issue 152668, here without alignment
    padding). Assignment i = t*k + s sends token t to expert topk_ids[t, s]; ids < 0 or
    >= E are dropped. Rows are ordered by expert, and within an expert by assignment index
    (a stable sort). Returns (offs int32[E] cumulative ends, row_of int32[T*k] with -1 for
    dropped assignments, A_packed bf16-as-uint16 [total, K], bad: any id >= E)."""
    ids = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    Xu = as_u16(X)
    k = np.asarray(topk_ids).shape[1]
    valid = (ids >= 0) & (ids < E)
    order = np.argsort(np.where(valid, ids, E), kind="stable")[: int(valid.sum())]
    counts = np.bincount(ids[valid], minlength=E)
    offs = np.cumsum(counts).astype(np.int32)
    row_of = np.full(len(ids), -1, np.int32)
    row_of[order] = np.arange(len(order), dtype=np.int32)
    A_packed = Xu[order // k]
    return offs, row_of, A_packed, bool(np.any(ids >= E))


def masked_forward(A, W, masked_m, rows=None, threads=None):
    """fp64 masked forward on flat rows e*mmax+r (default: all). Returns
    (out[nrows,N], active[nrows], bad)."""
    A, W = as_u16(A), as_u16(W)
    m = np.ascontiguousarray(np.asarray(masked_m, dtype=np.int32))
    E, mmax, K = A.shape
    E2, K2, N = W.shape
    assert E2 == E and K2 == K and len(m) == E
    r = _rows(rows, E * mmax)
    out = np.empty((len(r), N), np.float64)
    act = np.empty(len(r), np.int32)
    bad = _load().gg_oracle_masked_forward_rows(_ptr(A), _ptr(W), _ptr(m), E, mmax, K, N,
                                                _ptr(r), len(r), _ptr(out), _ptr(act),
                                                threads or default_threads())
    return out, act.astype(bool), bool(bad)


def round_bf16(x) -> np.ndarray:
    """Round fp64 values to bf16 bit patterns (nearest, ties to even)."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty(a.shape, np.uint16)
    _load().gg_oracle_round_bf16_array(_ptr(a), a.size, _ptr(out))
    return out


def bf16_to_f64(u16) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp64."""
    a = np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16
    return a.view(np.float32).astype(np.float64)


def untouched_rows(offs, rows_alloc: int) -> np.ndarray:
    """Rows of out/dX that no group covers (at and past the last effective end)."""
    _, ends, _ = group_bounds(offs, rows_alloc)
    last = int(ends[-1]) if len(ends) else 0
    return np.arange(last, rows_alloc, dtype=np.int64)
