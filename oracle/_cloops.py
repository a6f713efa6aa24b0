"""ctypes access to ``oracle/loops.c`` (fp64 loops), built with gcc on demand.

Test infrastructure only (see ``oracle/__init__``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "loops.c")
_LIB = os.path.join(_HERE, "liboracle_loops.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile loops.c into liboracle_loops.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            p = ctypes.c_void_p
            i64 = ctypes.c_int64
            d = ctypes.c_double
            L.oracle_causal_conv.argtypes = [p, p, p, p, i64, i64, p]
            L.oracle_causal_conv_at.argtypes = [p, p, p, p, i64, i64, p, i64, p]
            L.oracle_power_kernel.argtypes = [p, p, p, i64, i64, i64, i64, d, p, p, p]
            L.oracle_recurrence_dense.argtypes = [p, p, p, p, p, i64, i64, p, i64, p, p]
            L.oracle_recurrence_diag.argtypes = [p, p, p, p, p, i64, i64, p, i64, p, p]
            for f in (L.oracle_causal_conv, L.oracle_causal_conv_at, L.oracle_power_kernel,
                      L.oracle_recurrence_dense, L.oracle_recurrence_diag):
                f.restype = None
            _lib = L
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def causal_conv(u, K, D, row_h):
    """u: [rows, L]; K: [H, L]; D: [H]; row_h: [rows] -> y [rows, L] (fp64)."""
    u = _c(u, np.float64); K = _c(K, np.float64); D = _c(D, np.float64)
    row_h = _c(row_h, np.int64)
    rows, L = u.shape
    y = np.empty((rows, L), np.float64)
    lib().oracle_causal_conv(_ptr(u), _ptr(K), _ptr(D), _ptr(row_h), rows, L, _ptr(y))
    return y


def causal_conv_at(u, K, D, row_h, ts):
    u = _c(u, np.float64); K = _c(K, np.float64); D = _c(D, np.float64)
    row_h = _c(row_h, np.int64); ts = _c(ts, np.int64)
    rows, L = u.shape
    y = np.empty((rows, len(ts)), np.float64)
    lib().oracle_causal_conv_at(_ptr(u), _ptr(K), _ptr(D), _ptr(row_h), rows, L,
                                _ptr(ts), len(ts), _ptr(y))
    return y


def power_kernel(A, v0, C, L, max_periods, rel_tol):
    """A: [H,N,N], v0, C: [H,N] complex -> (K_re, K_im [H,L], periods [H])."""
    A = _c(A, np.complex128); v0 = _c(v0, np.complex128); C = _c(C, np.complex128)
    H, N = v0.shape
    if N > 512:
        raise ValueError("N > 512")
    Kr = np.empty((H, L)); Ki = np.empty((H, L)); per = np.empty(H, np.int64)
    lib().oracle_power_kernel(_ptr(A), _ptr(v0), _ptr(C), H, N, L, max_periods, rel_tol,
                              _ptr(Kr), _ptr(Ki), _ptr(per))
    return Kr, Ki, per


def recurrence_dense(A, B, C, D, row_h, u, x0=None):
    A = _c(A, np.complex128); B = _c(B, np.complex128); C = _c(C, np.complex128)
    D = _c(D, np.float64); row_h = _c(row_h, np.int64); u = _c(u, np.float64)
    rows, T = u.shape
    N = B.shape[1]
    x = np.zeros((rows, N), np.complex128) if x0 is None else _c(x0, np.complex128).copy()
    y = np.empty((rows, T))
    lib().oracle_recurrence_dense(_ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(row_h), rows, N,
                                  _ptr(u), T, _ptr(x), _ptr(y))
    return y, x


def recurrence_diag(a, b, c, D, row_h, u, x0=None):
    a = _c(a, np.complex128); b = _c(b, np.complex128); c = _c(c, np.complex128)
    D = _c(D, np.float64); row_h = _c(row_h, np.int64); u = _c(u, np.float64)
    rows, T = u.shape
    Nh = a.shape[1]
    x = np.zeros((rows, Nh), np.complex128) if x0 is None else _c(x0, np.complex128).copy()
    y = np.empty((rows, T))
    lib().oracle_recurrence_diag(_ptr(a), _ptr(b), _ptr(c), _ptr(D), _ptr(row_h), rows, Nh,
                                 _ptr(u), T, _ptr(x), _ptr(y))
    return y, x
