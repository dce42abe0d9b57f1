"""CPU oracle for the fused Linear + epilogue path (test infrastructure only).

This package wraps ``fle_oracle.c`` -- plain C loops in fp64 -- with ctypes.
Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline / reference leg may import it; the CUDA library never does, and the
two share no code.  What each function computes, and the page passage it
follows, is stated in ``fle_oracle.c``.

Epilogue numbering here is the oracle's own (``EPI_*`` below).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fle_oracle.c")
_LIB = os.path.join(_HERE, "liborc.so")

EPI_SCALE_HARDTANH_GELU = 0
EPI_SWISH_SCALE = 1
EPI_AVGPOOL_GELU_SCALE_ROWMAX = 2
EPI_NONE = 3

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2 -fopenmp, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    i64, dbl, vp = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    lib.orc_num_threads.restype = ctypes.c_int
    lib.orc_gelu.argtypes = [dbl]
    lib.orc_gelu.restype = dbl
    lib.orc_gelu_tanh.argtypes = [dbl]
    lib.orc_gelu_tanh.restype = dbl
    lib.orc_scale_hardtanh_gelu.argtypes = [dbl, dbl, dbl, dbl]
    lib.orc_scale_hardtanh_gelu.restype = dbl
    lib.orc_swish_scale.argtypes = [dbl, dbl]
    lib.orc_swish_scale.restype = dbl
    lib.orc_pool_windows.argtypes = [i64, i64, i64]
    lib.orc_pool_windows.restype = i64
    lib.orc_pool_gelu_scale_max.argtypes = [vp, i64, i64, i64, dbl]
    lib.orc_pool_gelu_scale_max.restype = dbl
    lib.orc_linear_rows.argtypes = [vp, vp, vp, i64, i64, i64, vp, i64, vp]
    lib.orc_linear_rows.restype = None
    lib.orc_forward_rows.argtypes = [vp, vp, vp, i64, i64, i64, ctypes.c_int,
                                     dbl, dbl, dbl, i64, i64, ctypes.c_int, vp, i64, vp, vp]
    lib.orc_forward_rows.restype = ctypes.c_int
    _lib = lib
    return lib


def _f32(a):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().orc_num_threads())


def gelu(v: float) -> float:
    return float(_load().orc_gelu(float(v)))


def gelu_tanh(v: float) -> float:
    """GELU in its tanh form (page l2_p53's first fused kernel)."""
    return float(_load().orc_gelu_tanh(float(v)))


def scale_hardtanh_gelu(y: float, s: float = 0.5, lo: float = -2.0, hi: float = 2.0) -> float:
    return float(_load().orc_scale_hardtanh_gelu(float(y), float(s), float(lo), float(hi)))


def swish_scale(y: float, s: float = 2.0) -> float:
    return float(_load().orc_swish_scale(float(y), float(s)))


def pool_windows(N: int, k: int = 16, stride: int | None = None) -> int:
    return int(_load().orc_pool_windows(int(N), int(k), int(k if stride is None else stride)))


def pool_gelu_scale_max(yrow, k: int = 16, stride: int | None = None, s: float = 2.0) -> float:
    y = np.ascontiguousarray(np.asarray(yrow, dtype=np.float64))
    return float(_load().orc_pool_gelu_scale_max(_ptr(y), y.shape[0], int(k),
                                                 int(k if stride is None else stride), float(s)))


def linear_rows(x, W, b, rows=None) -> np.ndarray:
    """fp64 y = x W^T + b for the given rows of x (all rows if None)."""
    x, W = _f32(x), _f32(W)
    b = None if b is None else _f32(b)
    M, K = x.shape
    N = W.shape[0]
    assert W.shape[1] == K and (b is None or b.shape == (N,))
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    y = np.empty((rows.shape[0], N), dtype=np.float64)
    _load().orc_linear_rows(_ptr(x), _ptr(W), _ptr(b), M, K, N, _ptr(rows), rows.shape[0], _ptr(y))
    return y


def forward_rows(x, W, b, kind: int, scale: float = 1.0, clamp_lo: float = -2.0,
                 clamp_hi: float = 2.0, pool_k: int = 16, pool_stride: int | None = None,
                 rows=None, gelu_tanh: bool = False) -> np.ndarray:
    """The whole path (linear + epilogue ``kind``) for the given rows, fp32 result.

    Returns [len(rows), N] for the elementwise kinds and [len(rows)] for the
    pool / row-max kind.  gelu_tanh: GELU in its tanh form for (a) and (c).
    """
    x, W = _f32(x), _f32(W)
    b = None if b is None else _f32(b)
    M, K = x.shape
    N = W.shape[0]
    assert W.shape[1] == K and (b is None or b.shape == (N,))
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    R = rows.shape[0]
    out = np.empty((R,) if kind == EPI_AVGPOOL_GELU_SCALE_ROWMAX else (R, N), dtype=np.float32)
    rc = _load().orc_forward_rows(_ptr(x), _ptr(W), _ptr(b), M, K, N, int(kind), float(scale),
                                  float(clamp_lo), float(clamp_hi), int(pool_k),
                                  int(pool_k if pool_stride is None else pool_stride), int(bool(gelu_tanh)),
                                  _ptr(rows), R, _ptr(out), None)
    if rc != 0:
        raise ValueError("oracle rejected the arguments (rc=%d)" % rc)
    return out


# The three page problems as (kind, scale) presets.
PROBLEMS = {
    "scale_hardtanh_gelu": dict(kind=EPI_SCALE_HARDTANH_GELU, scale=0.5, clamp_lo=-2.0, clamp_hi=2.0),
    "swish_scale": dict(kind=EPI_SWISH_SCALE, scale=2.0),
    "avgpool_gelu_scale_rowmax": dict(kind=EPI_AVGPOOL_GELU_SCALE_ROWMAX, scale=2.0, pool_k=16),
    "none": dict(kind=EPI_NONE),
}
