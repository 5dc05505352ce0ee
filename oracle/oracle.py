"""ctypes wrapper of the C oracle (test infrastructure).

Every function takes and returns numpy arrays. bf16 tensors are uint16 bit
patterns; codes are uint8; scales float32; GEMM references float64.
Layouts (all row-major):
  row-wise 1x128 : q [rows, cols], s [ceil(cols/128), rows]
  col-wise 128x1 : q_t [cols, rows], s_t [ceil(rows/128), cols]
  weight 128x128 : q [n, k], s [ceil(n/128), ceil(k/128)], q_t [k, n]
"""
import ctypes
import os

import numpy as np

from . import build as _build

__all__ = [
    "e4m3_decode", "e4m3_decode_table", "e4m3_encode", "group_scale",
    "bf16_round", "bf16_to_float", "quantize_rowwise", "quantize_colwise",
    "quantize_weight_block", "gemm_fprop", "gemm_dgrad", "gemm_wgrad",
    "gemm_fprop_points", "gemm_dgrad_points", "gemm_wgrad_points",
    "default_threads",
]

_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.orc_e4m3_decode.restype = ctypes.c_double
        lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
        lib.orc_e4m3_encode.restype = ctypes.c_uint8
        lib.orc_e4m3_encode_array.argtypes = [P, I64, P]
        lib.orc_e4m3_encode_array.restype = None
        for name in ("orc_group_scale", "orc_group_scale_pow2"):
            getattr(lib, name).argtypes = [ctypes.c_float, P, P]
            getattr(lib, name).restype = None
        lib.orc_bf16_round.argtypes = [ctypes.c_double]
        lib.orc_bf16_round.restype = ctypes.c_uint16
        lib.orc_bf16_to_float.argtypes = [ctypes.c_uint16]
        lib.orc_bf16_to_float.restype = ctypes.c_float
        for name in ("orc_quantize_rowwise", "orc_quantize_colwise",
                     "orc_quantize_rowwise_pow2", "orc_quantize_colwise_pow2"):
            getattr(lib, name).argtypes = [P, I64, I64, P, P]
            getattr(lib, name).restype = ctypes.c_int
        for name in ("orc_quantize_weight_block",
                     "orc_quantize_weight_block_pow2"):
            getattr(lib, name).argtypes = [P, I64, I64, P, P, P]
            getattr(lib, name).restype = ctypes.c_int
        for name in ("orc_gemm_fprop", "orc_gemm_dgrad", "orc_gemm_wgrad"):
            getattr(lib, name).argtypes = [P, P, P, P, I64, I64, I64, P, P,
                                           ctypes.c_int]
            getattr(lib, name).restype = ctypes.c_int
        for name in ("orc_gemm_fprop_points", "orc_gemm_dgrad_points",
                     "orc_gemm_wgrad_points"):
            getattr(lib, name).argtypes = [P, P, P, P, I64, I64, I64, P, P,
                                           I64, P, P, ctypes.c_int]
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


def default_threads() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") \
        else (os.cpu_count() or 1)


def _p(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError("expected %s, got %s" % (dtype, a.dtype))
    return a


def _cdiv(a, b):
    return (a + b - 1) // b


# ---------------------------------------------------------------- codec

def e4m3_decode(code: int) -> float:
    return _L().orc_e4m3_decode(int(code) & 0xFF)


def e4m3_decode_table() -> np.ndarray:
    return np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(t) -> np.ndarray:
    """fp32 values (array-like) -> E4M3 codes (RNE, satfinite)."""
    t = np.ascontiguousarray(np.asarray(t, dtype=np.float32))
    out = np.empty(t.shape, dtype=np.uint8)
    _L().orc_e4m3_encode_array(_p(t), t.size, _p(out))
    return out


def group_scale(amax: float, pow2=False):
    """(qscale, s) of a group with this amax; pow2 selects the power-of-two
    scale form."""
    q = ctypes.c_float()
    s = ctypes.c_float()
    fn = _L().orc_group_scale_pow2 if pow2 else _L().orc_group_scale
    fn(ctypes.c_float(amax), ctypes.byref(q), ctypes.byref(s))
    return np.float32(q.value), np.float32(s.value)


def bf16_round(v) -> np.ndarray:
    v = np.asarray(v, dtype=np.float64)
    f = _L().orc_bf16_round
    out = np.fromiter((f(float(x)) for x in v.ravel()), dtype=np.uint16,
                      count=v.size)
    return out.reshape(v.shape)


def bf16_to_float(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- quantisers

def quantize_rowwise(x, pow2=False):
    x = _c(x, np.uint16)
    rows, cols = x.shape
    q = np.empty((rows, cols), np.uint8)
    s = np.empty((_cdiv(cols, 128), rows), np.float32)
    fn = _L().orc_quantize_rowwise_pow2 if pow2 else _L().orc_quantize_rowwise
    rc = fn(_p(x), rows, cols, _p(q), _p(s))
    assert rc == 0
    return q, s


def quantize_colwise(x, pow2=False):
    x = _c(x, np.uint16)
    rows, cols = x.shape
    q_t = np.empty((cols, rows), np.uint8)
    s_t = np.empty((_cdiv(rows, 128), cols), np.float32)
    fn = _L().orc_quantize_colwise_pow2 if pow2 else _L().orc_quantize_colwise
    rc = fn(_p(x), rows, cols, _p(q_t), _p(s_t))
    assert rc == 0
    return q_t, s_t


def quantize_weight_block(w, want_transposed=True, pow2=False):
    w = _c(w, np.uint16)
    n, k = w.shape
    q = np.empty((n, k), np.uint8)
    s = np.empty((_cdiv(n, 128), _cdiv(k, 128)), np.float32)
    q_t = np.empty((k, n), np.uint8) if want_transposed else None
    fn = _L().orc_quantize_weight_block_pow2 if pow2 else \
        _L().orc_quantize_weight_block
    rc = fn(_p(w), n, k, _p(q), _p(s), _p(q_t))
    assert rc == 0
    return q, s, q_t


# ---------------------------------------------------------------- GEMMs

def _gemm(name, qa, sa, qb, sb, m, n, k, out_shape, with_bound, nthreads):
    qa = _c(qa, np.uint8)
    qb = _c(qb, np.uint8)
    sa = _c(sa, np.float32)
    sb = _c(sb, np.float32)
    acc = np.empty(out_shape, np.float64)
    bound = np.empty(out_shape, np.float64) if with_bound else None
    nt = default_threads() if nthreads is None else nthreads
    rc = getattr(_L(), name)(_p(qa), _p(sa), _p(qb), _p(sb), m, n, k,
                             _p(acc), _p(bound), nt)
    assert rc == 0
    return (acc, bound) if with_bound else acc


def gemm_fprop(qx, sx, qw, sw, with_bound=False, nthreads=None):
    """Y[m, n] (fp64) from row-wise qX [m, k] and weight qW [n, k]."""
    m, k = qx.shape
    n = qw.shape[0]
    return _gemm("orc_gemm_fprop", qx, sx, qw, sw, m, n, k, (m, n),
                 with_bound, nthreads)


def gemm_dgrad(qdy, sdy, qw, sw, with_bound=False, nthreads=None):
    """dX[m, k] (fp64) from row-wise qdY [m, n] and weight qW [n, k]."""
    m, n = qdy.shape
    k = qw.shape[1]
    return _gemm("orc_gemm_dgrad", qdy, sdy, qw, sw, m, n, k, (m, k),
                 with_bound, nthreads)


def gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t, with_bound=False, nthreads=None):
    """dW[n, k] (fp64) from col-wise qdY^T [n, m] and qX^T [k, m]."""
    n, m = qdy_t.shape
    k = qx_t.shape[0]
    return _gemm("orc_gemm_wgrad", qdy_t, sdy_t, qx_t, sx_t, m, n, k, (n, k),
                 with_bound, nthreads)


def _gemm_pts(name, qa, sa, qb, sb, m, n, k, pi, pj, nthreads):
    qa = _c(qa, np.uint8)
    qb = _c(qb, np.uint8)
    sa = _c(sa, np.float32)
    sb = _c(sb, np.float32)
    pi = _c(np.asarray(pi, dtype=np.int64), np.int64)
    pj = _c(np.asarray(pj, dtype=np.int64), np.int64)
    acc = np.empty(pi.shape, np.float64)
    bound = np.empty(pi.shape, np.float64)
    nt = default_threads() if nthreads is None else nthreads
    rc = getattr(_L(), name)(_p(qa), _p(sa), _p(qb), _p(sb), m, n, k,
                             _p(pi), _p(pj), pi.size, _p(acc), _p(bound), nt)
    if rc != 0:
        raise ValueError("bad point list")
    return acc, bound


def gemm_fprop_points(qx, sx, qw, sw, pi, pj, nthreads=None):
    m, k = qx.shape
    n = qw.shape[0]
    return _gemm_pts("orc_gemm_fprop_points", qx, sx, qw, sw, m, n, k, pi, pj,
                     nthreads)


def gemm_dgrad_points(qdy, sdy, qw, sw, pi, pj, nthreads=None):
    m, n = qdy.shape
    k = qw.shape[1]
    return _gemm_pts("orc_gemm_dgrad_points", qdy, sdy, qw, sw, m, n, k, pi,
                     pj, nthreads)


def gemm_wgrad_points(qdy_t, sdy_t, qx_t, sx_t, pi, pj, nthreads=None):
    n, m = qdy_t.shape
    k = qx_t.shape[0]
    return _gemm_pts("orc_gemm_wgrad_points", qdy_t, sdy_t, qx_t, sx_t, m, n,
                     k, pi, pj, nthreads)
