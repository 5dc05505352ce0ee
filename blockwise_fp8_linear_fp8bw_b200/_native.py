"""Loader of libfp8bw.so (the library's C ABI, include/fp8bw.h).

The shared library is built in-tree by build.py. There is no fallback: if it
cannot be loaded, importing this module raises.
"""
import ctypes
import os

from . import build as _build

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int

class WeightBlockJob(ctypes.Structure):
    """fp8bw_weight_block_job of include/fp8bw.h."""
    _fields_ = [("w", _P), ("n", _I64), ("k", _I64), ("q", _P), ("s", _P),
                ("q_t", _P)]


class WgradJob(ctypes.Structure):
    """fp8bw_wgrad_job of include/fp8bw.h."""
    _fields_ = [("qdy_t", _P), ("sdy_t", _P), ("qx_t", _P), ("sx_t", _P),
                ("m", _I64), ("n", _I64), ("k", _I64), ("dw", _P)]


# name -> (argtypes, restype), in the order of include/fp8bw.h
SIGNATURES = {
    "fp8bw_quantize_rowwise": ([_P, _I64, _I64, _P, _P, _P], _INT),
    "fp8bw_quantize_colwise": ([_P, _I64, _I64, _P, _P, _P, _P, _P], _INT),
    "fp8bw_quantize_weight_block": ([_P, _I64, _I64, _P, _P, _P, _P], _INT),
    "fp8bw_quantize_weight_block_batch": ([_P, _INT, _P], _INT),
    "fp8bw_gemm_fprop": ([_P, _P, _P, _P, _I64, _I64, _I64, _P, _P], _INT),
    "fp8bw_gemm_dgrad": ([_P, _P, _P, _INT, _P, _I64, _I64, _I64, _P, _P],
                         _INT),
    "fp8bw_gemm_wgrad": ([_P, _P, _P, _P, _I64, _I64, _I64, _P, _P], _INT),
    "fp8bw_gemm_wgrad_f32": ([_P, _P, _P, _P, _I64, _I64, _I64, _P, _INT,
                              _P], _INT),
    "fp8bw_gemm_wgrad_batch": ([_P, _INT, _P], _INT),
    "fp8bw_gemm_wgrad_f32_batch": ([_P, _INT, _INT, _P], _INT),
    "fp8bw_gemm_fprop_quant": ([_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P,
                                _P], _INT),
    "fp8bw_gemm_dgrad_quant": ([_P, _P, _P, _INT, _P, _I64, _I64, _I64, _P, _P,
                                _P, _P], _INT),
    "fp8bw_gemm_fprop_quant_rowcol": ([_P, _P, _P, _P, _I64, _I64, _I64, _P, _P,
                                       _P, _P, _P, _P], _INT),
    "fp8bw_gemm_dgrad_quant_rowcol": ([_P, _P, _P, _INT, _P, _I64, _I64, _I64, _P,
                                       _P, _P, _P, _P, _P], _INT),
    "fp8bw_quantize_rowwise_pow2": ([_P, _I64, _I64, _P, _P, _P], _INT),
    "fp8bw_quantize_colwise_pow2": ([_P, _I64, _I64, _P, _P, _P, _P, _P], _INT),
    "fp8bw_quantize_weight_block_pow2": ([_P, _I64, _I64, _P, _P, _P, _P], _INT),
    "fp8bw_quantize_weight_block_batch_pow2": ([_P, _INT, _P], _INT),
    "fp8bw_gemm_fprop_pow2": ([_P, _P, _P, _P, _I64, _I64, _I64, _P, _P], _INT),
    "fp8bw_gemm_dgrad_pow2": ([_P, _P, _P, _INT, _P, _I64, _I64, _I64, _P,
                               _P], _INT),
    "fp8bw_gemm_wgrad_pow2": ([_P, _P, _P, _P, _I64, _I64, _I64, _P, _P], _INT),
    "fp8bw_gemm_wgrad_f32_pow2": ([_P, _P, _P, _P, _I64, _I64, _I64, _P, _INT,
                                   _P], _INT),
    "fp8bw_gemm_wgrad_batch_pow2": ([_P, _INT, _P], _INT),
    "fp8bw_gemm_wgrad_f32_batch_pow2": ([_P, _INT, _INT, _P], _INT),
    "fp8bw_selftest_wait_timeout": ([_I64, _P], _INT),
    "fp8bw_check_device_error": ([_P], _INT),
    "fp8bw_status_string": ([_INT], ctypes.c_char_p),
    "fp8bw_version": ([], _INT),
}

LIB_PATH = _build.LIB
_lib = None


def load():
    """Load (building first if the sources are newer) and return the CDLL."""
    global _lib
    if _lib is None:
        if _build.needs_build():
            _build.build()
        if not os.path.exists(LIB_PATH):
            raise ImportError("libfp8bw.so is missing and could not be built")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (argtypes, restype) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = argtypes
            fn.restype = restype
        _lib = lib
    return _lib
