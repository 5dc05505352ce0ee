"""ctypes wrapper of synth.c (see that file for the generator definition)."""
import ctypes
import os
import subprocess

import numpy as np

__all__ = ["bf16_normal", "mix64", "normal_at", "stream_key", "build_synth"]

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "synth.c")
LIB = os.path.join(HERE, "libsynth.so")
_lib = None


def build_synth(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and \
            os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    subprocess.run(["gcc", "-std=c11", "-O2", "-fno-fast-math",
                    "-ffp-contract=off", "-fPIC", "-shared", "-Wall", "-o",
                    tmp, SRC, "-lm", "-lpthread"], check=True)
    os.replace(tmp, LIB)
    return LIB


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_synth())
        lib.synth_mix64.argtypes = [ctypes.c_uint64]
        lib.synth_mix64.restype = ctypes.c_uint64
        lib.synth_key.argtypes = [ctypes.c_uint64] * 3
        lib.synth_key.restype = ctypes.c_uint64
        lib.synth_normal_at.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_normal_at.restype = ctypes.c_double
        lib.synth_bf16_normal.argtypes = [
            ctypes.c_uint64, ctypes.c_uint64, ctypes.c_double,
            ctypes.c_double, ctypes.c_double, ctypes.c_void_p,
            ctypes.c_int64, ctypes.c_int]
        lib.synth_bf16_normal.restype = ctypes.c_int
        _lib = lib
    return _lib


def mix64(z: int) -> int:
    return _L().synth_mix64(z & (2**64 - 1))


def stream_key(seed: int, tensor_id: int, stream: int) -> int:
    return _L().synth_key(seed, tensor_id, stream)


def normal_at(key: int, i: int) -> float:
    return _L().synth_normal_at(key, i)


def _threads():
    try:
        return max(1, min(64, len(os.sched_getaffinity(0))))
    except AttributeError:
        return max(1, min(64, os.cpu_count() or 1))


def bf16_normal(shape, seed: int, tensor_id: int, std: float,
                outlier_p: float = 0.0, outlier_factor: float = 1.0,
                out=None) -> np.ndarray:
    """bf16 (uint16 bit patterns) ~ std*N(0,1), a fraction outlier_p scaled."""
    shape = tuple(int(s) for s in shape)
    count = int(np.prod(shape)) if shape else 1
    if out is None:
        out = np.empty(shape, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous
    assert out.size == count
    rc = _L().synth_bf16_normal(seed, tensor_id, std, outlier_p,
                                outlier_factor, out.ctypes.data, count,
                                _threads())
    assert rc == 0
    return out
