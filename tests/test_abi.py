"""The C ABI without a GPU: every symbol declared in include/fp8bw.h is
exported by libfp8bw.so, and the host-side argument checks reject bad calls
before anything touches the device (fake pointer values are never
dereferenced because each call below fails validation first)."""
import ctypes
import os
import re

import pytest

from blockwise_fp8_linear_fp8bw_b200 import _native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8bw.h")

OK, E_NULL, E_SHAPE, E_ALIGN, E_DEVICE, E_LAUNCH, E_TIMEOUT, E_CUDA, E_ALIAS = \
    0, -1, -2, -3, -4, -5, -6, -7, -8
E_SCALE = -9

A = 0x10000000   # fake, 16-byte aligned, never dereferenced
B = 0x20000000
C = 0x30000000
D = 0x40000000
E = 0x50000000


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp8bw_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return _native.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) == 28
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_native.SIGNATURES)


def test_status_strings_and_version(lib):
    assert lib.fp8bw_version() == 108
    for st in (OK, E_NULL, E_SHAPE, E_ALIGN, E_DEVICE, E_LAUNCH, E_TIMEOUT,
               E_CUDA, E_ALIAS, E_SCALE):
        s = lib.fp8bw_status_string(st).decode()
        assert s and s != "unknown status"
    assert lib.fp8bw_status_string(12345).decode() == "unknown status"


def test_null_pointers_rejected(lib):
    assert lib.fp8bw_quantize_rowwise(None, 128, 128, B, C, None) == E_NULL
    assert lib.fp8bw_quantize_colwise(A, 128, 128, None, C, None, None,
                                      None) == E_NULL
    # q_row without s_row
    assert lib.fp8bw_quantize_colwise(A, 128, 128, B, C, D, None,
                                      None) == E_NULL
    assert lib.fp8bw_quantize_weight_block(A, 128, 128, None, C, None,
                                           None) == E_NULL
    assert lib.fp8bw_gemm_fprop(A, B, C, None, 128, 128, 128, E,
                                None) == E_NULL
    assert lib.fp8bw_gemm_dgrad(A, B, None, 1, D, 128, 128, 128, E,
                                None) == E_NULL
    assert lib.fp8bw_gemm_wgrad(A, B, C, D, 128, 128, 128, None,
                                None) == E_NULL
    assert lib.fp8bw_gemm_wgrad_f32(A, B, C, D, 128, 128, 128, None, 1,
                                    None) == E_NULL
    assert lib.fp8bw_quantize_rowwise_pow2(None, 128, 128, B, C, None) == E_NULL
    assert lib.fp8bw_gemm_fprop_pow2(A, B, C, None, 128, 128, 128, E,
                                     None) == E_NULL
    assert lib.fp8bw_gemm_wgrad_pow2(A, B, C, D, 128, 128, 128, None,
                                     None) == E_NULL
    # the fused quantisation outputs are required
    assert lib.fp8bw_gemm_fprop_quant(A, B, C, D, 128, 128, 128, E, None,
                                      E + 0x100000, None) == E_NULL
    assert lib.fp8bw_gemm_dgrad_quant(A, B, C, 1, D, 128, 128, 128, E,
                                      E + 0x100000, None, None) == E_NULL


def test_tile_count_limit(lib):
    rows, cols = 65535 * 128, 1 << 30          # 65535 * 2^23 tiles of 128x128
    assert lib.fp8bw_quantize_rowwise(A, rows, cols, B, C, None) == E_SHAPE
    assert lib.fp8bw_quantize_colwise(A, rows, cols, B, C, None, None,
                                      None) == E_SHAPE
    assert lib.fp8bw_quantize_weight_block(A, rows, cols, B, C, None,
                                           None) == E_SHAPE


def test_selftest_limit_checked(lib):
    assert lib.fp8bw_selftest_wait_timeout(-1, None) == E_SHAPE
    assert lib.fp8bw_selftest_wait_timeout(2 * 10**9, None) == E_SHAPE


@pytest.mark.parametrize("rows,cols", [(-16, 128), (128, -16), (100, 128),
                                       (128, 8), (128, 130), (1 << 31, 16)])
def test_bad_shapes_rejected(lib, rows, cols):
    assert lib.fp8bw_quantize_rowwise(A, rows, cols, B, C, None) == E_SHAPE
    assert lib.fp8bw_quantize_colwise(A, rows, cols, B, C, None, None,
                                      None) == E_SHAPE
    assert lib.fp8bw_quantize_weight_block(A, rows, cols, B, C, None,
                                           None) == E_SHAPE
    assert lib.fp8bw_gemm_fprop(A, B, C, D, rows, cols, 128, E,
                                None) == E_SHAPE
    assert lib.fp8bw_gemm_dgrad(A, B, C, 0, D, 128, rows, cols, E,
                                None) == E_SHAPE
    assert lib.fp8bw_gemm_wgrad(A, B, C, D, cols, 128, rows, E,
                                None) == E_SHAPE
    assert lib.fp8bw_gemm_wgrad_f32(A, B, C, D, cols, 128, rows, E, 0,
                                    None) == E_SHAPE
    assert lib.fp8bw_quantize_colwise_pow2(A, rows, cols, B, C, None, None,
                                           None) == E_SHAPE
    assert lib.fp8bw_gemm_dgrad_pow2(A, B, C, 1, D, 128, rows, cols, E,
                                     None) == E_SHAPE


def test_misaligned_pointers_rejected(lib):
    assert lib.fp8bw_quantize_rowwise(A + 2, 128, 128, B, C, None) == E_ALIGN
    assert lib.fp8bw_quantize_colwise(A, 128, 128, B, C + 4, None, None,
                                      None) == E_ALIGN
    assert lib.fp8bw_quantize_weight_block(A, 128, 128, B, C, D + 8,
                                           None) == E_ALIGN
    assert lib.fp8bw_gemm_fprop(A, B + 1, C, D, 128, 128, 128, E,
                                None) == E_ALIGN
    assert lib.fp8bw_gemm_dgrad(A, B, C, 1, D, 128, 128, 128, E + 2,
                                None) == E_ALIGN
    assert lib.fp8bw_gemm_wgrad(A, B, C, D + 4, 128, 128, 128, E,
                                None) == E_ALIGN
    assert lib.fp8bw_gemm_wgrad_f32(A, B, C, D, 128, 128, 128, E + 8, 1,
                                    None) == E_ALIGN
    assert lib.fp8bw_quantize_weight_block_pow2(A, 128, 128, B, C, D + 8,
                                                None) == E_ALIGN
    assert lib.fp8bw_gemm_fprop_quant(A, B, C, D, 128, 128, 128, E,
                                      E + 0x100008, E + 0x200000,
                                      None) == E_ALIGN


def test_aliased_outputs_rejected(lib):
    # output codes overlapping the bf16 input
    assert lib.fp8bw_quantize_rowwise(A, 128, 128, A + 16, C, None) == E_ALIAS
    # GEMM output on top of the scales
    assert lib.fp8bw_gemm_fprop(A, B, C, D, 128, 128, 128, B,
                                None) == E_ALIAS
    assert lib.fp8bw_gemm_wgrad(A, B, C, D, 128, 128, 128, C + 256,
                                None) == E_ALIAS
    # fused quantisation: codes on top of the bf16 output
    assert lib.fp8bw_gemm_fprop_quant(A, B, C, D, 128, 128, 128, E, E + 64,
                                      E + 0x100000, None) == E_ALIAS
    # the fp32 dW is 4 bytes per element: [C - 128*128*4 + 16, C + 16)
    # reaches into qX^T at C
    assert lib.fp8bw_gemm_wgrad_f32(A, B, C, D, 128, 128, 128,
                                    C - 128 * 128 * 4 + 16, 1,
                                    None) == E_ALIAS


def _jobs(*specs):
    arr = (_native.WeightBlockJob * max(1, len(specs)))()
    for i, sp in enumerate(specs):
        arr[i] = _native.WeightBlockJob(*sp)
    return ctypes.cast(arr, ctypes.c_void_p), arr


def test_weight_block_batch_checks(lib):
    ok1 = (A, 256, 128, B, C, D)                  # w, n, k, q, s, q_t
    ok2 = (A + 0x100000, 128, 256, B + 0x100000, C + 0x100000, None)
    p, keep = _jobs(ok1, ok2)
    assert lib.fp8bw_quantize_weight_block_batch(p, 9, None) == E_SHAPE
    assert lib.fp8bw_quantize_weight_block_batch(p, -1, None) == E_SHAPE
    assert lib.fp8bw_quantize_weight_block_batch(None, 2, None) == E_NULL
    p, keep = _jobs(ok1, (A + 0x100000, 100, 256, B + 0x100000, C + 0x100000, None))
    assert lib.fp8bw_quantize_weight_block_batch(p, 2, None) == E_SHAPE
    p, keep = _jobs(ok1, (A + 0x100000, 128, 256, B + 0x100008, C + 0x100000, None))
    assert lib.fp8bw_quantize_weight_block_batch_pow2(p, 2, None) == E_ALIGN
    # job 2's codes on top of job 1's input, and two jobs sharing a scale buffer
    p, keep = _jobs(ok1, (A + 0x100000, 128, 256, A + 256, C + 0x100000, None))
    assert lib.fp8bw_quantize_weight_block_batch(p, 2, None) == E_ALIAS
    p, keep = _jobs(ok1, (A + 0x100000, 128, 256, B + 0x100000, C, None))
    assert lib.fp8bw_quantize_weight_block_batch(p, 2, None) == E_ALIAS


def _wjobs(*specs):
    arr = (_native.WgradJob * max(1, len(specs)))()
    for i, sp in enumerate(specs):
        arr[i] = _native.WgradJob(*sp)
    return ctypes.cast(arr, ctypes.c_void_p), arr


def test_wgrad_batch_checks(lib):
    M = 0x1000000
    # qdy_t, sdy_t, qx_t, sx_t, m, n, k, dw
    ok1 = (A, B, C, D, 256, 128, 256, E)
    ok2 = (A + M, B + M, C + M, D + M, 256, 256, 128, E + M)
    p, keep = _wjobs(ok1, ok2)
    for fn in (lib.fp8bw_gemm_wgrad_batch, lib.fp8bw_gemm_wgrad_batch_pow2):
        assert fn(p, 5, None) == E_SHAPE
        assert fn(p, -1, None) == E_SHAPE
        assert fn(None, 2, None) == E_NULL
    assert lib.fp8bw_gemm_wgrad_f32_batch(p, 5, 1, None) == E_SHAPE
    assert lib.fp8bw_gemm_wgrad_f32_batch_pow2(None, 1, 0, None) == E_NULL
    # different token counts
    p, keep = _wjobs(ok1, ok2[:4] + (384,) + ok2[5:])
    assert lib.fp8bw_gemm_wgrad_batch(p, 2, None) == E_SHAPE
    # a job's own checks: ragged size, null operand, misaligned dW
    p, keep = _wjobs(ok1, ok2[:5] + (100,) + ok2[6:])
    assert lib.fp8bw_gemm_wgrad_batch(p, 2, None) == E_SHAPE
    p, keep = _wjobs(ok1, (None,) + ok2[1:])
    assert lib.fp8bw_gemm_wgrad_f32_batch(p, 2, 0, None) == E_NULL
    p, keep = _wjobs(ok1, ok2[:7] + (E + M + 8,))
    assert lib.fp8bw_gemm_wgrad_batch(p, 2, None) == E_ALIGN
    # job 2's dW on top of job 1's operand, and two jobs sharing a dW
    p, keep = _wjobs(ok1, ok2[:7] + (C + 64,))
    assert lib.fp8bw_gemm_wgrad_batch(p, 2, None) == E_ALIAS
    p, keep = _wjobs(ok1, ok2[:7] + (E + 1024,))
    assert lib.fp8bw_gemm_wgrad_f32_batch(p, 2, 1, None) == E_ALIAS


@pytest.mark.skipif(
    __import__("torch").cuda.is_available(),
    reason="checks the no-device path; on a GPU host the call would launch")
def test_valid_call_without_device_reports_device_error(lib):
    p, keep = _wjobs((A, B, C, D, 256, 128, 256, E))
    assert lib.fp8bw_gemm_wgrad_batch(p, 1, None) == E_DEVICE
    p, keep = _jobs((A, 256, 128, B, C, D))
    assert lib.fp8bw_quantize_weight_block_batch(p, 1, None) == E_DEVICE
    assert lib.fp8bw_quantize_rowwise(A, 128, 128, B, C, None) == E_DEVICE
    assert lib.fp8bw_gemm_fprop(A, B, C, D, 128, 128, 128, E,
                                None) == E_DEVICE
    assert lib.fp8bw_gemm_wgrad_f32(A, B, C, D, 128, 128, 128, E, 1,
                                    None) == E_DEVICE


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "fp8bw.h"

typedef int (*gemm_fn)(const uint8_t*, const float*, const uint8_t*,
                       const float*, int64_t, int64_t, int64_t, uint16_t*,
                       void*);

int main(void) {
    gemm_fn f = fp8bw_gemm_fprop;
    uint8_t code = 0;
    float scale = 1.0f;
    uint16_t out = 0;
    /* no device needed: the null operand is rejected on the host */
    int st = f(NULL, &scale, &code, &scale, 128, 128, 128, &out, NULL);
    printf("%d %d %s|%s\n", fp8bw_version(), st, fp8bw_status_string(st),
           fp8bw_status_string(FP8BW_OK));
    return (st == FP8BW_ERR_NULL && out == 0) ? 0 : 1;
}
"""


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c11"),
                                          ("g++", "-std=c++17")])
def test_header_builds_a_plain_client(lib, tmp_path, compiler, std):
    """include/fp8bw.h is self-contained C: a C11 (and a C++17) program that
    includes it builds with -pedantic -Werror, links against libfp8bw.so and
    gets the host-side answers (version, status strings, a rejected call)."""
    import shutil
    import subprocess
    if shutil.which(compiler) is None:
        pytest.skip(compiler + " not available")
    src = tmp_path / ("client.c" if compiler == "gcc" else "client.cpp")
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(_native.LIB_PATH)
    cmd = [compiler, std, "-Wall", "-Wextra", "-pedantic", "-Werror",
           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
           "-L", libdir, "-l:" + os.path.basename(_native.LIB_PATH),
           "-Wl,-rpath," + libdir]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    run = subprocess.run([str(exe)], capture_output=True, text=True,
                         timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    version, status, rest = run.stdout.strip().split(" ", 2)
    assert int(version) == lib.fp8bw_version() and int(status) == E_NULL
    null_msg, ok_msg = rest.split("|")
    assert null_msg == lib.fp8bw_status_string(E_NULL).decode()
    assert ok_msg == lib.fp8bw_status_string(OK).decode()


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No CPU fallback: without libfp8bw.so (and nothing to build it from) the
    loader raises instead of returning anything callable."""
    from blockwise_fp8_linear_fp8bw_b200 import build as _build
    monkeypatch.setattr(_native, "_lib", None)
    monkeypatch.setattr(_native, "LIB_PATH", str(tmp_path / "libfp8bw.so"))
    monkeypatch.setattr(_build, "needs_build", lambda: False)
    with pytest.raises(ImportError, match="missing"):
        _native.load()


def test_binding_refuses_cpu_tensors(lib):
    """No CPU fallback in the binding either: CPU tensors are refused before
    the library is reached, and nothing is computed."""
    import torch
    from blockwise_fp8_linear_fp8bw_b200 import ops
    x = torch.zeros((128, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        ops.quantize_rowwise(x)
