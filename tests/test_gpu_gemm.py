"""GPU parity of the three blockwise GEMMs (paperlayer.ai summary of the
Puro-2B report, Appendix C, "FP8 implementation pipeline": forward
propagation, data-gradient and weight-gradient), through the C ABI.

Each output element must satisfy |y - ref| <= 1e-3 * sum_k |a_k b_k| + 1 bf16
ulp(ref), where ref is the oracle's fp64 value and the sum runs over the
dequantised operands. Small cases and the 8192 x 4096 x 2048 fprop compare
every element; the larger full-size cases compare >= 16 seeded points per
128x128 output tile plus two full rows and two full columns, in the launch
configuration the benchmark uses."""
import numpy as np
import pytest

import oracle
import synthetic as S
from helpers import (assert_gemm_close, bf16_np_to_torch, sample_points,
                     torch_bf16_to_np)

pytestmark = pytest.mark.gpu


def _ops():
    from blockwise_fp8_linear_fp8bw_b200 import ops
    return ops


def _fprop_case(m, n, k, seed_id, xdist=S.X_DIST, full=True):
    ops = _ops()
    x = S.bf16_normal((m, k), 0, seed_id, **xdist)
    w = S.bf16_normal((n, k), 0, seed_id + 1, **S.W_DIST)
    qx, sx = ops.quantize_rowwise(bf16_np_to_torch(x))
    qw, sw, _ = ops.quantize_weight_block(bf16_np_to_torch(w),
                                          transposed=False)
    y = torch_bf16_to_np(ops.gemm_fprop(qx, sx, qw, sw))
    rqx, rsx = oracle.quantize_rowwise(x)
    rqw, rsw, _ = oracle.quantize_weight_block(w, want_transposed=False)
    if full:
        acc, bound = oracle.gemm_fprop(rqx, rsx, rqw, rsw, with_bound=True)
        assert_gemm_close(y, acc, bound, "fprop %dx%dx%d" % (m, n, k))
    else:
        pi, pj = sample_points(m, n)
        acc, bound = oracle.gemm_fprop_points(rqx, rsx, rqw, rsw, pi, pj)
        assert_gemm_close(y[pi, pj], acc, bound, "fprop %dx%dx%d" % (m, n, k))


def _dgrad_case(m, n, k, seed_id, transposed, full=True):
    ops = _ops()
    dy = S.bf16_normal((m, n), 0, seed_id, **S.DY_DIST)
    w = S.bf16_normal((n, k), 0, seed_id + 1, **S.W_DIST)
    qdy, sdy = ops.quantize_rowwise(bf16_np_to_torch(dy))
    qw, sw, qw_t = ops.quantize_weight_block(bf16_np_to_torch(w),
                                             transposed=True)
    dx = ops.gemm_dgrad(qdy, sdy, qw_t if transposed else qw, sw,
                        qw_is_transposed=transposed)
    dx = torch_bf16_to_np(dx)
    rq, rs = oracle.quantize_rowwise(dy)
    rqw, rsw, _ = oracle.quantize_weight_block(w, want_transposed=False)
    if full:
        acc, bound = oracle.gemm_dgrad(rq, rs, rqw, rsw, with_bound=True)
        assert_gemm_close(dx, acc, bound, "dgrad %dx%dx%d" % (m, n, k))
    else:
        pi, pj = sample_points(m, k)
        acc, bound = oracle.gemm_dgrad_points(rq, rs, rqw, rsw, pi, pj)
        assert_gemm_close(dx[pi, pj], acc, bound, "dgrad %dx%dx%d" % (m, n, k))


def _wgrad_case(m, n, k, seed_id, full=True):
    ops = _ops()
    dy = S.bf16_normal((m, n), 0, seed_id, **S.DY_DIST)
    x = S.bf16_normal((m, k), 0, seed_id + 1, **S.X_DIST)
    qdy_t, sdy_t = ops.quantize_colwise(bf16_np_to_torch(dy))
    qx_t, sx_t = ops.quantize_colwise(bf16_np_to_torch(x))
    dw = torch_bf16_to_np(ops.gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t))
    rq, rs = oracle.quantize_colwise(dy)
    rqx, rsx = oracle.quantize_colwise(x)
    if full:
        acc, bound = oracle.gemm_wgrad(rq, rs, rqx, rsx, with_bound=True)
        assert_gemm_close(dw, acc, bound, "wgrad %dx%dx%d" % (m, n, k))
    else:
        pi, pj = sample_points(n, k)
        acc, bound = oracle.gemm_wgrad_points(rq, rs, rqx, rsx, pi, pj)
        assert_gemm_close(dw[pi, pj], acc, bound, "wgrad %dx%dx%d" % (m, n, k))


SMALL = [(256, 256, 256), (128, 128, 128), (272, 400, 528), (512, 768, 384),
         (16, 16, 16), (1040, 272, 144), (384, 1296, 640)]


@pytest.mark.parametrize("m,n,k", SMALL)
def test_fprop_small_and_ragged(m, n, k):
    _fprop_case(m, n, k, 601)


def test_fprop_256_no_outliers():
    # the single-GEMM 256x256x256 workload: X ~ N(0,1) without outliers
    _fprop_case(256, 256, 256, 1, xdist=S.X_DIST_PLAIN)


@pytest.mark.parametrize("m,n,k", SMALL)
@pytest.mark.parametrize("transposed", [True, False])
def test_dgrad_small_and_ragged(m, n, k, transposed):
    _dgrad_case(m, n, k, 611, transposed)


@pytest.mark.parametrize("m,n,k", SMALL)
def test_wgrad_small_and_ragged(m, n, k):
    _wgrad_case(m, n, k, 621)


def test_empty_contraction_writes_zeros():
    import torch
    ops = _ops()
    qx = torch.empty((128, 0), dtype=torch.uint8, device="cuda")
    sx = torch.empty((0, 128), dtype=torch.float32, device="cuda")
    qw = torch.empty((256, 0), dtype=torch.uint8, device="cuda")
    sw = torch.empty((2, 0), dtype=torch.float32, device="cuda")
    y = torch.full((128, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    ops.fp8bw_gemm_fprop(qx, sx, qw, sw, y)
    assert torch.count_nonzero(y).item() == 0


def test_full_size_qkv_fprop_every_element():
    _fprop_case(8192, 4096, 2048, S.tensor_id("qkv", "x"), full=True)


def test_full_size_mlp_fprop():
    _fprop_case(16384, 12288, 2048, S.tensor_id("gate_up", "x"), full=False)
    _fprop_case(16384, 2048, 6144, S.tensor_id("down", "x"), full=False)


def test_full_size_mlp_backward():
    _dgrad_case(16384, 2048, 6144, S.tensor_id("down", "dy"), True,
                full=False)
    _wgrad_case(16384, 2048, 6144, S.tensor_id("down", "dy"), full=False)
    _dgrad_case(16384, 12288, 2048, S.tensor_id("gate_up", "dy"), True,
                full=False)
    _wgrad_case(16384, 12288, 2048, S.tensor_id("gate_up", "dy"), full=False)
    _ops().fp8bw_check_device_error()


@pytest.mark.parametrize("kind", ["qkv", "o"])
def test_full_size_attention_linears(kind):
    """The QKV and O linears of the 28-layer stack at M = 16384 (the MLP
    linears are covered above): fprop, dgrad on transposed weight codes and
    wgrad, each on its own draws."""
    k, n = S.LINEARS[kind]
    _fprop_case(16384, n, k, S.tensor_id(kind, "x", 0), full=False)
    _dgrad_case(16384, n, k, S.tensor_id(kind, "dy", 0), True, full=False)
    _wgrad_case(16384, n, k, S.tensor_id(kind, "dy", 0), full=False)
    _ops().fp8bw_check_device_error()


@pytest.mark.parametrize("m,n,k", [(272, 400, 528), (16384, 2048, 2048)])
def test_wgrad_repeatable(m, n, k):
    """Repeated weight-gradient calls on the same operands give the same
    bits (no order-dependent accumulation anywhere in the kernel)."""
    import torch
    ops = _ops()
    dy = S.bf16_normal((m, n), 0, 641, **S.DY_DIST)
    x = S.bf16_normal((m, k), 0, 642, **S.X_DIST)
    qdy_t, sdy_t = ops.quantize_colwise(bf16_np_to_torch(dy))
    qx_t, sx_t = ops.quantize_colwise(bf16_np_to_torch(x))
    first = ops.gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t)
    for _ in range(3):
        again = ops.gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t)
        assert torch.equal(again.view(torch.int16), first.view(torch.int16))
    ops.fp8bw_check_device_error()
