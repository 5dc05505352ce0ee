"""GPU parity of the power-of-two-scale path: quantisers with s = 2^E (E the
smallest integer with 448 * 2^E >= amax) bit-exact against the oracle's
power-of-two mode, and the GEMMs on the tensor cores' UE8M0 block scaling
within the GEMM tolerance of the oracle (the pages leave the scale form open:
Puro-2B arxiv-wiki summary, Approach item (4) and developer notes, bullet 3).
Tolerance as for the other GEMMs: |y - ref| <= 1e-3 * sum_k |a_k b_k| + 1 bf16
ulp(ref)."""
import numpy as np
import pytest

import oracle
import synthetic as S
from helpers import (assert_gemm_close, bf16_np_to_torch, sample_points,
                     scale_bits, torch_bf16_to_np)

pytestmark = pytest.mark.gpu

SMALL = [(256, 256, 256), (128, 128, 128), (272, 400, 528), (512, 768, 384),
         (16, 16, 16), (1040, 272, 144), (384, 1296, 640)]


def _ops():
    from blockwise_fp8_linear_fp8bw_b200 import ops
    return ops


def _np(t):
    return t.cpu().numpy()


@pytest.mark.parametrize("rows,cols", [(256, 256), (272, 400), (16, 2064),
                                       (1040, 48), (8192, 2048)])
def test_pow2_quantisers_bit_exact(rows, cols):
    ops = _ops()
    x = S.bf16_normal((rows, cols), 0, 701, **S.X_DIST)
    xt = bf16_np_to_torch(x)
    q_t, s_t, q, s = ops.quantize_colwise(xt, with_rowwise=True, pow2=True)
    rq, rs = oracle.quantize_rowwise(x, pow2=True)
    rq_t, rs_t = oracle.quantize_colwise(x, pow2=True)
    assert np.array_equal(_np(q), rq) and np.array_equal(_np(q_t), rq_t)
    assert np.array_equal(scale_bits(_np(s)), scale_bits(rs))
    assert np.array_equal(scale_bits(_np(s_t)), scale_bits(rs_t))
    q2, s2 = ops.quantize_rowwise(xt, pow2=True)
    assert np.array_equal(_np(q2), rq) and np.array_equal(scale_bits(_np(s2)), scale_bits(rs))
    w = S.bf16_normal((rows, cols), 0, 702, **S.W_DIST)
    qw, sw, qw_t = ops.quantize_weight_block(bf16_np_to_torch(w), pow2=True)
    rqw, rsw, rqw_t = oracle.quantize_weight_block(w, pow2=True)
    assert np.array_equal(_np(qw), rqw) and np.array_equal(_np(qw_t), rqw_t)
    assert np.array_equal(scale_bits(_np(sw)), scale_bits(rsw))


def test_pow2_special_groups():
    ops = _ops()
    g = np.zeros((128, 256), np.float32)
    g[0, :128] = 0.0                       # all-zero group -> s = 1
    g[1, :] = 448.0                        # E = 0
    g[2, 0] = 450.0                        # E = 1
    g[3, 0] = 2.0 ** -133                  # clamps at E = -127
    g[4, 5] = -3.0
    x = (g.view(np.uint32) >> 16).astype(np.uint16)
    q, s = ops.quantize_rowwise(bf16_np_to_torch(x), pow2=True)
    rq, rs = oracle.quantize_rowwise(x, pow2=True)
    assert np.array_equal(_np(q), rq)
    assert np.array_equal(scale_bits(_np(s)), scale_bits(rs))


def _fprop(m, n, k, seed, full=True):
    ops = _ops()
    x = S.bf16_normal((m, k), 0, seed, **S.X_DIST)
    w = S.bf16_normal((n, k), 0, seed + 1, **S.W_DIST)
    qx, sx = ops.quantize_rowwise(bf16_np_to_torch(x), pow2=True)
    qw, sw, _ = ops.quantize_weight_block(bf16_np_to_torch(w), transposed=False, pow2=True)
    y = torch_bf16_to_np(ops.gemm_fprop(qx, sx, qw, sw, pow2=True))
    ops.fp8bw_check_device_error()
    rqx, rsx = oracle.quantize_rowwise(x, pow2=True)
    rqw, rsw, _ = oracle.quantize_weight_block(w, want_transposed=False, pow2=True)
    if full:
        acc, bound = oracle.gemm_fprop(rqx, rsx, rqw, rsw, with_bound=True)
        assert_gemm_close(y, acc, bound, "pow2 fprop %dx%dx%d" % (m, n, k))
    else:
        pi, pj = sample_points(m, n)
        acc, bound = oracle.gemm_fprop_points(rqx, rsx, rqw, rsw, pi, pj)
        assert_gemm_close(y[pi, pj], acc, bound, "pow2 fprop %dx%dx%d" % (m, n, k))


def _dgrad(m, n, k, seed, transposed, full=True):
    ops = _ops()
    dy = S.bf16_normal((m, n), 0, seed, **S.DY_DIST)
    w = S.bf16_normal((n, k), 0, seed + 1, **S.W_DIST)
    qdy, sdy = ops.quantize_rowwise(bf16_np_to_torch(dy), pow2=True)
    qw, sw, qw_t = ops.quantize_weight_block(bf16_np_to_torch(w), pow2=True)
    dx = torch_bf16_to_np(ops.gemm_dgrad(qdy, sdy, qw_t if transposed else qw, sw,
                                         qw_is_transposed=transposed, pow2=True))
    ops.fp8bw_check_device_error()
    rq, rs = oracle.quantize_rowwise(dy, pow2=True)
    rqw, rsw, _ = oracle.quantize_weight_block(w, want_transposed=False, pow2=True)
    if full:
        acc, bound = oracle.gemm_dgrad(rq, rs, rqw, rsw, with_bound=True)
        assert_gemm_close(dx, acc, bound, "pow2 dgrad %dx%dx%d" % (m, n, k))
    else:
        pi, pj = sample_points(m, k)
        acc, bound = oracle.gemm_dgrad_points(rq, rs, rqw, rsw, pi, pj)
        assert_gemm_close(dx[pi, pj], acc, bound, "pow2 dgrad %dx%dx%d" % (m, n, k))


def _wgrad(m, n, k, seed, full=True):
    ops = _ops()
    dy = S.bf16_normal((m, n), 0, seed, **S.DY_DIST)
    x = S.bf16_normal((m, k), 0, seed + 1, **S.X_DIST)
    qdy_t, sdy_t = ops.quantize_colwise(bf16_np_to_torch(dy), pow2=True)
    qx_t, sx_t = ops.quantize_colwise(bf16_np_to_torch(x), pow2=True)
    dw = torch_bf16_to_np(ops.gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t, pow2=True))
    ops.fp8bw_check_device_error()
    rq, rs = oracle.quantize_colwise(dy, pow2=True)
    rqx, rsx = oracle.quantize_colwise(x, pow2=True)
    if full:
        acc, bound = oracle.gemm_wgrad(rq, rs, rqx, rsx, with_bound=True)
        assert_gemm_close(dw, acc, bound, "pow2 wgrad %dx%dx%d" % (m, n, k))
    else:
        pi, pj = sample_points(n, k)
        acc, bound = oracle.gemm_wgrad_points(rq, rs, rqx, rsx, pi, pj)
        assert_gemm_close(dw[pi, pj], acc, bound, "pow2 wgrad %dx%dx%d" % (m, n, k))


@pytest.mark.parametrize("m,n,k", SMALL)
def test_pow2_fprop_small_and_ragged(m, n, k):
    _fprop(m, n, k, 711)


@pytest.mark.parametrize("m,n,k", SMALL)
@pytest.mark.parametrize("transposed", [True, False])
def test_pow2_dgrad_small_and_ragged(m, n, k, transposed):
    _dgrad(m, n, k, 721, transposed)


@pytest.mark.parametrize("m,n,k", SMALL)
def test_pow2_wgrad_small_and_ragged(m, n, k):
    _wgrad(m, n, k, 731)


def test_pow2_full_size_linears():
    _fprop(16384, 12288, 2048, S.tensor_id("gate_up", "x"), full=False)
    _dgrad(16384, 2048, 6144, S.tensor_id("down", "dy"), True, full=False)
    _wgrad(16384, 2048, 6144, S.tensor_id("down", "dy"), full=False)
    _wgrad(16384, 12288, 2048, S.tensor_id("gate_up", "dy"), full=False)


def test_pow2_gemm_rejects_other_scales():
    ops = _ops()
    x = S.bf16_normal((256, 256), 0, 741, **S.X_DIST)
    w = S.bf16_normal((256, 256), 0, 742, **S.W_DIST)
    qx, sx = ops.quantize_rowwise(bf16_np_to_torch(x))          # amax/448 scales
    qw, sw, _ = ops.quantize_weight_block(bf16_np_to_torch(w), transposed=False)
    ops.fp8bw_check_device_error()
    ops.gemm_fprop(qx, sx, qw, sw, pow2=True)
    with pytest.raises(ops.Fp8bwError) as e:
        ops.fp8bw_check_device_error()
    assert e.value.status == ops.FP8BW_ERR_SCALE
    ops.fp8bw_check_device_error()                              # record cleared
