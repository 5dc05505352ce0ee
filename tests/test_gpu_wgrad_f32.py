"""GPU parity of the weight-gradient GEMM with an fp32 result, stored or
added into an fp32 main-grad buffer (paperlayer.ai summary of the Puro-2B
report, Appendix C, "FP8 implementation pipeline": gradients stay in FP32),
for both scale forms (amax/448 scales with per-chunk promotion, and the
power-of-two scales applied by the tensor cores).

Checks, through the C ABI:
  * against the oracle: |dW - ref| <= 1e-3 * sum_k |a_k b_k| + 1 fp32 ulp,
    with ref the oracle's fp64 value (plus the old main-grad when adding);
  * that the fp32 result is the value the bf16 entry point rounds: bf16 RN of
    every fp32 element equals the bf16 wgrad output bit for bit;
  * that accumulation is one fp32 add per element: dW_after equals
    fp32(dW_before + P) bit for bit, P being the stored fp32 result (a
    subnormal sum may be flushed to zero by the add).
"""
import numpy as np
import pytest

import oracle
import synthetic as S
from helpers import (assert_gemm_close_f32, bf16_np_to_torch, sample_points)

pytestmark = pytest.mark.gpu

F32_TINY = np.float32(2.0 ** -126)


def _ops():
    from blockwise_fp8_linear_fp8bw_b200 import ops
    return ops


def _main_grad(n, k, seed_id):
    # an fp32 main-grad of the same magnitude as one micro-batch's dW
    g = S.bf16_normal((n, k), 0, seed_id, std=0.05)
    return (g.astype(np.uint32) << 16).view(np.float32) + np.float32(1e-5)


def _assert_add_exact(after, before, p, what):
    want = (before.astype(np.float32) + p.astype(np.float32)).astype(np.float32)
    same = after.view(np.uint32) == want.view(np.uint32)
    flushed = (np.abs(want) < F32_TINY) & (np.abs(after) < F32_TINY)
    bad = ~(same | flushed)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError("%s: %d elements differ from fp32(old + P); "
                             "first %s" % (what, int(bad.sum()),
                                           idx.tolist()))


def _wgrad_f32_case(m, n, k, seed_id, full=True, pow2=False):
    import torch
    ops = _ops()
    dy = S.bf16_normal((m, n), 0, seed_id, **S.DY_DIST)
    x = S.bf16_normal((m, k), 0, seed_id + 1, **S.X_DIST)
    qdy_t, sdy_t = ops.quantize_colwise(bf16_np_to_torch(dy), pow2=pow2)
    qx_t, sx_t = ops.quantize_colwise(bf16_np_to_torch(x), pow2=pow2)
    what = "wgrad_f32%s %dx%dx%d" % ("_pow2" if pow2 else "", m, n, k)

    p_dev = ops.gemm_wgrad_f32(qdy_t, sdy_t, qx_t, sx_t, pow2=pow2)
    dw_bf16 = ops.gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t, pow2=pow2)
    assert torch.equal(p_dev.to(torch.bfloat16).view(torch.int16),
                       dw_bf16.view(torch.int16)), what + ": bf16(fp32) != bf16"

    before = _main_grad(n, k, seed_id + 2)
    g_dev = torch.from_numpy(before.copy()).cuda()
    ops.gemm_wgrad_f32(qdy_t, sdy_t, qx_t, sx_t, main_grad=g_dev, pow2=pow2)
    # a second call adds the same product again
    after1 = g_dev.cpu().numpy()
    ops.gemm_wgrad_f32(qdy_t, sdy_t, qx_t, sx_t, main_grad=g_dev, pow2=pow2)
    after2 = g_dev.cpu().numpy()
    ops.fp8bw_check_device_error()
    p = p_dev.cpu().numpy()
    _assert_add_exact(after1, before, p, what + " add #1")
    _assert_add_exact(after2, after1, p, what + " add #2")

    rq, rs = oracle.quantize_colwise(dy, pow2=pow2)
    rqx, rsx = oracle.quantize_colwise(x, pow2=pow2)
    if full:
        acc, bound = oracle.gemm_wgrad(rq, rs, rqx, rsx, with_bound=True)
        assert_gemm_close_f32(p, acc, bound, what)
        assert_gemm_close_f32(after1, before.astype(np.float64) + acc, bound,
                              what + " accumulate")
    else:
        pi, pj = sample_points(n, k)
        acc, bound = oracle.gemm_wgrad_points(rq, rs, rqx, rsx, pi, pj)
        assert_gemm_close_f32(p[pi, pj], acc, bound, what)
        b = before[pi, pj].astype(np.float64)
        assert_gemm_close_f32(after1[pi, pj], b + acc, bound,
                              what + " accumulate")


SMALL = [(256, 256, 256), (128, 128, 128), (272, 400, 528), (512, 768, 384),
         (16, 16, 16), (1040, 272, 144), (384, 1296, 640)]


@pytest.mark.parametrize("pow2", [False, True])
@pytest.mark.parametrize("m,n,k", SMALL)
def test_wgrad_f32_small_and_ragged(m, n, k, pow2):
    _wgrad_f32_case(m, n, k, 631, pow2=pow2)


@pytest.mark.parametrize("pow2", [False, True])
def test_wgrad_f32_empty_contraction(pow2):
    import torch
    ops = _ops()
    q = torch.empty((256, 0), dtype=torch.uint8, device="cuda")
    s = torch.empty((0, 256), dtype=torch.float32, device="cuda")
    dw = torch.full((256, 256), 7.0, dtype=torch.float32, device="cuda")
    ops.fp8bw_gemm_wgrad_f32(q, s, q, s, dw, accumulate=True, pow2=pow2)
    assert bool((dw == 7.0).all())
    ops.fp8bw_gemm_wgrad_f32(q, s, q, s, dw, accumulate=False, pow2=pow2)
    assert torch.count_nonzero(dw).item() == 0


@pytest.mark.parametrize("pow2", [False, True])
def test_wgrad_f32_full_size_mlp(pow2):
    _wgrad_f32_case(16384, 2048, 6144, S.tensor_id("down", "dy"), full=False,
                    pow2=pow2)
    _wgrad_f32_case(16384, 12288, 2048, S.tensor_id("gate_up", "dy"),
                    full=False, pow2=pow2)
