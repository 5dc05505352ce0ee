"""Maximum sizes: tensors past 2^31 elements (64-bit offsets everywhere) and a
contraction over 2^20 tokens (8192 chunks), checked against the oracle on
sampled rows, column blocks and output points. Inputs are drawn on the GPU
(torch, seeded) and the sampled parts copied back for the oracle."""
import numpy as np
import pytest

import oracle
from helpers import assert_gemm_close, sample_points, scale_bits, torch_bf16_to_np

pytestmark = pytest.mark.gpu


def _ops():
    from blockwise_fp8_linear_fp8bw_b200 import ops
    return ops


def _bf16(shape, std, seed):
    import torch
    g = torch.Generator(device="cuda").manual_seed(seed)
    return (torch.randn(shape, generator=g, device="cuda") * std).to(torch.bfloat16)


def test_quantiser_past_2_31_elements():
    import torch
    ops = _ops()
    rows, cols = 65536, 33024                  # 2.16e9 elements
    x = _bf16((rows, cols), 1.0, 11)
    q_t, s_t, q, s = ops.quantize_colwise(x, with_rowwise=True)
    ops.fp8bw_check_device_error()
    for r in (0, 12345, 40000, rows - 1):
        xr = torch_bf16_to_np(x[r:r + 1])
        rq, rs = oracle.quantize_rowwise(xr)
        assert np.array_equal(q[r:r + 1].cpu().numpy(), rq), r
        assert np.array_equal(scale_bits(s[:, r:r + 1].cpu().numpy()), scale_bits(rs)), r
    for c0 in (0, 16400, cols - 16):
        xc = torch_bf16_to_np(x[:, c0:c0 + 16])
        rq_t, rs_t = oracle.quantize_colwise(xc)
        assert np.array_equal(q_t[c0:c0 + 16].cpu().numpy(), rq_t), c0
        assert np.array_equal(scale_bits(s_t[:, c0:c0 + 16].cpu().numpy()), scale_bits(rs_t)), c0
    del x, q_t, s_t, q, s
    torch.cuda.empty_cache()


def test_fprop_output_past_2_31_elements():
    import torch
    ops = _ops()
    m, n, k = 65536, 33024, 256                # y has 2.16e9 elements
    x = _bf16((m, k), 1.0, 12)
    w = _bf16((n, k), 0.02, 13)
    qx, sx = ops.quantize_rowwise(x)
    qw, sw, _ = ops.quantize_weight_block(w, transposed=False)
    y = ops.gemm_fprop(qx, sx, qw, sw)
    ops.fp8bw_check_device_error()
    pi, pj = sample_points(m, n, seed=5, per_tile=1, stripes=1)
    keep = np.random.default_rng(6).choice(pi.size, 20000, replace=False)
    pi, pj = np.concatenate([pi[keep], [m - 1]]), np.concatenate([pj[keep], [n - 1]])
    acc, bound = oracle.gemm_fprop_points(qx.cpu().numpy(), sx.cpu().numpy(), qw.cpu().numpy(),
                                          sw.cpu().numpy(), pi, pj)
    got = torch_bf16_to_np(y[torch.from_numpy(pi).cuda(), torch.from_numpy(pj).cuda()])
    assert_gemm_close(got, acc, bound, "fprop 65536x33024x256")
    del y
    torch.cuda.empty_cache()


def test_wgrad_over_2_20_tokens():
    import torch
    ops = _ops()
    m, n, k = 1 << 20, 256, 272                # 8192 chunks of 128 tokens
    dy = _bf16((m, n), 1e-3, 14)
    x = _bf16((m, k), 1.0, 15)
    qdy_t, sdy_t = ops.quantize_colwise(dy)
    qx_t, sx_t = ops.quantize_colwise(x)
    dw = torch_bf16_to_np(ops.gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t))
    ops.fp8bw_check_device_error()
    pi, pj = sample_points(n, k, seed=7)
    acc, bound = oracle.gemm_wgrad_points(qdy_t.cpu().numpy(), sdy_t.cpu().numpy(),
                                          qx_t.cpu().numpy(), sx_t.cpu().numpy(), pi, pj)
    assert_gemm_close(dw[pi, pj], acc, bound, "wgrad over 2^20 tokens")
