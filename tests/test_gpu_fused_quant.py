"""GPU checks of fprop / dgrad with the quantisation of their own bf16
output fused into the epilogue, row-wise only or row-wise plus column-wise
(transposed) (paperlayer.ai summary of the Puro-2B report, Appendix C: bf16
hidden flow between E4M3 GEMMs; 1x128 groups of the arxiv-wiki summary,
Approach item (4)). Bit-exact: the bf16 output equals the unfused GEMM's, and
the codes and scales equal both the library's quantiser and the oracle's,
applied to that bf16 output."""
import numpy as np
import pytest

import oracle
import synthetic as S
from helpers import bf16_np_to_torch, scale_bits, torch_bf16_to_np

pytestmark = pytest.mark.gpu

SMALL = [(256, 256, 256), (128, 128, 128), (272, 400, 528), (512, 768, 384),
         (16, 16, 16), (1040, 272, 144), (384, 1296, 640)]


def _ops():
    from blockwise_fp8_linear_fp8bw_b200 import ops
    return ops


def _check_quant(ops, out, q, s, what):
    import torch
    rq, rs = ops.quantize_rowwise(out)
    assert torch.equal(q, rq), what + ": codes differ from the quantiser's"
    assert torch.equal(s.view(torch.int32), rs.view(torch.int32)), what + ": scales"
    oq, os_ = oracle.quantize_rowwise(torch_bf16_to_np(out))
    assert np.array_equal(q.cpu().numpy(), oq), what + ": codes differ from the oracle's"
    assert np.array_equal(scale_bits(s.cpu().numpy()), scale_bits(os_)), what + ": scales"


def _check_quant_cols(ops, out, q_t, s_t, what):
    import torch
    rq_t, rs_t = ops.quantize_colwise(out)
    assert torch.equal(q_t, rq_t), what + ": column codes differ from the quantiser's"
    assert torch.equal(s_t.view(torch.int32), rs_t.view(torch.int32)), what + ": column scales"
    oq_t, os_t = oracle.quantize_colwise(torch_bf16_to_np(out))
    assert np.array_equal(q_t.cpu().numpy(), oq_t), what + ": column codes vs the oracle"
    assert np.array_equal(scale_bits(s_t.cpu().numpy()), scale_bits(os_t)), \
        what + ": column scales vs the oracle"


def _fprop_rowcol(m, n, k, seed):
    import torch
    ops = _ops()
    x = S.bf16_normal((m, k), 0, seed, **S.X_DIST)
    w = S.bf16_normal((n, k), 0, seed + 1, **S.W_DIST)
    qx, sx = ops.quantize_rowwise(bf16_np_to_torch(x))
    qw, sw, _ = ops.quantize_weight_block(bf16_np_to_torch(w), transposed=False)
    y, qy, sy, qy_t, sy_t = ops.gemm_fprop_quant_rowcol(qx, sx, qw, sw)
    ops.fp8bw_check_device_error()
    assert torch.equal(y.view(torch.int16), ops.gemm_fprop(qx, sx, qw, sw).view(torch.int16))
    what = "fprop_quant_rowcol %dx%dx%d" % (m, n, k)
    _check_quant(ops, y, qy, sy, what)
    _check_quant_cols(ops, y, qy_t, sy_t, what)


def _dgrad_rowcol(m, n, k, seed, transposed):
    import torch
    ops = _ops()
    dy = S.bf16_normal((m, n), 0, seed, **S.DY_DIST)
    w = S.bf16_normal((n, k), 0, seed + 1, **S.W_DIST)
    qdy, sdy = ops.quantize_rowwise(bf16_np_to_torch(dy))
    qw, sw, qw_t = ops.quantize_weight_block(bf16_np_to_torch(w))
    b = qw_t if transposed else qw
    dx, qdx, sdx, qdx_t, sdx_t = ops.gemm_dgrad_quant_rowcol(
        qdy, sdy, b, sw, qw_is_transposed=transposed)
    ops.fp8bw_check_device_error()
    ref = ops.gemm_dgrad(qdy, sdy, b, sw, qw_is_transposed=transposed)
    assert torch.equal(dx.view(torch.int16), ref.view(torch.int16))
    what = "dgrad_quant_rowcol %dx%dx%d" % (m, n, k)
    _check_quant(ops, dx, qdx, sdx, what)
    _check_quant_cols(ops, dx, qdx_t, sdx_t, what)


def _fprop(m, n, k, seed):
    import torch
    ops = _ops()
    x = S.bf16_normal((m, k), 0, seed, **S.X_DIST)
    w = S.bf16_normal((n, k), 0, seed + 1, **S.W_DIST)
    qx, sx = ops.quantize_rowwise(bf16_np_to_torch(x))
    qw, sw, _ = ops.quantize_weight_block(bf16_np_to_torch(w), transposed=False)
    y, qy, sy = ops.gemm_fprop_quant(qx, sx, qw, sw)
    assert torch.equal(y.view(torch.int16), ops.gemm_fprop(qx, sx, qw, sw).view(torch.int16))
    _check_quant(ops, y, qy, sy, "fprop_quant %dx%dx%d" % (m, n, k))


def _dgrad(m, n, k, seed, transposed):
    import torch
    ops = _ops()
    dy = S.bf16_normal((m, n), 0, seed, **S.DY_DIST)
    w = S.bf16_normal((n, k), 0, seed + 1, **S.W_DIST)
    qdy, sdy = ops.quantize_rowwise(bf16_np_to_torch(dy))
    qw, sw, qw_t = ops.quantize_weight_block(bf16_np_to_torch(w))
    b = qw_t if transposed else qw
    dx, qdx, sdx = ops.gemm_dgrad_quant(qdy, sdy, b, sw, qw_is_transposed=transposed)
    ref = ops.gemm_dgrad(qdy, sdy, b, sw, qw_is_transposed=transposed)
    assert torch.equal(dx.view(torch.int16), ref.view(torch.int16))
    _check_quant(ops, dx, qdx, sdx, "dgrad_quant %dx%dx%d" % (m, n, k))


@pytest.mark.parametrize("m,n,k", SMALL)
def test_fprop_quant_small_and_ragged(m, n, k):
    _fprop(m, n, k, 801)


@pytest.mark.parametrize("m,n,k", SMALL)
@pytest.mark.parametrize("transposed", [True, False])
def test_dgrad_quant_small_and_ragged(m, n, k, transposed):
    _dgrad(m, n, k, 811, transposed)


def test_fused_quant_full_size():
    _fprop(16384, 12288, 2048, S.tensor_id("gate_up", "x"))
    _dgrad(16384, 2048, 6144, S.tensor_id("down", "dy"), True)
    _ops().fp8bw_check_device_error()


def test_fused_quant_empty_contraction():
    import torch
    ops = _ops()
    qx = torch.empty((128, 0), dtype=torch.uint8, device="cuda")
    sx = torch.empty((0, 128), dtype=torch.float32, device="cuda")
    qw = torch.empty((256, 0), dtype=torch.uint8, device="cuda")
    sw = torch.empty((2, 0), dtype=torch.float32, device="cuda")
    y = torch.full((128, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    qy = torch.full((128, 256), 5, dtype=torch.uint8, device="cuda")
    sy = torch.zeros((2, 128), dtype=torch.float32, device="cuda")
    ops.fp8bw_gemm_fprop_quant(qx, sx, qw, sw, y, qy, sy)
    assert torch.count_nonzero(y).item() == 0 and torch.count_nonzero(qy).item() == 0
    assert bool((sy == 1.0).all())


@pytest.mark.parametrize("m,n,k", SMALL + [(400, 272, 256), (144, 528, 384)])
def test_fprop_quant_rowcol_small_and_ragged(m, n, k):
    _fprop_rowcol(m, n, k, 821)


@pytest.mark.parametrize("m,n,k", SMALL)
@pytest.mark.parametrize("transposed", [True, False])
def test_dgrad_quant_rowcol_small_and_ragged(m, n, k, transposed):
    _dgrad_rowcol(m, n, k, 831, transposed)


def test_fused_quant_rowcol_full_size():
    _fprop_rowcol(16384, 12288, 2048, S.tensor_id("gate_up", "x"))
    _dgrad_rowcol(16384, 2048, 6144, S.tensor_id("down", "dy"), True)
    _ops().fp8bw_check_device_error()


def test_fused_quant_rowcol_empty_contraction():
    import torch
    ops = _ops()
    qx = torch.empty((128, 0), dtype=torch.uint8, device="cuda")
    sx = torch.empty((0, 128), dtype=torch.float32, device="cuda")
    qw = torch.empty((256, 0), dtype=torch.uint8, device="cuda")
    sw = torch.empty((2, 0), dtype=torch.float32, device="cuda")
    y = torch.full((128, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    qy = torch.full((128, 256), 5, dtype=torch.uint8, device="cuda")
    sy = torch.zeros((2, 128), dtype=torch.float32, device="cuda")
    qy_t = torch.full((256, 128), 5, dtype=torch.uint8, device="cuda")
    sy_t = torch.zeros((1, 256), dtype=torch.float32, device="cuda")
    ops.fp8bw_gemm_fprop_quant_rowcol(qx, sx, qw, sw, y, qy, sy, qy_t, sy_t)
    assert torch.count_nonzero(y).item() == 0 and torch.count_nonzero(qy).item() == 0
    assert torch.count_nonzero(qy_t).item() == 0
    assert bool((sy == 1.0).all()) and bool((sy_t == 1.0).all())
