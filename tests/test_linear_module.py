"""The blockwise-FP8 training linear (linear.py): forward y = x W^T, backward
dX and dW (returned in the weight's dtype, or added in fp32 into
weight.main_grad), against the oracle's quantisers and GEMMs on the same
inputs; plus its argument checks on CPU (no CPU fallback)."""
import numpy as np
import pytest

import oracle
import synthetic as S
from helpers import (assert_gemm_close, assert_gemm_close_f32, bf16_np_to_torch,
                     torch_bf16_to_np)


def test_rejects_cpu_tensors_and_bad_sizes():
    import torch
    from blockwise_fp8_linear_fp8bw_b200.linear import BlockwiseFp8Linear
    with pytest.raises(ValueError):
        BlockwiseFp8Linear(100, 128)
    lin = BlockwiseFp8Linear(256, 128)
    with pytest.raises(ValueError):
        lin(torch.zeros((16, 256), dtype=torch.bfloat16))


def _case(pow2, main_grad, shape=(2, 144), k=400, n=528, seed=950):
    import torch
    from blockwise_fp8_linear_fp8bw_b200.linear import BlockwiseFp8Linear
    m = shape[0] * shape[1]
    x = S.bf16_normal((m, k), 0, seed, **S.X_DIST)
    w = S.bf16_normal((n, k), 0, seed + 1, **S.W_DIST)
    dy = S.bf16_normal((m, n), 0, seed + 2, **S.DY_DIST)
    lin = BlockwiseFp8Linear(k, n, device="cuda", pow2=pow2)
    with torch.no_grad():
        lin.weight.copy_(bf16_np_to_torch(w))
    if main_grad:
        lin.weight.main_grad = torch.zeros((n, k), dtype=torch.float32, device="cuda")
    xt = bf16_np_to_torch(x).reshape(*shape, k).requires_grad_(True)
    y = lin(xt)
    assert y.shape == (*shape, n) and y.dtype == torch.bfloat16
    y.backward(bf16_np_to_torch(dy).reshape(*shape, n))
    torch.cuda.synchronize()

    rqx, rsx = oracle.quantize_rowwise(x, pow2=pow2)
    rqw, rsw, _ = oracle.quantize_weight_block(w, want_transposed=False, pow2=pow2)
    acc, bound = oracle.gemm_fprop(rqx, rsx, rqw, rsw, with_bound=True)
    assert_gemm_close(torch_bf16_to_np(y.reshape(m, n)), acc, bound, "linear forward")
    rq, rs = oracle.quantize_rowwise(dy, pow2=pow2)
    acc, bound = oracle.gemm_dgrad(rq, rs, rqw, rsw, with_bound=True)
    assert_gemm_close(torch_bf16_to_np(xt.grad.reshape(m, k)), acc, bound, "linear dX")
    rq_t, rs_t = oracle.quantize_colwise(dy, pow2=pow2)
    rqx_t, rsx_t = oracle.quantize_colwise(x, pow2=pow2)
    acc, bound = oracle.gemm_wgrad(rq_t, rs_t, rqx_t, rsx_t, with_bound=True)
    if main_grad:
        assert lin.weight.grad is None
        got = lin.weight.main_grad.cpu().numpy()
        if pow2:      # the power-of-two wgrad is bf16, added into a zeroed fp32 buffer
            bits = (got.view(np.uint32) >> 16).astype(np.uint16)
            assert_gemm_close(bits, acc, bound, "linear dW (main_grad, pow2)")
        else:
            assert_gemm_close_f32(got, acc, bound, "linear dW (main_grad)")
    else:
        assert lin.weight.grad.dtype == torch.bfloat16
        assert_gemm_close(torch_bf16_to_np(lin.weight.grad), acc, bound, "linear dW")


@pytest.mark.gpu
@pytest.mark.parametrize("pow2", [False, True])
@pytest.mark.parametrize("main_grad", [False, True])
def test_linear_forward_backward(pow2, main_grad):
    _case(pow2, main_grad)


@pytest.mark.gpu
def test_library_call_from_a_fresh_thread():
    """A thread that has done no CUDA work of its own (as autograd's backward
    thread may be) can call the library: the entry points make the device's
    context current before encoding tensor maps."""
    import threading
    import torch
    from blockwise_fp8_linear_fp8bw_b200 import ops
    x = bf16_np_to_torch(S.bf16_normal((256, 384), 0, 960, **S.X_DIST))
    ref_q, ref_s = ops.quantize_rowwise(x)
    torch.cuda.synchronize()
    out, err = {}, []

    def work():
        try:
            out["qs"] = ops.quantize_colwise(x, with_rowwise=True)
            torch.cuda.synchronize()
        except Exception as e:          # reported to the main thread
            err.append(e)

    t = threading.Thread(target=work)
    t.start()
    t.join()
    assert not err, err
    q_t, s_t, q, s = out["qs"]
    assert torch.equal(q, ref_q) and torch.equal(s.view(torch.int32), ref_s.view(torch.int32))
