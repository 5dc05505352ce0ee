"""The blockwise-FP8 training linear (linear.py): forward y = x W^T, backward
dX and dW (returned in the weight's dtype, or added in fp32 into
weight.main_grad), against the oracle's quantisers and GEMMs on the same
inputs; plus its argument checks on CPU (no CPU fallback)."""
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
        # both scale forms add the fp32 dW into main_grad in the GEMM epilogue
        assert lin.weight.grad is None
        got = lin.weight.main_grad.cpu().numpy()
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


@pytest.mark.gpu
@pytest.mark.parametrize("main_grad", [False, True])
def test_chain_equals_the_linears_one_by_one(main_grad):
    """Three linears that feed one another: the chain (quantisation of the
    intermediate activations and gradients fused into the producing GEMMs)
    gives, bit for bit, the output, dX and dW of the same linears run one by
    one with their own quantisers; and the first linear's dW is within the
    acceptance bound of the oracle's, given the gradient that reached its
    output."""
    import torch
    from blockwise_fp8_linear_fp8bw_b200.linear import (BlockwiseFp8Chain,
                                                         BlockwiseFp8Linear)
    feats = [400, 272, 528, 144]
    m = 288
    chain = BlockwiseFp8Chain(feats, device="cuda")
    singles = [BlockwiseFp8Linear(a, b, device="cuda")
               for a, b in zip(feats[:-1], feats[1:])]
    for i, lin in enumerate(singles):
        w = S.bf16_normal((feats[i + 1], feats[i]), 0, 970 + i, **S.W_DIST)
        with torch.no_grad():
            lin.weight.copy_(bf16_np_to_torch(w))
            chain.weights[i].copy_(bf16_np_to_torch(w))
        if main_grad:
            lin.weight.main_grad = torch.zeros(lin.weight.shape, dtype=torch.float32,
                                               device="cuda")
            chain.weights[i].main_grad = torch.zeros(lin.weight.shape,
                                                     dtype=torch.float32, device="cuda")
    x = S.bf16_normal((m, feats[0]), 0, 975, **S.X_DIST)
    dy = S.bf16_normal((m, feats[-1]), 0, 976, **S.DY_DIST)
    xa = bf16_np_to_torch(x).requires_grad_(True)
    xb = bf16_np_to_torch(x).requires_grad_(True)
    g = bf16_np_to_torch(dy)
    ya = chain(xa)
    ya.backward(g)
    outs = []
    h = xb
    for lin in singles:
        h = lin(h)
        outs.append(h)
    seen = {}
    outs[0].register_hook(lambda t: seen.setdefault("dy0", t.detach().clone()))
    outs[-1].backward(g)
    torch.cuda.synchronize()

    eq = lambda a, b: torch.equal(a.view(torch.int16), b.view(torch.int16))  # noqa: E731
    assert eq(ya, outs[-1]) and eq(xa.grad, xb.grad)
    for i, lin in enumerate(singles):
        if main_grad:
            assert chain.weights[i].grad is None
            assert torch.equal(chain.weights[i].main_grad.view(torch.int32),
                               lin.weight.main_grad.view(torch.int32))
        else:
            assert eq(chain.weights[i].grad, lin.weight.grad)

    rq_t, rs_t = oracle.quantize_colwise(torch_bf16_to_np(seen["dy0"]))
    rqx_t, rsx_t = oracle.quantize_colwise(x)
    acc, bound = oracle.gemm_wgrad(rq_t, rs_t, rqx_t, rsx_t, with_bound=True)
    if main_grad:
        assert_gemm_close_f32(chain.weights[0].main_grad.cpu().numpy(), acc, bound,
                              "chain dW_0 (main_grad)")
    else:
        assert_gemm_close(torch_bf16_to_np(chain.weights[0].grad), acc, bound,
                          "chain dW_0")
