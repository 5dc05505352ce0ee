"""Calls are asynchronous on the stream they are given and keep no state
between calls (no shared scratch): two streams running the linear step (with
a batched wgrad launch) at the same time give the serial results, and the
whole step captured in a CUDA graph and replayed gives the eager results."""
import pytest

import synthetic as S
from helpers import bf16_np_to_torch

pytestmark = pytest.mark.gpu


def _inputs(seed, m=1040, n=528, k=400):
    x = bf16_np_to_torch(S.bf16_normal((m, k), 0, seed, **S.X_DIST))
    w = bf16_np_to_torch(S.bf16_normal((n, k), 0, seed + 1, **S.W_DIST))
    dy = bf16_np_to_torch(S.bf16_normal((m, n), 0, seed + 2, **S.DY_DIST))
    return x, w, dy


def _step(ops, x, w, dy, stream):
    qw, sw, qw_t = ops.quantize_weight_block(w, stream=stream)
    qx_t, sx_t, qx, sx = ops.quantize_colwise(x, with_rowwise=True, stream=stream)
    y = ops.gemm_fprop(qx, sx, qw, sw, stream=stream)
    qdy_t, sdy_t, qdy, sdy = ops.quantize_colwise(dy, with_rowwise=True, stream=stream)
    dx = ops.gemm_dgrad(qdy, sdy, qw_t, sw, stream=stream)
    dw = ops.gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t, stream=stream)
    # the batched form, with a second job of another shape (dW transposed)
    dwb = ops.gemm_wgrad_batch([(qdy_t, sdy_t, qx_t, sx_t), (qx_t, sx_t, qdy_t, sdy_t)],
                               stream=stream)
    return (y, dx, dw, *dwb)


def _same(a, b):
    import torch
    return all(torch.equal(u.view(torch.int16), v.view(torch.int16)) for u, v in zip(a, b))


def test_two_streams_concurrently():
    import torch
    from blockwise_fp8_linear_fp8bw_b200 import ops
    a, b = _inputs(990), _inputs(995)
    ref_a = _step(ops, *a, torch.cuda.current_stream())
    ref_b = _step(ops, *b, torch.cuda.current_stream())
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for _ in range(3):
        with torch.cuda.stream(s1):
            oa = _step(ops, *a, s1)
        with torch.cuda.stream(s2):
            ob = _step(ops, *b, s2)
        outs.append((oa, ob))
    torch.cuda.synchronize()
    ops.fp8bw_check_device_error()
    for oa, ob in outs:
        assert _same(oa, ref_a) and _same(ob, ref_b)


def test_step_in_a_cuda_graph():
    import torch
    from blockwise_fp8_linear_fp8bw_b200 import ops
    x, w, dy = _inputs(1000)
    ref = _step(ops, x, w, dy, torch.cuda.current_stream())
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):           # warm-up outside the capture
        _step(ops, x, w, dy, s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        out = _step(ops, x, w, dy, s)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    ops.fp8bw_check_device_error()
    assert _same(out, ref)
    assert _same(out[3:4], out[2:3])     # the batch's first job is the single wgrad
    # new inputs copied into the captured buffers are picked up by a replay
    x2, w2, dy2 = _inputs(1005)
    ref2 = _step(ops, x2, w2, dy2, torch.cuda.current_stream())
    x.copy_(x2)
    w.copy_(w2)
    dy.copy_(dy2)
    g.replay()
    torch.cuda.synchronize()
    assert _same(out, ref2)
    del g
