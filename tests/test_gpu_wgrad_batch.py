"""GPU parity of the batched weight-gradient GEMM (several linears' dW over the
same tokens in one launch; paperlayer.ai summary of the Puro-2B report,
Appendix C, "FP8 implementation pipeline": the weight-gradient GEMM of each
linear), through the C ABI.

Checks:
  * against the oracle, job by job: every dW within the acceptance bound of
    the oracle's fp64 value on the same quantised operands;
  * that a batch computes exactly what the single-problem entry point does:
    bf16 dW, fp32 dW and the fp32 add into a main-grad, bit for bit, for jobs
    of different shapes (ragged edges, tile counts that do not fill a wave,
    a job of one tile), for both scale forms;
  * that empty jobs (n or k zero) are skipped and an empty contraction writes
    zeros (or leaves a main-grad unchanged);
  * the bench step's launch at full size: a layer's four linears at M =
    16384, bit-equal to the single calls and within the bound of the oracle
    on sampled points.
"""
import numpy as np
import pytest

import oracle
import synthetic as S
from helpers import assert_gemm_close, bf16_np_to_torch, torch_bf16_to_np

pytestmark = pytest.mark.gpu


def _ops():
    from blockwise_fp8_linear_fp8bw_b200 import ops
    return ops


def _operands(m, shapes, seed, pow2=False):
    """Quantised (dY^T, X^T) of each (n, k) in `shapes`, and the bf16 inputs."""
    ops = _ops()
    out = []
    for i, (n, k) in enumerate(shapes):
        dy = S.bf16_normal((m, n), 0, seed + 2 * i, **S.DY_DIST)
        x = S.bf16_normal((m, k), 0, seed + 2 * i + 1, **S.X_DIST)
        qdy_t, sdy_t = ops.quantize_colwise(bf16_np_to_torch(dy), pow2=pow2)
        qx_t, sx_t = ops.quantize_colwise(bf16_np_to_torch(x), pow2=pow2)
        out.append(((qdy_t, sdy_t, qx_t, sx_t), dy, x))
    return out


def _eq(a, b):
    import torch
    return torch.equal(a.view(torch.int32) if a.dtype == torch.float32 else
                       a.view(torch.int16),
                       b.view(torch.int32) if b.dtype == torch.float32 else
                       b.view(torch.int16))


# (m, [(n, k), ...]): jobs with 1, 2 and 6 row tiles, ragged n and k, a job
# of a single tile, and several partial waves
CASES = [
    (400, [(272, 400), (128, 144), (528, 256)]),
    (256, [(1024, 512), (256, 256), (768, 1280), (160, 96)]),
    (1152, [(4096, 2048), (2048, 2048)]),
]


@pytest.mark.parametrize("pow2", [False, True])
@pytest.mark.parametrize("m,shapes", CASES)
def test_batch_equals_one_by_one(m, shapes, pow2):
    import torch
    ops = _ops()
    ops_in = _operands(m, shapes, 1200 + m, pow2=pow2)
    operands = [o[0] for o in ops_in]

    got = ops.gemm_wgrad_batch(operands, pow2=pow2)
    want = [ops.gemm_wgrad(*o, pow2=pow2) for o in operands]
    got32 = ops.gemm_wgrad_f32_batch(operands, pow2=pow2)
    want32 = [ops.gemm_wgrad_f32(*o, pow2=pow2) for o in operands]
    g_batch = [torch.full((o[0].shape[0], o[2].shape[0]), 0.25, device="cuda")
               for o in operands]
    g_single = [g.clone() for g in g_batch]
    ops.gemm_wgrad_f32_batch(operands, main_grads=g_batch, pow2=pow2)
    for o, g in zip(operands, g_single):
        ops.gemm_wgrad_f32(*o, main_grad=g, pow2=pow2)
    ops.fp8bw_check_device_error()
    for i in range(len(shapes)):
        what = "job %d %s of m=%d" % (i, shapes[i], m)
        assert _eq(got[i], want[i]), what + ": bf16 dW differs from the single call"
        assert _eq(got32[i], want32[i]), what + ": fp32 dW differs from the single call"
        assert _eq(g_batch[i], g_single[i]), what + ": main-grad add differs"


@pytest.mark.parametrize("m,shapes", CASES[:2])
def test_batch_against_oracle(m, shapes):
    ops = _ops()
    ops_in = _operands(m, shapes, 1300 + m)
    dws = ops.gemm_wgrad_batch([o[0] for o in ops_in])
    ops.fp8bw_check_device_error()
    for i, (_, dy, x) in enumerate(ops_in):
        rq, rs = oracle.quantize_colwise(dy)
        rqx, rsx = oracle.quantize_colwise(x)
        acc, bound = oracle.gemm_wgrad(rq, rs, rqx, rsx, with_bound=True)
        assert_gemm_close(torch_bf16_to_np(dws[i]), acc, bound,
                          "batched wgrad job %d %s" % (i, shapes[i]))


def test_empty_jobs_and_empty_contraction():
    import torch
    ops = _ops()
    u8, f32 = torch.uint8, torch.float32
    e = lambda *s, dt=u8: torch.empty(s, dtype=dt, device="cuda")  # noqa: E731
    ops_in = _operands(256, [(256, 128)], 1400)
    live = ops_in[0][0]
    # a job with k = 0 next to a real one: the real one is unaffected
    empty_k = (e(128, 256), e(2, 128, dt=f32), e(0, 256), e(2, 0, dt=f32))
    got = ops.gemm_wgrad_batch([live, empty_k])
    assert got[1].shape == (128, 0)
    assert _eq(got[0], ops.gemm_wgrad(*live))
    # m = 0: dW = 0 (stored), a main-grad unchanged (accumulated)
    z = (e(256, 0), e(0, 256, dt=f32), e(128, 0), e(0, 128, dt=f32))
    dw = torch.full((256, 128), 3.0, dtype=torch.bfloat16, device="cuda")
    ops.fp8bw_gemm_wgrad_batch([z + (dw,)])
    g = torch.full((256, 128), 0.5, device="cuda")
    ops.fp8bw_gemm_wgrad_f32_batch([z + (g,)], accumulate=True)
    ops.fp8bw_check_device_error()
    assert not dw.float().abs().sum().item()
    assert np.all(g.cpu().numpy() == np.float32(0.5))


def test_full_size_layer_batch():
    """The bench step's launch: the four linears of a layer (QKV, O, gate/up,
    down) at M = 16384 in one batched wgrad. Each dW equals the single-problem
    wgrad bit for bit, and sampled points (>= 16 per 128x128 tile plus two
    full rows and columns) are within the acceptance bound of the oracle."""
    from helpers import sample_points
    ops = _ops()
    m = 16384
    jobs, ins = [], []
    for kind in ("qkv", "o", "gate_up", "down"):
        k, n = S.LINEARS[kind]
        dy = S.bf16_normal((m, n), 0, S.tensor_id(kind, "dy", 0), **S.DY_DIST)
        x = S.bf16_normal((m, k), 0, S.tensor_id(kind, "x", 0), **S.X_DIST)
        jobs.append(ops.quantize_colwise(bf16_np_to_torch(dy)) +
                    ops.quantize_colwise(bf16_np_to_torch(x)))
        ins.append((dy, x, n, k))
    dws = ops.gemm_wgrad_batch(jobs)
    singles = [ops.gemm_wgrad(*j) for j in jobs]
    ops.fp8bw_check_device_error()
    for (dy, x, n, k), dw, single in zip(ins, dws, singles):
        assert _eq(dw, single), "batched dW %dx%d differs from the single call" % (n, k)
        rq, rs = oracle.quantize_colwise(dy)
        rqx, rsx = oracle.quantize_colwise(x)
        pi, pj = sample_points(n, k)
        acc, bound = oracle.gemm_wgrad_points(rq, rs, rqx, rsx, pi, pj)
        assert_gemm_close(torch_bf16_to_np(dw)[pi, pj], acc, bound,
                          "batched wgrad %dx%dx%d" % (m, n, k))
