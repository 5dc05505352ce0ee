"""Out-of-bounds writes and unwritten outputs (in place of a memory checker):
every output of every entry point is placed in a larger buffer filled with
0xCD, 4 KB of guard bytes on each side; after the call the guards must be
untouched and the output must equal the result of a normal call (whose values
the parity tests check against the oracle) -- so every byte was written, and
nothing outside it. Ragged shapes."""
import pytest

import synthetic as S
from helpers import bf16_np_to_torch

pytestmark = pytest.mark.gpu

GUARD = 4096
SHAPES = [(272, 400, 528), (16, 16, 16), (1040, 272, 144), (384, 1296, 640)]


def _ops():
    from blockwise_fp8_linear_fp8bw_b200 import ops
    return ops


class Guarded:
    """Output tensors carved out of one poisoned byte buffer."""

    def __init__(self):
        self.parts = []

    def make(self, shape, dtype):
        import torch
        n = 1
        for d in shape:
            n *= d
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        buf = torch.full((GUARD + nbytes + GUARD,), 0xCD, dtype=torch.uint8, device="cuda")
        t = buf[GUARD:GUARD + nbytes].view(dtype).view(shape)
        self.parts.append((buf, nbytes))
        return t

    def check(self, what):
        import torch
        torch.cuda.synchronize()
        for buf, nbytes in self.parts:
            head, tail = buf[:GUARD], buf[GUARD + nbytes:]
            assert bool((head == 0xCD).all()) and bool((tail == 0xCD).all()), \
                what + ": a write outside the output"


def _eq(a, b):
    import torch
    return torch.equal(a.view(torch.uint8), b.view(torch.uint8))


@pytest.mark.parametrize("m,n,k", SHAPES)
@pytest.mark.parametrize("pow2", [False, True])
def test_quantisers_write_exactly_their_outputs(m, n, k, pow2):
    import torch
    ops = _ops()
    x = bf16_np_to_torch(S.bf16_normal((m, k), 0, 970, **S.X_DIST))
    w = bf16_np_to_torch(S.bf16_normal((n, k), 0, 971, **S.W_DIST))
    cd = lambda a: (a + 127) // 128  # noqa: E731
    g = Guarded()
    q, s = g.make((m, k), torch.uint8), g.make((cd(k), m), torch.float32)
    q_t, s_t = g.make((k, m), torch.uint8), g.make((cd(m), k), torch.float32)
    q2, s2 = g.make((m, k), torch.uint8), g.make((cd(k), m), torch.float32)
    qw, sw, qw_t = (g.make((n, k), torch.uint8), g.make((cd(n), cd(k)), torch.float32),
                    g.make((k, n), torch.uint8))
    ops.fp8bw_quantize_rowwise(x, q, s, pow2=pow2)
    ops.fp8bw_quantize_colwise(x, q_t, s_t, q2, s2, pow2=pow2)
    ops.fp8bw_quantize_weight_block(w, qw, sw, qw_t, pow2=pow2)
    g.check("quantisers")
    rq, rs = ops.quantize_rowwise(x, pow2=pow2)
    rq_t, rs_t = ops.quantize_colwise(x, pow2=pow2)
    rqw, rsw, rqw_t = ops.quantize_weight_block(w, pow2=pow2)
    assert _eq(q, rq) and _eq(s, rs) and _eq(q2, rq) and _eq(s2, rs)
    assert _eq(q_t, rq_t) and _eq(s_t, rs_t)
    assert _eq(qw, rqw) and _eq(sw, rsw) and _eq(qw_t, rqw_t)


@pytest.mark.parametrize("m,n,k", SHAPES)
def test_gemms_write_exactly_their_outputs(m, n, k):
    import torch
    ops = _ops()
    x = bf16_np_to_torch(S.bf16_normal((m, k), 0, 980, **S.X_DIST))
    w = bf16_np_to_torch(S.bf16_normal((n, k), 0, 981, **S.W_DIST))
    dy = bf16_np_to_torch(S.bf16_normal((m, n), 0, 982, **S.DY_DIST))
    cd = lambda a: (a + 127) // 128  # noqa: E731
    for pow2 in (False, True):
        qx_t, sx_t, qx, sx = ops.quantize_colwise(x, with_rowwise=True, pow2=pow2)
        qdy_t, sdy_t, qdy, sdy = ops.quantize_colwise(dy, with_rowwise=True, pow2=pow2)
        qw, sw, qw_t = ops.quantize_weight_block(w, pow2=pow2)
        g = Guarded()
        y, dx, dx2, dw = (g.make((m, n), torch.bfloat16), g.make((m, k), torch.bfloat16),
                          g.make((m, k), torch.bfloat16), g.make((n, k), torch.bfloat16))
        ops.fp8bw_gemm_fprop(qx, sx, qw, sw, y, pow2=pow2)
        ops.fp8bw_gemm_dgrad(qdy, sdy, qw_t, 1, sw, dx, pow2=pow2)
        ops.fp8bw_gemm_dgrad(qdy, sdy, qw, 0, sw, dx2, pow2=pow2)
        ops.fp8bw_gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t, dw, pow2=pow2)
        g.check("GEMMs pow2=%s" % pow2)
        assert _eq(y, ops.gemm_fprop(qx, sx, qw, sw, pow2=pow2))
        ref_dx = ops.gemm_dgrad(qdy, sdy, qw_t, sw, pow2=pow2)
        assert _eq(dx, ref_dx) and _eq(dx2, ops.gemm_dgrad(qdy, sdy, qw, sw, False, pow2=pow2))
        assert _eq(dw, ops.gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t, pow2=pow2))
    # fp32 wgrad (store and add) and the fused-quantisation outputs
    qx_t, sx_t, qx, sx = ops.quantize_colwise(x, with_rowwise=True)
    qdy_t, sdy_t, qdy, sdy = ops.quantize_colwise(dy, with_rowwise=True)
    qw, sw, qw_t = ops.quantize_weight_block(w)
    g = Guarded()
    dw32 = g.make((n, k), torch.float32)
    acc32 = g.make((n, k), torch.float32)
    y, qy, sy = g.make((m, n), torch.bfloat16), g.make((m, n), torch.uint8), \
        g.make((cd(n), m), torch.float32)
    dx, qdx, sdx = g.make((m, k), torch.bfloat16), g.make((m, k), torch.uint8), \
        g.make((cd(k), m), torch.float32)
    acc32.zero_()
    ops.fp8bw_gemm_wgrad_f32(qdy_t, sdy_t, qx_t, sx_t, dw32)
    ops.fp8bw_gemm_wgrad_f32(qdy_t, sdy_t, qx_t, sx_t, acc32, accumulate=True)
    ops.fp8bw_gemm_fprop_quant(qx, sx, qw, sw, y, qy, sy)
    ops.fp8bw_gemm_dgrad_quant(qdy, sdy, qw_t, 1, sw, dx, qdx, sdx)
    g.check("fp32 wgrad and fused quantisation")
    ref32 = ops.gemm_wgrad_f32(qdy_t, sdy_t, qx_t, sx_t)
    assert _eq(dw32, ref32) and _eq(acc32, ref32)     # 0 + P == P exactly
    ry, rqy, rsy = ops.gemm_fprop_quant(qx, sx, qw, sw)
    rdx, rqdx, rsdx = ops.gemm_dgrad_quant(qdy, sdy, qw_t, sw)
    assert _eq(y, ry) and _eq(qy, rqy) and _eq(sy, rsy)
    assert _eq(dx, rdx) and _eq(qdx, rqdx) and _eq(sdx, rsdx)


@pytest.mark.parametrize("m,n,k", SHAPES + [(400, 272, 256)])
def test_newer_outputs_write_exactly_their_outputs(m, n, k):
    """The power-of-two fp32 wgrad (store and add) and the fused row +
    column output quantisation of fprop and dgrad."""
    import torch
    ops = _ops()
    x = bf16_np_to_torch(S.bf16_normal((m, k), 0, 990, **S.X_DIST))
    w = bf16_np_to_torch(S.bf16_normal((n, k), 0, 991, **S.W_DIST))
    dy = bf16_np_to_torch(S.bf16_normal((m, n), 0, 992, **S.DY_DIST))
    cd = lambda a: (a + 127) // 128  # noqa: E731
    pqx_t, psx_t = ops.quantize_colwise(x, pow2=True)
    pqdy_t, psdy_t = ops.quantize_colwise(dy, pow2=True)
    qx_t, sx_t, qx, sx = ops.quantize_colwise(x, with_rowwise=True)
    qdy_t, sdy_t, qdy, sdy = ops.quantize_colwise(dy, with_rowwise=True)
    qw, sw, qw_t = ops.quantize_weight_block(w)
    g = Guarded()
    dw32, acc32 = g.make((n, k), torch.float32), g.make((n, k), torch.float32)
    y, qy, sy = (g.make((m, n), torch.bfloat16), g.make((m, n), torch.uint8),
                 g.make((cd(n), m), torch.float32))
    qy_t, sy_t = g.make((n, m), torch.uint8), g.make((cd(m), n), torch.float32)
    dx, qdx, sdx = (g.make((m, k), torch.bfloat16), g.make((m, k), torch.uint8),
                    g.make((cd(k), m), torch.float32))
    qdx_t, sdx_t = g.make((k, m), torch.uint8), g.make((cd(m), k), torch.float32)
    acc32.zero_()
    ops.fp8bw_gemm_wgrad_f32(pqdy_t, psdy_t, pqx_t, psx_t, dw32, pow2=True)
    ops.fp8bw_gemm_wgrad_f32(pqdy_t, psdy_t, pqx_t, psx_t, acc32, accumulate=True,
                             pow2=True)
    ops.fp8bw_gemm_fprop_quant_rowcol(qx, sx, qw, sw, y, qy, sy, qy_t, sy_t)
    ops.fp8bw_gemm_dgrad_quant_rowcol(qdy, sdy, qw_t, 1, sw, dx, qdx, sdx, qdx_t, sdx_t)
    ops.fp8bw_check_device_error()
    g.check("power-of-two fp32 wgrad and fused row + column quantisation")
    ref32 = ops.gemm_wgrad_f32(pqdy_t, psdy_t, pqx_t, psx_t, pow2=True)
    assert _eq(dw32, ref32) and _eq(acc32, ref32)
    r = ops.gemm_fprop_quant_rowcol(qx, sx, qw, sw)
    assert all(_eq(a, b) for a, b in zip((y, qy, sy, qy_t, sy_t), r))
    r = ops.gemm_dgrad_quant_rowcol(qdy, sdy, qw_t, sw)
    assert all(_eq(a, b) for a, b in zip((dx, qdx, sdx, qdx_t, sdx_t), r))


@pytest.mark.parametrize("pow2", [False, True])
def test_weight_block_batch_writes_exactly_its_outputs(pow2):
    import torch
    ops = _ops()
    shapes = [(272, 400), (16, 16), (1040, 144), (384, 1296)]
    ws = [bf16_np_to_torch(S.bf16_normal(sh, 0, 995 + i, **S.W_DIST))
          for i, sh in enumerate(shapes)]
    cd = lambda a: (a + 127) // 128  # noqa: E731
    g = Guarded()
    qs = [g.make(sh, torch.uint8) for sh in shapes]
    ss = [g.make((cd(sh[0]), cd(sh[1])), torch.float32) for sh in shapes]
    qts = [g.make((sh[1], sh[0]), torch.uint8) for sh in shapes]
    ops.fp8bw_quantize_weight_block_batch(ws, qs, ss, qts, pow2=pow2)
    g.check("batched weight quantisation")
    for w, q, s, q_t in zip(ws, qs, ss, qts):
        rq, rs, rq_t = ops.quantize_weight_block(w, pow2=pow2)
        assert _eq(q, rq) and _eq(s, rs) and _eq(q_t, rq_t)


@pytest.mark.parametrize("pow2", [False, True])
def test_wgrad_batch_writes_exactly_its_outputs(pow2):
    """Four wgrad jobs of ragged shapes over the same tokens in one call: bf16
    dW, fp32 dW and the fp32 add into a main-grad, each in its own guarded
    buffer."""
    import torch
    ops = _ops()
    m = 400
    shapes = [(272, 400), (16, 16), (1040, 144), (384, 1296)]   # (n, k)
    operands = []
    for i, (n, k) in enumerate(shapes):
        dy = bf16_np_to_torch(S.bf16_normal((m, n), 0, 1500 + 2 * i, **S.DY_DIST))
        x = bf16_np_to_torch(S.bf16_normal((m, k), 0, 1501 + 2 * i, **S.X_DIST))
        operands.append(ops.quantize_colwise(dy, pow2=pow2) + ops.quantize_colwise(x, pow2=pow2))
    g = Guarded()
    dws = [g.make(sh, torch.bfloat16) for sh in shapes]
    dw32 = [g.make(sh, torch.float32) for sh in shapes]
    acc32 = [g.make(sh, torch.float32) for sh in shapes]
    for a in acc32:
        a.zero_()
    ops.fp8bw_gemm_wgrad_batch([tuple(o) + (d,) for o, d in zip(operands, dws)], pow2=pow2)
    ops.fp8bw_gemm_wgrad_f32_batch([tuple(o) + (d,) for o, d in zip(operands, dw32)],
                                   pow2=pow2)
    ops.fp8bw_gemm_wgrad_f32_batch([tuple(o) + (d,) for o, d in zip(operands, acc32)],
                                   accumulate=True, pow2=pow2)
    ops.fp8bw_check_device_error()
    g.check("batched wgrad")
    for o, d, d32, a32 in zip(operands, dws, dw32, acc32):
        assert _eq(d, ops.gemm_wgrad(*o, pow2=pow2))
        ref32 = ops.gemm_wgrad_f32(*o, pow2=pow2)
        assert _eq(d32, ref32) and _eq(a32, ref32)
