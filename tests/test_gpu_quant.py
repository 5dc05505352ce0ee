"""GPU parity of the quantisers: codes and scales bit-identical to the oracle
on every element, through the C ABI (blockwise_fp8_linear_fp8bw_b200.ops).
Reading of the pages: E4M3, 1x128 activation groups, 128x128 weight blocks
(Puro-2B arxiv-wiki summary, Approach item (4)); qscale = 448/amax,
s = amax/448, all-zero groups get qscale = s = 1."""
import numpy as np
import pytest

import oracle
import synthetic as S
from helpers import bf16_np_to_torch, hand_groups, scale_bits, torch_bf16_to_np

pytestmark = pytest.mark.gpu


def _ops():
    from blockwise_fp8_linear_fp8bw_b200 import ops
    return ops


def _check_rowwise(x):
    ops = _ops()
    q, s = ops.quantize_rowwise(bf16_np_to_torch(x))
    rq, rs = oracle.quantize_rowwise(x)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(scale_bits(s.cpu().numpy()), scale_bits(rs))


def _check_colwise(x, with_rowwise):
    ops = _ops()
    out = ops.quantize_colwise(bf16_np_to_torch(x), with_rowwise=with_rowwise)
    rq_t, rs_t = oracle.quantize_colwise(x)
    assert np.array_equal(out[0].cpu().numpy(), rq_t)
    assert np.array_equal(scale_bits(out[1].cpu().numpy()), scale_bits(rs_t))
    if with_rowwise:
        rq, rs = oracle.quantize_rowwise(x)
        assert np.array_equal(out[2].cpu().numpy(), rq)
        assert np.array_equal(scale_bits(out[3].cpu().numpy()),
                              scale_bits(rs))


def _check_weight(w, transposed=True):
    ops = _ops()
    q, s, q_t = ops.quantize_weight_block(bf16_np_to_torch(w),
                                          transposed=transposed)
    rq, rs, rq_t = oracle.quantize_weight_block(w)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(scale_bits(s.cpu().numpy()), scale_bits(rs))
    if transposed:
        assert np.array_equal(q_t.cpu().numpy(), rq_t)


SMALL = [(256, 256), (128, 128), (272, 400), (16, 16), (16, 2064),
         (1040, 48), (384, 640)]


@pytest.mark.parametrize("rows,cols", SMALL)
def test_rowwise_small_and_ragged(rows, cols):
    _check_rowwise(S.bf16_normal((rows, cols), 0, 501, 1.0, 1e-2, 50.0))


@pytest.mark.parametrize("rows,cols", SMALL)
@pytest.mark.parametrize("with_rowwise", [False, True])
def test_colwise_small_and_ragged(rows, cols, with_rowwise):
    _check_colwise(S.bf16_normal((rows, cols), 0, 502, 1e-3, 1e-2, 100.0),
                   with_rowwise)


@pytest.mark.parametrize("n,k", SMALL)
@pytest.mark.parametrize("transposed", [False, True])
def test_weight_block_small_and_ragged(n, k, transposed):
    _check_weight(S.bf16_normal((n, k), 0, 503, 0.02), transposed)


def test_special_groups():
    # all-zero rows/cols, signed zeros, bf16 subnormals (qscale overflows ->
    # s = 1, codes +-0), a group holding +-448 and RNE ties, huge values.
    rows, cols = 256, 384
    f = np.zeros((rows, cols), np.float32)
    f[1, :128] = -0.0
    f[2, :] = np.float32(2.0 ** -133)        # smallest bf16 subnormal
    f[3, :] = -np.float32(2.0 ** -130)
    f[4, :9] = [448, -448, 17, 19, 2 ** -10, 3 * 2 ** -10, 15 * 2 ** -10,
                7 * 2 ** -9, -0.0]
    f[5, :] = 3.0e38
    f[6, 128:256] = np.float32(1e-36)
    f[7:140, 300] = np.linspace(-5, 5, 133).astype(np.float32)
    x = (f.view(np.uint32) >> 16).astype(np.uint16)   # truncate to bf16
    _check_rowwise(x)
    _check_colwise(x, True)
    _check_weight(x)


@pytest.mark.parametrize("pow2,fname", [(False, "quant_group_hand.txt"),
                                         (True, "quant_pow2_hand.txt")])
def test_hand_worked_groups(pow2, fname):
    """The hand-worked golden groups (values, codes and scale bits derived by
    hand, tests/golden/) through every quantiser: each group as a row-wise
    1x128 group, as a column-wise 128x1 group and as the only non-zero row of
    a 128x128 weight block (whose amax is then the group's). The file's
    r2_* groups sit on E4M3 midpoints where multiplying by fl32(448/amax) and
    dividing by fl32(amax/448) give different codes."""
    ops = _ops()
    groups = hand_groups(fname)
    n = len(groups)
    f = np.zeros((128 * n, 128), np.float32)
    for i, (_name, vals, fill, _codes, _sbits) in enumerate(groups):
        f[128 * i + 3, :] = fill
        f[128 * i + 3, :len(vals)] = vals
    x = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((x.astype(np.uint32) << 16).view(np.float32), f)
    xt = np.ascontiguousarray(x.T)                     # groups as columns
    q, s = ops.quantize_rowwise(bf16_np_to_torch(x), pow2=pow2)
    q_t, s_t = ops.quantize_colwise(bf16_np_to_torch(xt), pow2=pow2)
    qb, sb, _ = ops.quantize_weight_block(bf16_np_to_torch(x), pow2=pow2)
    ops.fp8bw_check_device_error()
    q, s = q.cpu().numpy(), scale_bits(s.cpu().numpy())
    q_t, s_t = q_t.cpu().numpy(), scale_bits(s_t.cpu().numpy())
    qb, sb = qb.cpu().numpy(), scale_bits(sb.cpu().numpy())
    for i, (name, vals, _fill, codes, sbits) in enumerate(groups):
        r = 128 * i + 3
        assert q[r, :len(codes)].tolist() == codes, name
        assert s[0, r] == sbits, name
        assert q_t[r, :len(codes)].tolist() == codes, name     # q_t[col][tok]
        assert s_t[0, r] == sbits, name
        assert qb[r, :len(codes)].tolist() == codes, name
        assert sb[i, 0] == sbits, name


def test_empty_is_a_noop():
    import torch
    ops = _ops()
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    q, s = ops.quantize_rowwise(x)
    assert q.shape == (0, 256) and s.shape == (2, 0)
    x = torch.empty((128, 0), dtype=torch.bfloat16, device="cuda")
    q_t, s_t = ops.quantize_colwise(x)
    assert q_t.shape == (0, 128)


def test_misaligned_view_is_rejected():
    import torch
    ops = _ops()
    base = torch.zeros(128 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    x = base[1:1 + 128 * 128].view(128, 128)          # 2-byte offset
    with pytest.raises(ops.Fp8bwError) as e:
        ops.quantize_rowwise(x)
    assert e.value.status == ops.FP8BW_ERR_ALIGN


FULL = {
    "qkv_fprop_m8192": [("x", 8192, 2048)],
    "mlp_fprop_m16384": [("x", 16384, 2048), ("x", 16384, 6144)],
    "mlp_backward_m16384": [("dy", 16384, 2048), ("dy", 16384, 12288)],
}


@pytest.mark.parametrize("kind", ["qkv", "o"])
def test_full_size_attention_quantisers(kind):
    """Every element of the 28-layer stack's QKV and O inputs, output
    gradients (row + column, one pass) and weights at M = 16384."""
    lin = [l for l in S.workload("stack28_m16384")
           if l.kind == kind and l.layer == 0][0]
    _check_colwise(S.draw_x(lin), True)
    _check_colwise(S.draw_dy(lin), True)
    _check_weight(S.draw_w(lin))
    _ops().fp8bw_check_device_error()


@pytest.mark.parametrize("name", sorted(FULL))
def test_full_size_activation_quantisers(name):
    """Every element of the workloads' activations and gradients, row-wise and
    column-wise in one pass, and the weights of those linears."""
    for lin in S.workload(name):
        x = S.draw_dy(lin) if "backward" in name else S.draw_x(lin)
        _check_colwise(x, True)
        _check_weight(S.draw_w(lin))
    _ops().fp8bw_check_device_error()


@pytest.mark.parametrize("pow2", [False, True])
def test_weight_block_batch_equals_one_by_one(pow2):
    """Several weights in one launch (ragged shapes, an empty one, with and
    without transposed codes): each job's codes and scales equal, bit for bit,
    the single-weight quantiser's and the oracle's."""
    import torch
    ops = _ops()
    shapes = [(12288, 2048), (272, 400), (0, 256), (2048, 6144), (16, 16), (1040, 48)]
    ws = [bf16_np_to_torch(S.bf16_normal(sh, 0, 560 + i, 0.02)) if sh[0] else
          torch.empty(sh, dtype=torch.bfloat16, device="cuda")
          for i, sh in enumerate(shapes)]
    outs = ops.quantize_weight_block_batch(ws, pow2=pow2)
    qts = [o[2] for o in outs]
    qts[3] = None                        # one job without transposed codes
    qs = [o[0] for o in outs]
    ss = [o[1] for o in outs]
    ops.fp8bw_quantize_weight_block_batch(ws, qs, ss, qts, pow2=pow2)
    ops.fp8bw_check_device_error()
    for i, (w, q, s) in enumerate(zip(ws, qs, ss)):
        if w.numel() == 0:
            continue
        rq, rs, rq_t = ops.quantize_weight_block(w, pow2=pow2)
        assert torch.equal(q, rq), i
        assert torch.equal(s.view(torch.int32), rs.view(torch.int32)), i
        if qts[i] is not None:
            assert torch.equal(qts[i], rq_t), i
        if w.shape[0] * w.shape[1] <= 1 << 22:
            oq, os_, _ = oracle.quantize_weight_block(torch_bf16_to_np(w), pow2=pow2)
            assert np.array_equal(q.cpu().numpy(), oq), i
            assert np.array_equal(scale_bits(s.cpu().numpy()), scale_bits(os_)), i
