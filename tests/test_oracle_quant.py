"""Pins of the oracle's quantisers: hand-worked groups, the special cases of
the scale reading, cross-layout identities, an independent amax, and the
dequantisation error bound that E4M3 rounding guarantees.

Reading of the pages (Puro-2B arxiv-wiki summary, Approach item (4): E4M3,
activation 1-D groups of 128, weight 128x128 blocks): qscale = fl(448/amax),
s = fl(amax/448), all-zero groups get qscale = s = 1.
"""
import numpy as np
import pytest

import oracle
import synthetic as S
from helpers import hand_groups


def bf16_bits(vals):
    f = np.asarray(vals, dtype=np.float32)
    u = f.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not exactly bf16"
    return (u >> 16).astype(np.uint16)


def f32_of(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("name,vals,fill,codes,sbits", hand_groups())
def test_hand_worked_group(name, vals, fill, codes, sbits):
    g = np.full(128, fill, dtype=np.float32)
    g[: len(vals)] = vals
    q, s = oracle.quantize_rowwise(bf16_bits(g)[None, :])
    assert q[0, : len(codes)].tolist() == codes, name
    assert s.view(np.uint32)[0, 0] == sbits, (name, hex(s.view(np.uint32)[0, 0]))


def test_amax_element_saturates_exactly_to_448():
    x = S.bf16_normal((64, 512), 0, 101, 1.0, 1e-2, 50.0)
    q, s = oracle.quantize_rowwise(x)
    f = f32_of(x).reshape(64, 4, 128)
    qq = q.reshape(64, 4, 128)
    idx = np.abs(f).argmax(axis=2)
    top = np.take_along_axis(qq, idx[..., None], axis=2)[..., 0]
    assert np.all((top & 0x7F) == 0x7E)


def test_scale_special_cases():
    assert oracle.group_scale(0.0) == (1.0, 1.0)
    # 448/1e-38 overflows fp32 -> the all-zero reading applies
    q, s = oracle.group_scale(np.float32(1e-38))
    assert (q, s) == (1.0, 1.0)
    # 448/2e-36 is finite: ordinary scales (s is an fp32 subnormal)
    q, s = oracle.group_scale(np.float32(2e-36))
    assert np.isfinite(q) and q > 1e38
    assert s == np.float32(np.float32(2e-36) / np.float32(448.0))


def test_tiny_group_encodes_to_signed_zero():
    b = np.zeros(128, np.uint16)
    b[0] = 0x0001          # smallest bf16 subnormal, 2^-133
    b[1] = 0x8001          # its negative
    q, s = oracle.quantize_rowwise(b[None, :])
    assert s[0, 0] == 1.0
    assert q[0, 0] == 0x00 and q[0, 1] == 0x80


def _independent_amax(f, axis_groups):
    return np.abs(f).max(axis=axis_groups)


@pytest.mark.parametrize("rows,cols", [(128, 256), (200, 300), (1, 129),
                                       (257, 1)])
def test_rowwise_scales_from_independent_amax(rows, cols):
    x = S.bf16_normal((rows, cols), 0, 102, 1.0, 1e-2, 50.0)
    q, s = oracle.quantize_rowwise(x)
    f = f32_of(x)
    G = -(-cols // 128)
    assert s.shape == (G, rows)
    for g in range(G):
        amax = np.abs(f[:, g * 128:(g + 1) * 128]).max(axis=1)
        exp = (amax / np.float32(448.0)).astype(np.float32)
        exp[amax == 0] = 1.0
        assert np.array_equal(s[g], exp)


@pytest.mark.parametrize("rows,cols", [(256, 128), (300, 200), (129, 3)])
def test_colwise_equals_rowwise_of_transpose(rows, cols):
    x = S.bf16_normal((rows, cols), 0, 103, 1e-3, 1e-2, 100.0)
    q_t, s_t = oracle.quantize_colwise(x)
    q_r, s_r = oracle.quantize_rowwise(np.ascontiguousarray(x.T))
    assert np.array_equal(q_t, q_r)
    assert np.array_equal(s_t, s_r)


@pytest.mark.parametrize("n,k", [(256, 384), (200, 130), (128, 128)])
def test_weight_block_scales_and_transpose(n, k):
    w = S.bf16_normal((n, k), 0, 104, 0.02)
    q, s, q_t = oracle.quantize_weight_block(w)
    assert np.array_equal(q_t, q.T)
    f = np.abs(f32_of(w))
    nb, kb = -(-n // 128), -(-k // 128)
    for i in range(nb):
        for j in range(kb):
            blk = f[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            assert s[i, j] == np.float32(blk.max() / np.float32(448.0))
    # every block's largest element encodes to +-448
    for i in range(nb):
        for j in range(kb):
            blk = f[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            r, c = np.unravel_index(blk.argmax(), blk.shape)
            assert q[i * 128 + r, j * 128 + c] & 0x7F == 0x7E


def _roundtrip_check(codes, scale_of_elem, f):
    """E4M3 has 3 mantissa bits: an element whose scaled value is normal
    (|x*qscale| >= 2^-6) dequantises within 2^-4 relative; a subnormal one
    within half the subnormal quantum, 2^-10 * s. (1 + 2^-20) absorbs the
    fp32 rounding of qscale and s."""
    dec = oracle.e4m3_decode_table()[codes]
    deq = dec * scale_of_elem.astype(np.float64)
    x = f.astype(np.float64)
    err = np.abs(deq - x)
    normal = np.abs(x) >= (2.0 ** -6) * scale_of_elem * (1 + 2 ** -20)
    tol_n = 2.0 ** -4 * np.abs(x) * (1 + 2 ** -20)
    tol_s = 2.0 ** -10 * scale_of_elem.astype(np.float64) * (1 + 2 ** -20)
    assert np.all(err[normal] <= tol_n[normal])
    assert np.all(err[~normal] <= tol_s[~normal])
    assert normal.mean() > 0.9


def test_roundtrip_bound_rowwise_colwise_weight():
    x = S.bf16_normal((384, 640), 0, 105, 1.0, 1e-3, 50.0)
    f = f32_of(x)
    q, s = oracle.quantize_rowwise(x)
    _roundtrip_check(q, np.repeat(s.T, 128, axis=1)[:, :640], f)
    q_t, s_t = oracle.quantize_colwise(x)
    _roundtrip_check(q_t, np.repeat(s_t.T, 128, axis=1)[:, :384], f.T)
    w = S.bf16_normal((384, 640), 0, 106, 0.02)
    qw, sw, _ = oracle.quantize_weight_block(w)
    full = np.repeat(np.repeat(sw, 128, axis=0), 128, axis=1)[:384, :640]
    _roundtrip_check(qw, full, f32_of(w))


# ------------------------------------------------------------------ pow2 scales
# Power-of-two reading (the form B200 tensor cores apply in hardware): s = 2^E,
# E the smallest integer with 448 * 2^E >= amax, clamped to [-127, 127].

@pytest.mark.parametrize("name,vals,fill,codes,sbits",
                         hand_groups("quant_pow2_hand.txt"))
def test_pow2_hand_worked_group(name, vals, fill, codes, sbits):
    g = np.full(128, fill, dtype=np.float32)
    g[: len(vals)] = vals
    q, s = oracle.quantize_rowwise(bf16_bits(g)[None, :], pow2=True)
    assert q[0, : len(codes)].tolist() == codes, name
    assert s.view(np.uint32)[0, 0] == sbits, (name, hex(s.view(np.uint32)[0, 0]))


def _exact_pow2_exponent(amax):
    """Smallest integer E with 448 * 2^E >= amax, by exact rational
    arithmetic (independent of the oracle's binary64 search)."""
    from fractions import Fraction
    a = Fraction(float(amax))
    e = 0
    while Fraction(448) * Fraction(2) ** e < a:
        e += 1
    while Fraction(448) * Fraction(2) ** (e - 1) >= a:
        e -= 1
    return max(-127, min(127, e))


def test_pow2_scale_is_the_smallest_covering_power_of_two():
    rng = np.random.default_rng(7)
    # bf16 magnitudes spread over the whole exponent range, plus ties at 448*2^k
    bits = rng.integers(1, 0x7F80, 4000).astype(np.uint16)
    amaxes = list(f32_of(bits)) + [448.0 * 2.0 ** k for k in range(-40, 40)]
    for a in amaxes:
        qscale, s = oracle.group_scale(float(a), pow2=True)
        e = _exact_pow2_exponent(a)
        assert float(s) == 2.0 ** e and float(qscale) == 2.0 ** -e, a


def test_pow2_codes_match_an_independent_encoder():
    import torch
    x = S.bf16_normal((96, 640), 0, 111, 1.0, 1e-2, 50.0)
    q, s = oracle.quantize_rowwise(x, pow2=True)
    f = f32_of(x).reshape(96, 5, 128)
    inv = (1.0 / s.T.astype(np.float64)).astype(np.float32)[:, :, None]
    t = torch.from_numpy(np.ascontiguousarray(f * inv))   # exact: power of two
    ref = t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().reshape(96, 640)
    assert np.array_equal(q, ref)
    # the group's largest magnitude lands in (224, 448]
    amax = np.abs(f).max(axis=2) / s.T
    assert np.all((amax > 224) & (amax <= 448))


def test_pow2_layouts_agree():
    x = S.bf16_normal((272, 400), 0, 112, 1.0, 1e-3, 50.0)
    q_r, s_r = oracle.quantize_rowwise(np.ascontiguousarray(x.T), pow2=True)
    q_t, s_t = oracle.quantize_colwise(x, pow2=True)
    assert np.array_equal(q_r, q_t) and np.array_equal(s_r, s_t)
    w = S.bf16_normal((272, 400), 0, 113, **S.W_DIST)
    qw, sw, qw_t = oracle.quantize_weight_block(w, pow2=True)
    assert np.array_equal(qw_t, qw.T)
    fw = np.abs(f32_of(w))
    for nb in range(3):
        for kb in range(4):
            blk = fw[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            assert float(sw[nb, kb]) == 2.0 ** _exact_pow2_exponent(blk.max())
