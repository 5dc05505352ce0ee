"""Pins of the oracle's three GEMMs (paperlayer.ai summary of the Puro-2B
report, Appendix C, "FP8 implementation pipeline": the E4M3 GEMMs are forward
propagation, data-gradient and weight-gradient).

  fprop  Y  = X W^T     groups of X along K, W in 128x128 blocks
  dgrad  dX = dY W      groups of dY along N, the same W blocks
  wgrad  dW = dY^T X    groups of dY and X along M (tokens)

Pins, none of which re-types the oracle's formula:
  * lossless inputs (every group's amax is 448*2^-j and every value lies on
    the E4M3 grid scaled by 2^-j): quantisation is exact, so the result must
    equal the exact product of the bf16 inputs, computed by numpy in fp64
    (exact here: every partial sum is a multiple of 2^-24 below 2^26);
  * brute force at 4x4x256 in exact rational arithmetic (fractions);
  * a hand-worked one-chunk product;
  * numpy fp64 matmul of the dequantised operands at ragged sizes.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synthetic as S

DEC = None


def dec():
    global DEC
    if DEC is None:
        DEC = oracle.e4m3_decode_table()
    return DEC


def f32_of(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def to_bf16(f):
    u = np.asarray(f, np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0)
    return (u >> 16).astype(np.uint16)


# ------------------------------------------------------------ lossless inputs

def lossless(shape, group_of, rng):
    """Values on the E4M3 grid times 2^-j(g), with one +-448*2^-j(g) per group.

    group_of(i, j) -> group index arrays (numpy broadcasting)."""
    mags = dec()[:0x7F]                      # finite non-negative magnitudes
    ii, jj = np.meshgrid(np.arange(shape[0]), np.arange(shape[1]),
                         indexing="ij")
    gid = group_of(ii, jj)
    ng = int(gid.max()) + 1
    exps = rng.integers(-3, 4, size=ng)      # per-group power of two
    v = rng.choice(mags[:0x7E], size=shape) * rng.choice([-1.0, 1.0],
                                                          size=shape)
    v = v * np.exp2(-exps[gid].astype(np.float64))
    # put one +-448*2^-j in every group
    flat_g = gid.ravel()
    first = np.unique(flat_g, return_index=True)[1]
    vf = v.ravel()
    vf[first] = 448.0 * np.exp2(-exps[flat_g[first]].astype(np.float64)) * \
        rng.choice([-1.0, 1.0], size=first.size)
    v = vf.reshape(shape).astype(np.float32)
    return to_bf16(v)


def rowgroups(ii, jj):     # 1x128 groups along the second index
    return ii * 10_000 + jj // 128


def colgroups(ii, jj):     # 128x1 groups along the first index
    return jj * 10_000 + ii // 128


def blocks(ii, jj):
    return (ii // 128) * 1000 + jj // 128


def _compact(g):
    return np.unique(g, return_inverse=True)[1].reshape(g.shape)


def grp(fn):
    return lambda ii, jj: _compact(fn(ii, jj))


@pytest.mark.parametrize("m,n,k", [(128, 256, 384), (64, 200, 300)])
def test_lossless_fprop_equals_exact_product(m, n, k):
    rng = np.random.default_rng(10)
    x = lossless((m, k), grp(rowgroups), rng)
    w = lossless((n, k), grp(blocks), rng)
    qx, sx = oracle.quantize_rowwise(x)
    qw, sw, _ = oracle.quantize_weight_block(w)
    # quantisation really is lossless
    assert np.array_equal(dec()[qx] * np.repeat(sx.T, 128, 1)[:, :k],
                          f32_of(x).astype(np.float64))
    y = oracle.gemm_fprop(qx, sx, qw, sw)
    exact = f32_of(x).astype(np.float64) @ f32_of(w).astype(np.float64).T
    assert np.array_equal(y, exact)


@pytest.mark.parametrize("m,n,k", [(128, 384, 256), (96, 300, 200)])
def test_lossless_dgrad_equals_exact_product(m, n, k):
    rng = np.random.default_rng(11)
    dy = lossless((m, n), grp(rowgroups), rng)
    w = lossless((n, k), grp(blocks), rng)
    qdy, sdy = oracle.quantize_rowwise(dy)
    qw, sw, _ = oracle.quantize_weight_block(w)
    dx = oracle.gemm_dgrad(qdy, sdy, qw, sw)
    exact = f32_of(dy).astype(np.float64) @ f32_of(w).astype(np.float64)
    assert np.array_equal(dx, exact)


@pytest.mark.parametrize("m,n,k", [(384, 256, 128), (300, 100, 200)])
def test_lossless_wgrad_equals_exact_product(m, n, k):
    rng = np.random.default_rng(12)
    dy = lossless((m, n), grp(colgroups), rng)
    x = lossless((m, k), grp(colgroups), rng)
    qdy_t, sdy_t = oracle.quantize_colwise(dy)
    qx_t, sx_t = oracle.quantize_colwise(x)
    dw = oracle.gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t)
    exact = f32_of(dy).astype(np.float64).T @ f32_of(x).astype(np.float64)
    assert np.array_equal(dw, exact)


# ------------------------------------------------------------ brute force

def _exact(a_codes, a_scale, b_codes, b_scale):
    """sum_k (q_a*s_a)*(q_b*s_b) in exact rationals, one output element."""
    total = Fraction(0)
    for qa, sa, qb, sb in zip(a_codes, a_scale, b_codes, b_scale):
        total += (Fraction(float(dec()[qa])) * Fraction(float(sa)) *
                  Fraction(float(dec()[qb])) * Fraction(float(sb)))
    return total


def test_bruteforce_4x4x256_all_roles():
    M = N = 4
    K = 256
    x = S.bf16_normal((M, K), 0, 201, 1.0, 0.05, 50.0)
    w = S.bf16_normal((N, K), 0, 202, 0.02)
    qx, sx = oracle.quantize_rowwise(x)
    qw, sw, _ = oracle.quantize_weight_block(w)
    y, yb = oracle.gemm_fprop(qx, sx, qw, sw, with_bound=True)
    for i in range(M):
        for j in range(N):
            ex = _exact(qx[i], [sx[c // 128, i] for c in range(K)],
                        qw[j], [sw[j // 128, c // 128] for c in range(K)])
            assert abs(y[i, j] - float(ex)) <= 2.0 ** -50 * yb[i, j]

    # dgrad: dY [4, 256] (contract over N=256), W [256, 4]
    dy = S.bf16_normal((4, 256), 0, 203, 1e-3, 0.05, 100.0)
    w2 = S.bf16_normal((256, 4), 0, 204, 0.02)
    qdy, sdy = oracle.quantize_rowwise(dy)
    qw2, sw2, _ = oracle.quantize_weight_block(w2)
    dx, dxb = oracle.gemm_dgrad(qdy, sdy, qw2, sw2, with_bound=True)
    for i in range(4):
        for j in range(4):
            ex = _exact(qdy[i], [sdy[c // 128, i] for c in range(256)],
                        qw2[:, j], [sw2[c // 128, j // 128] for c in range(256)])
            assert abs(dx[i, j] - float(ex)) <= 2.0 ** -50 * dxb[i, j]

    # wgrad: dY [256, 4], X [256, 4] (contract over M=256)
    dy3 = S.bf16_normal((256, 4), 0, 205, 1e-3, 0.05, 100.0)
    x3 = S.bf16_normal((256, 4), 0, 206, 1.0, 0.05, 50.0)
    qdy_t, sdy_t = oracle.quantize_colwise(dy3)
    qx_t, sx_t = oracle.quantize_colwise(x3)
    dw, dwb = oracle.gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t, with_bound=True)
    for i in range(4):
        for j in range(4):
            ex = _exact(qdy_t[i], [sdy_t[c // 128, i] for c in range(256)],
                        qx_t[j], [sx_t[c // 128, j] for c in range(256)])
            assert abs(dw[i, j] - float(ex)) <= 2.0 ** -50 * dwb[i, j]


def test_hand_worked_single_chunk():
    # X row = 128 ones, W row = 128 ones: amax 1 -> qscale 448, codes 0x7E,
    # s = fl(1/448); Y = 128 * (448 * fl(1/448))^2 = 128 (1 + O(2^-23)),
    # which rounds to bf16 128.0 = 0x4300.
    ones = np.full((1, 128), 0x3F80, np.uint16)
    qx, sx = oracle.quantize_rowwise(ones)
    qw, sw, _ = oracle.quantize_weight_block(ones)
    assert np.all(qx == 0x7E) and np.all(qw == 0x7E)
    y, b = oracle.gemm_fprop(qx, sx, qw, sw, with_bound=True)
    s = float(np.float32(1.0) / np.float32(448.0))
    assert y[0, 0] == 128 * (448 * s) ** 2
    assert abs(y[0, 0] - 128.0) < 128 * 2 ** -21
    assert b[0, 0] == y[0, 0]
    assert oracle.bf16_round(y)[0, 0] == 0x4300


# ------------------------------------------------------------ numpy cross-check

def _deq_rows(q, s, L):        # 1xL groups along axis 1, s [G][rows]
    return dec()[q] * np.repeat(s.T.astype(np.float64), 128, 1)[:, :L]


def test_dequantise_then_matmul_ragged():
    m, n, k = 200, 300, 400
    x = S.bf16_normal((m, k), 0, 301, 1.0, 1e-2, 50.0)
    w = S.bf16_normal((n, k), 0, 302, 0.02)
    dy = S.bf16_normal((m, n), 0, 303, 1e-3, 1e-2, 100.0)
    qx, sx = oracle.quantize_rowwise(x)
    qw, sw, _ = oracle.quantize_weight_block(w)
    wfull = dec()[qw] * np.repeat(np.repeat(sw.astype(np.float64), 128, 0),
                                  128, 1)[:n, :k]
    y, yb = oracle.gemm_fprop(qx, sx, qw, sw, with_bound=True)
    ref = _deq_rows(qx, sx, k) @ wfull.T
    assert np.all(np.abs(y - ref) <= 1e-12 * yb + 1e-300)
    assert np.allclose(yb, np.abs(_deq_rows(qx, sx, k)) @ np.abs(wfull).T,
                       rtol=1e-12, atol=0)

    qdy, sdy = oracle.quantize_rowwise(dy)
    dx, dxb = oracle.gemm_dgrad(qdy, sdy, qw, sw, with_bound=True)
    ref = _deq_rows(qdy, sdy, n) @ wfull
    assert np.all(np.abs(dx - ref) <= 1e-12 * dxb + 1e-300)

    qdy_t, sdy_t = oracle.quantize_colwise(dy)
    qx_t, sx_t = oracle.quantize_colwise(x)
    dw, dwb = oracle.gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t, with_bound=True)
    ref = _deq_rows(qdy_t, sdy_t, m) @ _deq_rows(qx_t, sx_t, m).T
    assert np.all(np.abs(dw - ref) <= 1e-12 * dwb + 1e-300)


def test_points_and_threads_agree_with_full():
    m, n, k = 256, 384, 512
    x = S.bf16_normal((m, k), 0, 401, 1.0, 1e-2, 50.0)
    w = S.bf16_normal((n, k), 0, 402, 0.02)
    qx, sx = oracle.quantize_rowwise(x)
    qw, sw, _ = oracle.quantize_weight_block(w)
    y1, b1 = oracle.gemm_fprop(qx, sx, qw, sw, with_bound=True, nthreads=1)
    y8 = oracle.gemm_fprop(qx, sx, qw, sw, nthreads=8)
    assert np.array_equal(y1, y8)
    rng = np.random.default_rng(0)
    pi = rng.integers(0, m, 500)
    pj = rng.integers(0, n, 500)
    pa, pb = oracle.gemm_fprop_points(qx, sx, qw, sw, pi, pj)
    assert np.array_equal(pa, y1[pi, pj]) and np.array_equal(pb, b1[pi, pj])
    with pytest.raises(ValueError):
        oracle.gemm_fprop_points(qx, sx, qw, sw, [m], [0])
