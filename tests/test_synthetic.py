"""The seeded input generator (no method arithmetic): SplitMix64 pin,
determinism, and the value distributions of the workload recipes."""
import numpy as np

import synthetic as S


def test_splitmix64_published_first_output():
    # SplitMix64 started from state 0 first returns mix64(0x9E3779B97F4A7C15)
    # = 0xE220A8397B1DCDAF (Steele, Lea, Flood 2014; java.util.SplittableRandom).
    assert S.mix64(0x9E3779B97F4A7C15) == 0xE220A8397B1DCDAF


def test_deterministic_and_stream_independent():
    a = S.bf16_normal((64, 128), 0, 1, 1.0)
    b = S.bf16_normal((64, 128), 0, 1, 1.0)
    c = S.bf16_normal((64, 128), 0, 2, 1.0)
    d = S.bf16_normal((64, 128), 1, 1, 1.0)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)
    assert not np.array_equal(a, d)
    # counter based: a prefix of a longer draw equals the shorter draw
    e = S.bf16_normal((64 * 128 + 77,), 0, 1, 1.0)
    assert np.array_equal(e[: 64 * 128], a.ravel())


def _f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_normal_moments():
    x = _f32(S.bf16_normal((1 << 20,), 0, 7, 1.0))
    assert abs(x.mean()) < 5e-3
    assert abs(x.std() - 1.0) < 5e-3
    w = _f32(S.bf16_normal((1 << 20,), 0, 8, 0.02))
    assert abs(w.std() / 0.02 - 1.0) < 5e-3


def test_outlier_fraction_and_factor():
    n = 1 << 21
    base = _f32(S.bf16_normal((n,), 0, 9, 1.0))
    out = _f32(S.bf16_normal((n,), 0, 9, 1.0, 1e-3, 50.0))
    changed = base != out
    frac = changed.mean()
    assert 0.0008 < frac < 0.0012
    ratio = out[changed] / base[changed]
    assert np.all(np.abs(ratio - 50.0) < 50.0 * 2 ** -7)


def test_workload_shapes():
    wl = S.workload("stack28_m16384")
    assert len(wl) == 28 * 4
    total = sum(l.flops() for l in wl)
    assert total == 28 * 3 * 2 * 16384 * (2048 * 4096 + 2048 * 2048 +
                                          2048 * 12288 + 6144 * 2048)
    assert S.workload("qkv_fprop_m8192")[0].n == 4096
