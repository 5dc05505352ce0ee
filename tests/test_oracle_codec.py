"""Pins of the oracle's E4M3 codec and bf16 rounding against things other than
itself: torch's float8_e4m3fn / bfloat16 conversions (library routines of the
same formats) and the hand-worked cases in tests/golden/e4m3_encode_hand.txt.
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_decode_all_256_codes_match_torch_float8_e4m3fn():
    ours = oracle.e4m3_decode_table()
    ref = torch.arange(256, dtype=torch.uint8).view(
        torch.float8_e4m3fn).to(torch.float64).numpy()
    nan_ours = np.isnan(ours)
    assert np.array_equal(nan_ours, np.isnan(ref))
    assert set(np.nonzero(nan_ours)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan_ours], ref[~nan_ours])
    assert ours[0x7E] == 448.0 and ours[0x08] == 2.0 ** -6
    assert ours[0x01] == 2.0 ** -9


def _torch_encode(f32):
    return torch.from_numpy(f32).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def test_encode_all_bf16_patterns_match_torch():
    # Every bf16 bit pattern as an fp32 input. torch's cast is round-to-
    # nearest-even but not saturating (it gives NaN above 464), so compare
    # where |t| <= 464 and check saturation separately.
    f = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    keep = np.isfinite(f) & (np.abs(f) <= 464.0)
    f = f[keep]
    assert np.array_equal(oracle.e4m3_encode(f), _torch_encode(f))


def test_encode_random_fp32_patterns_match_torch():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 2 ** 32, size=2_000_000, dtype=np.uint64)
    f = bits.astype(np.uint32).view(np.float32)
    keep = np.isfinite(f) & (np.abs(f) <= 464.0)
    f = f[keep]
    assert f.size > 500_000
    assert np.array_equal(oracle.e4m3_encode(f), _torch_encode(f))


def test_encode_every_fp32_in_the_rounding_range_matches_torch():
    # Every fp32 bit pattern with 2^-12 <= |t| <= 464, both signs: all the
    # rounding decisions of the format (the smallest one is at 2^-10).
    # Below 2^-12 every value must give a signed zero.
    lo = int(np.float32(2.0 ** -12).view(np.uint32))
    hi = int(np.float32(464.0).view(np.uint32))
    step = 1 << 24
    for start in range(lo, hi + 1, step):
        bits = np.arange(start, min(start + step, hi + 1), dtype=np.uint32)
        for sign in (0, 0x80000000):
            f = (bits | np.uint32(sign)).view(np.float32)
            assert np.array_equal(oracle.e4m3_encode(f), _torch_encode(f)), \
                hex(start | sign)
    tiny = np.arange(0, lo, 997, dtype=np.uint32)
    for sign, code in ((0, 0x00), (0x80000000, 0x80)):
        f = (tiny | np.uint32(sign)).view(np.float32)
        assert np.all(oracle.e4m3_encode(f) == code)


def test_encode_midpoints_and_neighbours_match_torch():
    # All midpoints between adjacent E4M3 magnitudes, and the fp32 values one
    # ulp either side of each: the rounding decision points.
    mags = torch.arange(0, 0x7F, dtype=torch.uint8).view(
        torch.float8_e4m3fn).to(torch.float64).numpy()
    mids = ((mags[:-1] + mags[1:]) / 2).astype(np.float32)
    pts = np.concatenate([mids, np.nextafter(mids, np.float32(0)),
                          np.nextafter(mids, np.float32(1e9)),
                          mags.astype(np.float32)])
    pts = np.concatenate([pts, -pts]).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(pts), _torch_encode(pts))


def _load_hand_cases():
    cases = []
    with open(os.path.join(GOLDEN, "e4m3_encode_hand.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            expr, code, _why = [p.strip() for p in line.split("|")]
            cases.append((float(eval(expr, {"__builtins__": {}})),
                          int(code, 16)))
    return cases


@pytest.mark.parametrize("value,code", _load_hand_cases())
def test_encode_hand_worked(value, code):
    got = int(oracle.e4m3_encode(np.array([value], dtype=np.float32))[0])
    assert got == code, (value, hex(got), hex(code))


def test_encode_saturates_above_range():
    big = np.array([448.0, 450.0, 463.9, 464.0, 464.1, 479.0, 480.0, 1e6,
                    3.4e38, np.inf], dtype=np.float32)
    assert np.all(oracle.e4m3_encode(big) == 0x7E)
    assert np.all(oracle.e4m3_encode(-big) == 0xFE)


def test_bf16_round_matches_torch_on_fp32_values():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2 ** 32, size=200_000, dtype=np.uint64)
    f = bits.astype(np.uint32).view(np.float32)
    f = f[np.isfinite(f) & (np.abs(f) < 3.38e38)]
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy()
    ours = oracle.bf16_round(f.astype(np.float64))
    assert np.array_equal(ours.view(np.int16), ref)


def test_bf16_round_hand_worked():
    # 1 + 2^-8 is the midpoint of 1 and 1 + 2^-7: ties to even -> 1.0 (0x3F80)
    # 1 + 3*2^-8 is the midpoint of 1+2^-7 (odd) and 1+2^-6 (even) -> 0x3F82
    # 128*(1+2^-23) -> 128 (0x4300); -2.0 -> 0xC000
    vals = [1 + 2 ** -8, 1 + 3 * 2 ** -8, 128 * (1 + 2 ** -23), -2.0, 0.0]
    assert oracle.bf16_round(vals).tolist() == [0x3F80, 0x3F82, 0x4300,
                                                 0xC000, 0x0000]
