"""Shared test helpers: tensor conversion, parity tolerance, sample points,
the hand-worked golden groups."""
import os

import numpy as np

import oracle


def bf16_np_to_torch(a, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def torch_bf16_to_np(t):
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(
        np.uint16)


def bf16_bits_to_f64(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(
        np.float32).astype(np.float64)


def ulp_bf16(v):
    """Spacing of bf16 at |v|: 2^(max(floor(log2|v|), -126) - 7); 2^-133 at 0."""
    v = np.abs(np.asarray(v, np.float64))
    e = np.full(v.shape, -126.0)
    nz = v > 0
    e[nz] = np.maximum(np.floor(np.log2(v[nz])), -126.0)
    return np.exp2(e - 7.0)


def gemm_tolerance(acc, bound):
    """Acceptance bound per output element: 1e-3 * sum_k |a_k b_k| (of the
    dequantised operands) plus one bf16 ulp of the exact value."""
    return 1e-3 * np.asarray(bound) + ulp_bf16(acc)


def assert_gemm_close(got_bits, acc, bound, what=""):
    got = bf16_bits_to_f64(got_bits)
    err = np.abs(got - acc)
    tol = gemm_tolerance(acc, bound)
    bad = ~(err <= tol)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            "%s: %d of %d elements outside tolerance; first %s: got %s ref %s "
            "tol %s" % (what, int(bad.sum()), bad.size, idx.tolist(),
                        got[bad][:5], np.asarray(acc)[bad][:5], tol[bad][:5]))


def ulp_f32(v):
    """Spacing of fp32 at |v|: 2^(max(floor(log2|v|), -126) - 23)."""
    v = np.abs(np.asarray(v, np.float64))
    e = np.full(v.shape, -126.0)
    nz = v > 0
    e[nz] = np.maximum(np.floor(np.log2(v[nz])), -126.0)
    return np.exp2(e - 23.0)


def assert_gemm_close_f32(got, ref, bound, what=""):
    """fp32 outputs: |got - ref| <= 1e-3 * sum_k |a_k b_k| + 1 fp32 ulp(ref)."""
    got = np.asarray(got, np.float64)
    err = np.abs(got - ref)
    tol = 1e-3 * np.asarray(bound) + ulp_f32(ref)
    bad = ~(err <= tol)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            "%s: %d of %d elements outside tolerance; first %s: got %s ref %s "
            "tol %s" % (what, int(bad.sum()), bad.size, idx.tolist(),
                        got[bad][:5], np.asarray(ref)[bad][:5], tol[bad][:5]))


def sample_points(rows, cols, seed=0, per_tile=16, stripes=2, tile=128):
    """At least `per_tile` seeded points in every 128x128 output tile, plus
    `stripes` full rows and full columns."""
    rng = np.random.default_rng(seed)
    pi, pj = [], []
    for r0 in range(0, rows, tile):
        for c0 in range(0, cols, tile):
            h = min(tile, rows - r0)
            w = min(tile, cols - c0)
            pi.append(r0 + rng.integers(0, h, per_tile))
            pj.append(c0 + rng.integers(0, w, per_tile))
    for r in rng.choice(rows, size=min(stripes, rows), replace=False):
        pi.append(np.full(cols, r))
        pj.append(np.arange(cols))
    for c in rng.choice(cols, size=min(stripes, cols), replace=False):
        pi.append(np.arange(rows))
        pj.append(np.full(rows, c))
    return (np.concatenate(pi).astype(np.int64),
            np.concatenate(pj).astype(np.int64))


def scale_bits(s):
    return np.ascontiguousarray(s, np.float32).view(np.uint32)


__all__ = ["bf16_np_to_torch", "torch_bf16_to_np", "bf16_bits_to_f64",
           "ulp_bf16", "gemm_tolerance", "assert_gemm_close", "ulp_f32",
           "assert_gemm_close_f32",
           "sample_points", "scale_bits", "oracle"]


GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def hand_groups(fname="quant_group_hand.txt"):
    """Rows of a hand-worked group file: (name, listed values, fill value,
    expected codes of the listed values, expected scale bits)."""
    rows = []
    with open(os.path.join(GOLDEN, fname)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, vals, fill, codes, sbits = [p.strip() for p in line.split("|")]
            ev = lambda e: float(eval(e, {"__builtins__": {}}))  # noqa: E731
            rows.append((name, [ev(v) for v in vals.split(",")], ev(fill),
                         [int(c, 16) for c in codes.split(",")],
                         int(sbits, 16)))
    return rows
