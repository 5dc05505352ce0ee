"""Workload recipes: Qwen3-1.7B-shaped linears (hidden 2048, ffn 6144, 16 query
and 8 key/value heads of 128), tokens M = micro-batch x 4096.

Each linear has X [M, K] (tokens x in), W [N, K] (out x in) and dY [M, N].
Value distributions: X ~ N(0, 1) with 0.1% of entries x50, W ~ N(0, 0.02),
dY ~ N(0, 1e-3) with 0.1% of entries x100 (the single-GEMM 256^3 case draws
X without outliers). Seed 0 everywhere; each tensor has its own id so every
tensor is an independent stream.
"""
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np

from .gen import bf16_normal

__all__ = ["LINEARS", "Linear", "WORKLOADS", "workload", "tensor_id",
           "draw_x", "draw_w", "draw_dy", "X_DIST", "X_DIST_PLAIN", "W_DIST",
           "DY_DIST", "gemm_flops"]

# kind -> (K = in_features, N = out_features)
LINEARS = {
    "qkv": (2048, 4096),       # 16 q + 8 k + 8 v heads x 128
    "o": (2048, 2048),
    "gate_up": (2048, 12288),  # fused gate and up projections (2 x 6144)
    "down": (6144, 2048),
}
_KIND_INDEX = {"qkv": 0, "o": 1, "gate_up": 2, "down": 3}
_ROLE_INDEX = {"x": 1, "w": 2, "dy": 3}

X_DIST = dict(std=1.0, outlier_p=1e-3, outlier_factor=50.0)
X_DIST_PLAIN = dict(std=1.0, outlier_p=0.0, outlier_factor=1.0)
W_DIST = dict(std=0.02, outlier_p=0.0, outlier_factor=1.0)
DY_DIST = dict(std=1e-3, outlier_p=1e-3, outlier_factor=100.0)


def tensor_id(kind: str, role: str, layer: Optional[int] = None) -> int:
    base = 10 * _KIND_INDEX[kind] + _ROLE_INDEX[role]
    return base if layer is None else 1000 * (layer + 1) + base


@dataclass
class Linear:
    kind: str
    m: int
    k: int
    n: int
    ops: Tuple[str, ...]              # subset of ("fprop", "dgrad", "wgrad")
    layer: Optional[int] = None
    x_dist: dict = field(default_factory=lambda: dict(X_DIST))

    def flops(self) -> int:
        return 2 * self.m * self.n * self.k * len(self.ops)


def gemm_flops(lin: Linear) -> int:
    return lin.flops()


def draw_x(lin: Linear, seed: int = 0) -> np.ndarray:
    return bf16_normal((lin.m, lin.k), seed,
                       tensor_id(lin.kind, "x", lin.layer), **lin.x_dist)


def draw_w(lin: Linear, seed: int = 0) -> np.ndarray:
    return bf16_normal((lin.n, lin.k), seed,
                       tensor_id(lin.kind, "w", lin.layer), **W_DIST)


def draw_dy(lin: Linear, seed: int = 0) -> np.ndarray:
    return bf16_normal((lin.m, lin.n), seed,
                       tensor_id(lin.kind, "dy", lin.layer), **DY_DIST)


def _stack(m: int, layers: int) -> List[Linear]:
    out = []
    for layer in range(layers):
        for kind in ("qkv", "o", "gate_up", "down"):
            k, n = LINEARS[kind]
            out.append(Linear(kind, m, k, n, ("fprop", "dgrad", "wgrad"),
                              layer))
    return out


# name -> list of linears. Names describe the workload and its sizes.
WORKLOADS = {
    "fprop_256x256x256": [
        Linear("qkv", 256, 256, 256, ("fprop",), None, dict(X_DIST_PLAIN))],
    "qkv_fprop_m8192": [
        Linear("qkv", 8192, 2048, 4096, ("fprop",))],
    "mlp_fprop_m16384": [
        Linear("gate_up", 16384, 2048, 12288, ("fprop",)),
        Linear("down", 16384, 6144, 2048, ("fprop",))],
    "mlp_backward_m16384": [
        Linear("down", 16384, 6144, 2048, ("dgrad", "wgrad")),
        Linear("gate_up", 16384, 2048, 12288, ("dgrad", "wgrad"))],
    "stack28_m16384": _stack(16384, 28),
}


def workload(name: str) -> List[Linear]:
    return WORKLOADS[name]
