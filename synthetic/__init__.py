"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

Holds no arithmetic of the FP8 method: it only draws bf16 tensors (raw uint16
bit patterns) from a counter-based SplitMix64 stream, and names the workloads
(shapes and value distributions of Qwen3-1.7B-shaped linears).
"""
from .gen import *  # noqa: F401,F403
from .workloads import *  # noqa: F401,F403
