"""Blockwise-FP8 (E4M3) training linear layer for B200 (sm_100a).

The computation lives in the CUDA library libfp8bw.so (C ABI in
include/fp8bw.h); `ops` is its thin Python binding. Importing `ops` loads the
library and raises if it is missing.
"""
__all__ = ["ops", "build"]
