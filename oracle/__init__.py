"""CPU oracle for the blockwise-FP8 training linear (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package. The library's product path never does.
"""
from .oracle import *  # noqa: F401,F403
