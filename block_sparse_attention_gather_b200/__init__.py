"""B200 (sm_100a) Spark-Attn two-branch block-sparse attention forward.

The compute lives in ``libspark_bsa.so`` (hand-written CUDA for sm_100a, C ABI declared in
``include/spark_bsa.h``); this package is its ctypes binding plus the seeded input
generators.  The library is loaded on first use and its absence is an error: there is no
CPU or PyTorch fallback.
"""
from ._native import *  # noqa: F401,F403
from ._native import EXPORTED, lib  # noqa: F401
