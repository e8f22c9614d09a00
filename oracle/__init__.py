"""Independent double-precision CPU oracle (test infrastructure, not the product).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  It shares no code with the CUDA path.
"""
from .spark_oracle import *  # noqa: F401,F403
