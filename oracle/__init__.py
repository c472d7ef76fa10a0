"""CPU oracle for scaled_mm and its quantizers (test infrastructure only).

Only tests, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package.  The library does not depend on it.
"""
from .lq_oracle import *  # noqa: F401,F403
