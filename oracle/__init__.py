"""fp64 CPU oracle for the DP-SGD per-sample clip + sum + noise step (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and reference
legs may import this package.  The CUDA library never does, and it shares no code with it.
"""
from .dp_oracle import *  # noqa: F401,F403
from .dp_oracle import __all__  # noqa: F401
