"""FP64 CPU oracle for the BCQ LUT-GEMM path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  See ``bcq_oracle`` for what it computes.
"""
from .bcq_oracle import *  # noqa: F401,F403
from .bcq_oracle import __all__  # noqa: F401
