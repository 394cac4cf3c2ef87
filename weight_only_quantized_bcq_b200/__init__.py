"""B200-native LUT-GEMM for binary-coding-quantised (BCQ) weights.

The compute path is the C-ABI library ``liblutgemm.so`` (hand-written sm_100a
CUDA, declared in ``include/lutgemm.h``).  This package is a thin binding over
it: ``lutgemm`` marshals torch device tensors into the C calls, nothing more.
"""
from .roofline import algorithmic_bytes, bits_per_weight, lookups  # noqa: F401

__all__ = ["algorithmic_bytes", "bits_per_weight", "lookups"]
