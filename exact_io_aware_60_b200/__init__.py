"""Exact IO-aware tiled attention (FlashAttention forward and backward) for B200 (sm_100a).

The compute path is the C-ABI library ``libfa.so`` (declared in ``include/fa.h``) built
from ``csrc/``; :mod:`exact_io_aware_60_b200.fa` is the ctypes binding over it.  The
library is loaded on first use and a missing library raises: there is no fallback.
"""
__all__ = ["fa", "workloads"]
