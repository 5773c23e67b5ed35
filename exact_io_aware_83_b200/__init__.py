"""B200-native exact attention (online-softmax forward, recomputing backward).

The compute path is the C-ABI library ``libfa_sm100.so`` built from ``csrc/``; the
Python binding in :mod:`exact_io_aware_83_b200.fa` only marshals pointers and streams.
Nothing is loaded at import time, so host-only modules (``inputs``) stay importable on a
machine without a GPU; the binding raises when the library is missing.
"""

__all__ = ["fa", "inputs"]
