"""B200-native Lighthouse Attention hot path.

The compute lives in ``liblh.so`` (hand-written sm_100a CUDA kernels behind a
C ABI declared in ``include/lh.h``); ``long_context_symmetric_b200.lh`` is the
thin ctypes binding over it. Importing the package does not load the library;
the first call into the binding does, and raises if it is missing.
"""

__all__ = ["lh", "synth"]
