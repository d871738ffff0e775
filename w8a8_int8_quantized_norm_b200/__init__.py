"""SmoothQuant W8A8 linear layer for NVIDIA B200 (sm_100a).

The compute lives in the CUDA library ``libsq.so`` (built from ``csrc/``) behind
the C ABI declared in ``include/sq.h``; :mod:`.sq` is the thin ctypes binding
that marshals torch tensors into that ABI.  :mod:`.synthetic` draws the seeded
workload inputs.  Importing the package loads nothing; the binding loads the
library on first use and raises if it is missing.
"""
__all__ = ["sq", "synthetic"]
