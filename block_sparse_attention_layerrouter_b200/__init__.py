"""Layer-routed hybrid attention (full / 64-token block-sparse) for B200.

The compute lives in a C-ABI shared library of hand-written sm_100a CUDA
kernels (``csrc/``, declared in ``include/fa_hybrid.h``).  ``capi`` is the thin
ctypes binding with the same entry-point names; ``inputs`` draws seeded
synthetic workloads.  Importing this package loads nothing; the library is
loaded on the first call into ``capi`` and the call fails loudly if the
library is missing.
"""
__all__ = ["capi", "inputs"]
