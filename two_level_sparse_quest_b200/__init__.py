"""B200-native two-level sparse decode attention (AsyncTLS hot path).

Submodules:
  * ``tls``       -- ctypes binding of the C-ABI library ``libtls.so`` (loaded on first use).
  * ``workloads`` -- seeded synthetic decode workloads.
  * ``build``     -- nvcc build of ``libtls.so`` for sm_100a.

Importing the package loads nothing; ``from two_level_sparse_quest_b200 import tls``
loads the CUDA library and raises if it is missing.
"""
__all__ = ["tls", "workloads", "build"]
