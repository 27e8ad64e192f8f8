"""DSpark per-step speculative-decoding hot path for B200 (sm_100a).

The compute lives in libdspark.so (C ABI: include/dspark.h); this package
holds its ctypes binding (``dspark``), the in-tree build (``build``), a
step runner (``step``) and the seeded synthetic workloads (``workloads``).
Importing the package does not load the CUDA library; the first binding
call does, and fails loudly if it is missing.
"""
__all__ = ["build", "dspark", "step", "workloads"]
