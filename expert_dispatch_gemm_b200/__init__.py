"""B200-native MoE routing-and-dispatch layer (sm_100a).

The compute lives in ``libmoe.so`` (hand-written CUDA behind a C ABI, see
``include/moe.h``); ``expert_dispatch_gemm_b200.moe`` is the thin ctypes
binding over torch-allocated device memory. Importing this package does not
load the library; the binding loads it on first use and raises if it is
missing.
"""
__all__ = ["moe", "workloads"]
