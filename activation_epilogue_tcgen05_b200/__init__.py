"""Fused GEMM + bias + ReLU/GELU (+ packed ReLU sign mask, + FP8 scales) for B200.

The compute path is the C-ABI CUDA library ``libgemm_epi.so`` (sm_100a, built by
``activation_epilogue_tcgen05_b200.build``); ``gemm_epi`` is its ctypes
binding.  Importing this package loads nothing: the library is opened on the
first call that needs it and raises if it is missing.
"""
__all__ = ["gemm_epi", "workloads", "build"]
