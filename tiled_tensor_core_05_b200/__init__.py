"""fp16 GEMM with a fused ReLU epilogue for NVIDIA B200 (sm_100a).

The compute lives in ``libttc05.so`` (hand-written CUDA, C ABI declared in
``include/gemm_f16.h``).  The Python layer in ``ops.py`` only marshals
pointers, sizes and the current CUDA stream into that library; it never
computes anything itself and raises if the library is missing.

Importing this package does not load the library (so that ``workloads`` can be
used on machines without a GPU); the first call does.
"""
from __future__ import annotations

__all__ = ["gemm_relu_f16", "gemm_f16", "gemm_f16_ex", "gemm_bias_act_f16", "gemm_general",
           "lib"]


def __getattr__(name):
    if name in __all__:
        from . import ops
        return getattr(ops, name)
    raise AttributeError(name)
