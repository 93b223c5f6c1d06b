"""fp16 GEMM with a fused ReLU (or bias + GELU) epilogue for NVIDIA B200 (sm_100a).

The compute lives in ``libttc05.so`` (hand-written CUDA, C ABI declared in
``include/gemm_f16.h``).  The Python layer in ``ops.py`` only marshals
pointers, sizes and the current CUDA stream into that library; it never
computes anything itself and raises if the library is missing.

    from tiled_tensor_core_05_b200 import gemm_relu_f16, gemm_bias_act_f16
    c = gemm_relu_f16(a, b)                        # ReLU(a @ b), a (M, K), b (K, N) fp16
    y = gemm_bias_act_f16(x, w, bias, "gelu")      # GELU(x @ w + bias)
    z = gemm_general(x, w_nk, bias, "relu", trans_b=True)  # w stored N x K
    c_host = gemm_host(a_cpu, b_cpu)               # CPU tensors in and out, copies pipelined

``tune`` is the offline configuration sweep (``python -m
tiled_tensor_core_05_b200.tune``), ``shard`` the column-sharded product across
ranks, ``build`` compiles the library in-tree.

Importing this package does not load the library (so that ``workloads`` can be
used on machines without a GPU); the first call does.
"""
from __future__ import annotations

__all__ = ["gemm_relu_f16", "gemm_f16", "gemm_f16_ex", "gemm_bias_act_f16", "gemm_general",
           "gemm_config_run", "GemmConfig", "auto_config", "config_list", "config_smem_bytes",
           "activation_f32", "read_probe", "select_path", "device_status", "status_string",
           "gemm_host", "host_plan", "host_release", "lib"]


def __getattr__(name):
    if name in __all__:
        from . import ops
        return getattr(ops, name)
    raise AttributeError(name)
