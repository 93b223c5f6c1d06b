"""Seeded synthetic inputs for the fp16 GEMM(+ReLU) workloads.

This module only draws random numbers: it holds none of the GEMM arithmetic,
so both the CUDA path and the CPU oracle can take their inputs from it.

Recipe (the same on every machine, because it runs on the CPU generator):
``torch.Generator('cpu').manual_seed(seed)``; A is drawn first, then B, each
as ``torch.randn`` in fp32, multiplied by its scale in fp32 and cast to fp16
with round-to-nearest-even.  Everything is row-major and contiguous.

The shapes and distributions are the workloads named for the fused GEMM+ReLU
in "Writing high-performance kernels in TileLang" (atlascloud.ai blog, section
"Escribamos un GEMM": ``torch.randn`` fp16 at M = N = K = 1024) widened to the
compute-bound cube, an MLP up-projection and a decode-shaped skinny product.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    N: int
    K: int
    seed: int
    a_scale: float
    b_scale: float
    description: str

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K

    @property
    def bytes_min(self) -> int:
        """A and B read once and C written once, fp16."""
        return 2 * (self.M * self.K + self.K * self.N + self.M * self.N)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("cube256", 256, 256, 256, 0, 1.0, 1.0,
                 "M=N=K=256, A,B ~ N(0,1), seed 0"),
        Workload("cube1024", 1024, 1024, 1024, 1, 1.0, 1.0,
                 "M=N=K=1024, A,B ~ N(0,1), seed 1"),
        Workload("ragged1000", 1000, 1000, 1000, 1, 1.0, 1.0,
                 "M=N=K=1000 (ragged edges), A,B ~ N(0,1), seed 1"),
        Workload("cube8192", 8192, 8192, 8192, 2, 1.0 / math.sqrt(8192), 1.0 / math.sqrt(8192),
                 "M=N=K=8192, A,B ~ N(0,1)/sqrt(K), seed 2 (tensor-pipe bound)"),
        Workload("mlp_up", 8192, 14336, 4096, 3, 1.0, 0.02,
                 "MLP up-projection M=8192 tokens, K=4096, N=14336; A ~ N(0,1), "
                 "B ~ N(0, 0.02^2), seed 3"),
        Workload("decode", 32, 28672, 8192, 4, 1.0, 0.02,
                 "decode-shaped M=32, K=8192, N=28672; A ~ N(0,1), B ~ N(0, 0.02^2), "
                 "seed 4 (HBM bound on B)"),
        # further small-M shapes (the configuration sweep's; few column tiles)
        Workload("decode_n4096", 32, 4096, 8192, 5, 1.0, 0.02,
                 "M=32, K=8192, N=4096; A ~ N(0,1), B ~ N(0, 0.02^2), seed 5"),
        Workload("decode_m16_n8192_k4096", 16, 8192, 4096, 6, 1.0, 0.02,
                 "M=16, K=4096, N=8192; A ~ N(0,1), B ~ N(0, 0.02^2), seed 6"),
        Workload("decode_m64_n2048_k8192", 64, 2048, 8192, 7, 1.0, 0.02,
                 "M=64, K=8192, N=2048; A ~ N(0,1), B ~ N(0, 0.02^2), seed 7"),
        Workload("decode_n1024_k16384", 32, 1024, 16384, 8, 1.0, 0.02,
                 "M=32, K=16384, N=1024; A ~ N(0,1), B ~ N(0, 0.02^2), seed 8"),
        Workload("decode_n14336_k4096", 32, 14336, 4096, 9, 1.0, 0.02,
                 "M=32, K=4096, N=14336; A ~ N(0,1), B ~ N(0, 0.02^2), seed 9"),
    ]
}


def randn_f16(shape, generator: torch.Generator, scale: float = 1.0) -> torch.Tensor:
    """fp16 CPU tensor of N(0, scale^2) draws (fp32 draw, fp32 scale, RNE cast)."""
    x = torch.randn(*shape, generator=generator, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(torch.float16)


def make_inputs(M: int, N: int, K: int, seed: int, a_scale: float = 1.0,
                b_scale: float = 1.0):
    """Return (A, B) as contiguous fp16 CPU tensors of shapes (M, K), (K, N)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    a = randn_f16((M, K), g, a_scale)
    b = randn_f16((K, N), g, b_scale)
    return a, b


def workload_inputs(name: str):
    """(A, B) for one of the named workloads."""
    w = WORKLOADS[name]
    return make_inputs(w.M, w.N, w.K, w.seed, w.a_scale, w.b_scale)
