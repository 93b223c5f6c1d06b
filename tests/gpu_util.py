"""Helpers for the GPU parity tests: device placement, padded (strided)
operands, canary guard bands and the acceptance check against the oracle.

Acceptance (the fused GEMM + ReLU of "Writing high-performance kernels in
TileLang", atlascloud.ai blog, section "Escribamos un GEMM", checks its kernel
with rtol = atol = 1e-2): for every element |c - ref| <= 1e-2 + 1e-2 |ref|,
and wherever |ref| > 1e-2 the sign of c equals the sign of ref (for ReLU
output: c > 0 wherever ref > 1e-2).  ReLU output must also be >= 0, never -0,
never NaN.
"""
from __future__ import annotations

import numpy as np
import torch

ATOL = 1e-2
RTOL = 1e-2
CANARY = 0x7BFF  # 65504: far from anything a ReLU GEMM of these inputs writes


def to_dev(x: torch.Tensor, ld: int | None = None, rows_pad: int = 0) -> torch.Tensor:
    """Copy a CPU fp16 matrix to the GPU with row stride `ld` (>= cols)."""
    r, c = x.shape
    ld = c if ld is None else ld
    buf = torch.full((r + rows_pad, ld), float("nan"), dtype=torch.float16, device="cuda")
    buf[:r, :c] = x.cuda()
    return buf[:r, :c]


def round8(n: int) -> int:
    return (n + 7) // 8 * 8


class GuardedOut:
    """An (M, N) output view inside a larger buffer filled with a canary, so
    that writes outside the M x N window can be detected."""

    def __init__(self, M: int, N: int, ld: int | None = None, pad_rows: int = 3,
                 pad_cols: int = 8):
        ld = round8(N + pad_cols) if ld is None else ld
        self.M, self.N, self.ld, self.pad_rows = M, N, ld, pad_rows
        self.buf = torch.empty((pad_rows + M + pad_rows, ld), dtype=torch.float16,
                               device="cuda")
        self.buf.view(torch.int16).fill_(CANARY)
        self.view = self.buf[pad_rows:pad_rows + M, :N]

    def untouched(self) -> bool:
        b = self.buf.view(torch.int16).cpu().numpy().view(np.uint16)
        mask = np.ones(b.shape, dtype=bool)
        mask[self.pad_rows:self.pad_rows + self.M, :self.N] = False
        return bool((b[mask] == CANARY).all())


def check_parity(c: np.ndarray, ref: np.ndarray, relu: bool, what: str = ""):
    """Assert the acceptance criterion; returns (max_abs_err, max_rel_err)."""
    c = np.asarray(c, dtype=np.float16)
    ref = np.asarray(ref, dtype=np.float16)
    assert c.shape == ref.shape, (what, c.shape, ref.shape)
    c64 = c.astype(np.float64)
    r64 = ref.astype(np.float64)
    assert not np.isnan(c64).any(), f"{what}: NaN in output"
    with np.errstate(invalid="ignore"):
        err = np.where(c64 == r64, 0.0, np.abs(c64 - r64))  # equal infinities count as equal
    bad = err > ATOL + RTOL * np.abs(r64)
    if bad.any():
        idx = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements out of "
                             f"tolerance; first {idx}: got {c[idx]!r}, want {ref[idx]!r}")
    big = np.abs(r64) > ATOL
    assert (np.sign(c64[big]) == np.sign(r64[big])).all(), f"{what}: sign pattern differs"
    if relu:
        assert (c64 >= 0).all(), f"{what}: negative ReLU output"
        assert not (c.view(np.uint16) == 0x8000).any(), f"{what}: -0 in ReLU output"
    rel = err / np.maximum(np.abs(r64), 1e-30)
    return float(err.max(initial=0.0)), float(rel[big].max(initial=0.0))


def dev_to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()
