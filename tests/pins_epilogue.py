"""Pins for a fused bias + activation GEMM epilogue: act(A @ B + bias).

The epilogue is the one of "TileLang simplifica la creación de kernels GPU de
alto rendimiento" (posicionamiento-web.ar), section "Fusionar operaciones para
reducir viajes a memoria": bias added and GELU applied to the accumulator
before the single write.  Read as a per-column fp16 bias and the exact GELU,
x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2)).

Each ``pin_*`` takes ``fn(a, b, bias, act) -> float16 (M, N)`` with numpy
float16 inputs (bias: length-N float16 or None; act: "none" | "relu" | "gelu")
and returns a list of failures.  ``exact=True`` compares bits; ``exact=False``
(fp32 accumulation on the GPU) compares within |c - ref| <= 1e-2 + 1e-2 |ref|
where the answer is not exact in fp32.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import torch

from pins import fraction_to_f16_bits, within_tol


def gelu64(x: np.ndarray) -> np.ndarray:
    """torch's exact (erf) GELU in fp64: a library routine with the same
    definition, independent of the oracle's own code."""
    return torch.nn.functional.gelu(torch.from_numpy(np.asarray(x, dtype=np.float64)),
                                    approximate="none").numpy()


def act64(x, act):
    x = np.asarray(x, dtype=np.float64)
    if act == "relu":
        return np.where(x > 0, x, 0.0)
    if act == "gelu":
        return gelu64(x)
    return x


def to_f16_bits(x64: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return np.asarray(x64, dtype=np.float64).astype(np.float16).view(np.uint16)


def _cmp(name, got, want_bits, exact, fails, strict_zero=True):
    got = np.asarray(got, dtype=np.float16)
    want_bits = np.asarray(want_bits, dtype=np.uint16)
    if got.shape != want_bits.shape:
        fails.append(f"{name}: shape {got.shape} vs {want_bits.shape}")
        return
    if exact:
        gb, wb = got.view(np.uint16), want_bits
        if not strict_zero:
            gb = np.where(gb == 0x8000, 0, gb)
            wb = np.where(wb == 0x8000, 0, wb)
        bad = gb != wb
        if bad.any():
            i = tuple(np.argwhere(bad)[0])
            fails.append(f"{name}: {int(bad.sum())} bit mismatches, first {i}: got "
                         f"{got[i]!r} want {want_bits[i].view(np.float16)!r}")
    else:
        ok = within_tol(got, want_bits.view(np.float16))
        if not ok.all():
            i = tuple(np.argwhere(~ok)[0])
            fails.append(f"{name}: {int((~ok).sum())} out of tolerance, first {i}: got "
                         f"{got[i]!r} want {want_bits[i].view(np.float16)!r}")


def _r16(rng, shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float16)


def pin_bias_broadcast(fn, exact=True, m=37, n=200, k=40, seed=31):
    """A = 0: every row of C is act(bias) rounded; with no activation C = bias
    bit for bit; with no bias it is act(0) = +0."""
    fails = []
    rng = np.random.default_rng(seed)
    a = np.zeros((m, k), dtype=np.float16)
    b = _r16(rng, (k, n), 2.0)
    bias = _r16(rng, (n,), 3.0)
    for act in ("none", "relu", "gelu"):
        want = np.broadcast_to(to_f16_bits(act64(bias.astype(np.float64), act)), (m, n))
        # act(bias) of an exactly representable input: bit exact everywhere
        # except GELU on an fp32 path, whose erf is not correctly rounded
        _cmp(f"A=0 bias act={act}", fn(a, b, bias, act), want,
             exact or act != "gelu", fails, strict_zero=exact)
    _cmp("A=0 no bias gelu", fn(a, b, None, "gelu"), np.zeros((m, n), np.uint16), True, fails,
         strict_zero=exact)
    return fails


def pin_identity_bias(fn, exact=True, n=150, seed=32):
    """A = I: C = act(B + bias) (B + bias is exact in fp64 and in fp32)."""
    fails = []
    rng = np.random.default_rng(seed)
    k = 129
    a = np.eye(k, dtype=np.float16)
    b = _r16(rng, (k, n), 3.0)
    bias = _r16(rng, (n,), 1.0)
    x = b.astype(np.float64) + bias.astype(np.float64)[None, :]
    for act in ("none", "relu", "gelu"):
        want = to_f16_bits(act64(x, act))
        _cmp(f"I@B + bias act={act}", fn(a, b, bias, act), want, exact or act != "gelu", fails,
             strict_zero=exact)
    return fails


def pin_bruteforce_bias_relu(fn, exact=True, seed=33):
    """Exact rationals on tiny ragged shapes: ReLU(sum + bias), RNE."""
    fails = []
    rng = np.random.default_rng(seed)
    for (m, n, k) in ((1, 1, 1), (3, 5, 7), (5, 9, 17), (9, 2, 33), (17, 33, 5)):
        a = _r16(rng, (m, k), 2.0)
        b = _r16(rng, (k, n), 2.0)
        bias = _r16(rng, (n,), 4.0)
        want = np.zeros((m, n), dtype=np.uint16)
        for i in range(m):
            for j in range(n):
                s = Fraction(float(bias[j]))
                for t in range(k):
                    s += Fraction(float(a[i, t])) * Fraction(float(b[t, j]))
                want[i, j] = fraction_to_f16_bits(s if s > 0 else Fraction(0))
        _cmp(f"brute bias+relu {m}x{n}x{k}", fn(a, b, bias, "relu"), want, exact, fails)
    return fails


def pin_gelu_random(fn, exact=True, m=64, n=96, k=48, seed=34):
    """Generic inputs against fp64 sums + torch's GELU, rounded by numpy."""
    fails = []
    rng = np.random.default_rng(seed)
    a = _r16(rng, (m, k))
    b = _r16(rng, (k, n), 0.3)
    bias = _r16(rng, (n,), 0.5)
    x = a.astype(np.float64) @ b.astype(np.float64) + bias.astype(np.float64)[None, :]
    want = to_f16_bits(gelu64(x))
    got = np.asarray(fn(a, b, bias, "gelu"), dtype=np.float16)
    if exact:
        # another summation order (BLAS) can move a value across an fp16 tie
        # only with negligible probability; allow none
        _cmp("gelu random", got, want, True, fails)
    else:
        _cmp("gelu random", got, want, False, fails)
    return fails


EPILOGUE_PINS = [pin_bias_broadcast, pin_identity_bias, pin_bruteforce_bias_relu,
                 pin_gelu_random]
