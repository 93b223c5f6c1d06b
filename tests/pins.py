"""Pins for an fp16 GEMM(+ReLU) implementation: cases whose answer is fixed by
the mathematics rather than by another implementation.

Each ``pin_*`` function takes ``fn(a, b, relu) -> float16 (M, N) array`` (``a``
and ``b`` are float16 numpy arrays, possibly strided views) and returns a list
of failure messages (empty = pass).  With ``exact=True`` (the oracle) every
pin must hold bit for bit; with ``exact=False`` (the fp32-accumulating GPU
path) the pins whose answer is exact in fp32 still compare bits, and the
others use the acceptance tolerance |c - ref| <= 1e-2 + 1e-2 |ref|.

The operation is the fused GEMM + ReLU of "Writing high-performance kernels in
TileLang" (atlascloud.ai blog), section "Escribamos un GEMM".
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

ATOL = 1e-2
RTOL = 1e-2


# ---------------------------------------------------------------- helpers ---

def f16(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float16)


def bits(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float16).view(np.uint16)


def relu_bits_expected(x16: np.ndarray) -> np.ndarray:
    """Bits of max(x, 0) for fp16 data: negatives, -0 and NaN become +0."""
    x = np.asarray(x16, dtype=np.float16)
    out = x.copy()
    out[~(x > 0)] = np.float16(0.0)
    return out.view(np.uint16)


def plus_zero_bits(x16: np.ndarray) -> np.ndarray:
    """x with -0 replaced by +0 (a sum that starts from +0 never yields -0)."""
    x = np.asarray(x16, dtype=np.float16).copy()
    x[x == 0] = np.float16(0.0)
    return x.view(np.uint16)


_F16_TABLE = None


def _f16_table():
    """Sorted exact values of all finite non-negative fp16 numbers, plus a
    sentinel at 65536 standing for +Inf (the next value after 65504 with an
    even significand), built from numpy's fp16 decoder."""
    global _F16_TABLE
    if _F16_TABLE is None:
        pos = np.arange(0x0000, 0x7C00, dtype=np.uint16)
        vals = [Fraction(float(v)) for v in pos.view(np.float16).astype(np.float64)]
        _F16_TABLE = (vals + [Fraction(65536)], list(range(0x0000, 0x7C00)) + [0x7C00])
    return _F16_TABLE


def fraction_to_f16_bits(q: Fraction) -> int:
    """Exact round-to-nearest-even of a rational to fp16, by search over the
    table of representable values (independent of any float arithmetic)."""
    import bisect
    vals, codes = _f16_table()
    sign = 0x8000 if q < 0 else 0
    mag = -q if q < 0 else q
    if mag == 0:
        return 0  # an exact zero sum is +0
    i = bisect.bisect_left(vals, mag)
    if i < len(vals) and vals[i] == mag:
        return sign | codes[i]
    lo, hi = i - 1, i
    if hi >= len(vals):
        return sign | 0x7C00
    dlo, dhi = mag - vals[lo], vals[hi] - mag
    if dlo < dhi:
        pick = lo
    elif dhi < dlo:
        pick = hi
    else:
        pick = lo if (codes[lo] & 1) == 0 else hi
    return sign | codes[pick]


def exact_gemm_bits(a16: np.ndarray, b16: np.ndarray, relu: bool) -> np.ndarray:
    """Brute force over exact rationals: sum, ReLU, RNE to fp16.  Tiny shapes."""
    a = np.asarray(a16, dtype=np.float16)
    b = np.asarray(b16, dtype=np.float16)
    M, K = a.shape
    _, N = b.shape
    af = [[Fraction(float(a[i, k])) for k in range(K)] for i in range(M)]
    bf = [[Fraction(float(b[k, j])) for j in range(N)] for k in range(K)]
    out = np.zeros((M, N), dtype=np.uint16)
    for i in range(M):
        for j in range(N):
            s = Fraction(0)
            for k in range(K):
                s += af[i][k] * bf[k][j]
            if relu and not s > 0:
                s = Fraction(0)
            out[i, j] = fraction_to_f16_bits(s)
    return out


def within_tol(c16, ref16) -> np.ndarray:
    c = np.asarray(c16, dtype=np.float16).astype(np.float64)
    r = np.asarray(ref16, dtype=np.float16).astype(np.float64)
    with np.errstate(invalid="ignore"):
        return (c == r) | (np.abs(c - r) <= ATOL + RTOL * np.abs(r))


def _cmp(name, got, want_bits, exact_ok: bool, fails: list, strict_zero: bool = True):
    """Compare bits (exact_ok) or values within tolerance.  With
    strict_zero=False, -0 and +0 count as equal: a tensor-core sum of signed
    zero products has no leading +0 term, so its zero sign may differ from the
    oracle's 0 + sum (ReLU outputs are checked for -0 separately)."""
    got = np.asarray(got, dtype=np.float16)
    if got.shape != want_bits.shape:
        fails.append(f"{name}: shape {got.shape} != {want_bits.shape}")
        return
    if exact_ok:
        gb = got.view(np.uint16)
        wb = np.asarray(want_bits, dtype=np.uint16)
        if not strict_zero:
            gb = np.where(gb == 0x8000, 0, gb)
            wb = np.where(wb == 0x8000, 0, wb)
        bad = gb != wb
        if bad.any():
            idx = np.argwhere(bad)[0]
            fails.append(f"{name}: {int(bad.sum())} elements differ in bits, first at "
                         f"{tuple(idx)}: got {got[tuple(idx)]!r} want "
                         f"{want_bits[tuple(idx)].view(np.float16)!r}")
    else:
        ref = want_bits.view(np.float16)
        ok = within_tol(got, ref)
        if not ok.all():
            idx = np.argwhere(~ok)[0]
            fails.append(f"{name}: {int((~ok).sum())} elements out of tolerance, first at "
                         f"{tuple(idx)}: got {got[tuple(idx)]!r} want {ref[tuple(idx)]!r}")


def _rng(seed):
    return np.random.default_rng(seed)


def _randn16(rng, shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float16)


# ------------------------------------------------------------------- pins ---

def pin_identity(fn, exact=True, sizes=((37, 53), (128, 200), (200, 129))):
    """A = I gives C = ReLU(B) (or B, with -0 -> +0); B = I gives ReLU(A)."""
    fails = []
    for t, (k, n) in enumerate(sizes):
        rng = _rng(100 + t)
        b = _randn16(rng, (k, n), 4.0)
        b[0, : min(3, n)] = np.float16(-0.0)
        eye = np.eye(k, dtype=np.float16)
        _cmp(f"I@B relu {k}x{n}", fn(eye, b, True), relu_bits_expected(b), True, fails, exact)
        _cmp(f"I@B plain {k}x{n}", fn(eye, b, False), plus_zero_bits(b), True, fails, exact)
        a = _randn16(rng, (n, k), 4.0)
        _cmp(f"A@I relu {n}x{k}", fn(a, eye, True), relu_bits_expected(a), True, fails, exact)
    return fails


def pin_permutation(fn, exact=True, k=150, n=77, seed=7):
    """A = P (a permutation) gives C = ReLU(B[perm])."""
    fails = []
    rng = _rng(seed)
    perm = rng.permutation(k)
    p = np.zeros((k, k), dtype=np.float16)
    p[np.arange(k), perm] = 1
    b = _randn16(rng, (k, n), 3.0)
    _cmp("P@B relu", fn(p, b, True), relu_bits_expected(b[perm]), True, fails, exact)
    _cmp("P@B plain", fn(p, b, False), plus_zero_bits(b[perm]), True, fails, exact)
    # and on the right: A @ P permutes columns: (A P)[:, j] = A[:, inv(perm)[j]]
    a = _randn16(rng, (n, k), 3.0)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(k)
    _cmp("A@P relu", fn(a, p, True), relu_bits_expected(a[:, inv]), True, fails, exact)
    return fails


def pin_all_ones(fn, exact=True, ks=(256, 1000, 1024, 4096, 8192), m=3, n=5):
    """A = 1, B = 1 gives C = K exactly; A = -1 gives 0 with ReLU, -K without."""
    fails = []
    for k in ks:
        a = np.ones((m, k), dtype=np.float16)
        b = np.ones((k, n), dtype=np.float16)
        want = np.full((m, n), k, dtype=np.float16).view(np.uint16)
        _cmp(f"ones K={k}", fn(a, b, True), want, True, fails, exact)
        _cmp(f"neg ones relu K={k}", fn(-a, b, True),
             np.zeros((m, n), dtype=np.uint16), True, fails, exact)
        _cmp(f"neg ones plain K={k}", fn(-a, b, False), (-want.view(np.float16)).view(np.uint16),
             True, fails, exact)
    return fails


def pin_rank1(fn, exact=True, m=70, n=90, k=33, seed=11):
    """Only column kk of A and row kk of B are non-zero: C[i,j] = u_i v_j,
    whose fp16 rounding is numpy's (the product of two fp16 values is exact in
    fp64, and in fp32)."""
    fails = []
    rng = _rng(seed)
    for kk in (0, k - 1, k // 2):
        u = _randn16(rng, (m,), 2.0)
        v = _randn16(rng, (n,), 2.0)
        a = np.zeros((m, k), dtype=np.float16)
        b = np.zeros((k, n), dtype=np.float16)
        a[:, kk] = u
        b[kk, :] = v
        outer = np.outer(u.astype(np.float64), v.astype(np.float64))
        o16 = outer.astype(np.float16)
        # a tiny negative product rounds to -0; only an exact zero sum is +0
        want_plain = o16.view(np.uint16).copy()
        want_plain[outer == 0] = 0
        want_relu = relu_bits_expected(o16)
        _cmp(f"rank1 kk={kk} relu", fn(a, b, True), want_relu, True, fails, exact)
        _cmp(f"rank1 kk={kk} plain", fn(a, b, False), want_plain, True, fails, exact)
    return fails


def pin_block_diagonal(fn, exact=True, blocks=((100, 60, 129), (29, 128, 7), (129, 3, 100)),
                       seed=13):
    """Block-diagonal A (blocks m_i x k_i) times block-diagonal B (k_i x n_i):
    off-block outputs are exactly +0 and each diagonal block equals the
    product of its own blocks."""
    fails = []
    rng = _rng(seed)
    ms = [bl[0] for bl in blocks]
    ks = [bl[1] for bl in blocks]
    ns = [bl[2] for bl in blocks]
    M, K, N = sum(ms), sum(ks), sum(ns)
    a = np.zeros((M, K), dtype=np.float16)
    b = np.zeros((K, N), dtype=np.float16)
    subs = []
    mo = ko = no = 0
    for (mi, ki, ni) in blocks:
        ab = _randn16(rng, (mi, ki))
        bb = _randn16(rng, (ki, ni))
        a[mo:mo + mi, ko:ko + ki] = ab
        b[ko:ko + ki, no:no + ni] = bb
        subs.append((mo, no, mi, ni, ab, bb))
        mo, ko, no = mo + mi, ko + ki, no + ni
    for relu in (True, False):
        c = np.asarray(fn(a, b, relu), dtype=np.float16)
        mask = np.ones((M, N), dtype=bool)
        for (mo, no, mi, ni, ab, bb) in subs:
            mask[mo:mo + mi, no:no + ni] = False
            blk = np.asarray(fn(ab, bb, relu), dtype=np.float16)
            # the block inside the big product is summed with other k-offsets
            # than the block alone: bit-equal only for an exact summation
            _cmp(f"block ({mo},{no}) relu={relu}", c[mo:mo + mi, no:no + ni],
                 blk.view(np.uint16), exact, fails, exact)
        off = c[mask].view(np.uint16)
        if not exact:
            off = np.where(off == 0x8000, 0, off)
        if (off != 0).any():
            fails.append(f"block-diag relu={relu}: {int((off != 0).sum())} off-block "
                         f"elements are not +0")
    return fails


TINY_SHAPES = ((1, 1, 1), (2, 3, 5), (3, 5, 8), (5, 8, 17), (8, 17, 33),
               (17, 33, 3), (33, 2, 17), (1, 33, 33), (33, 1, 2))


def pin_bruteforce(fn, exact=True, shapes=TINY_SHAPES, seed=17):
    """Exact-rational brute force on tiny ragged shapes, with both generic
    fp16 inputs and inputs on a coarse grid (whose fp64 sums are exact)."""
    fails = []
    rng = _rng(seed)
    for t, (m, n, k) in enumerate(shapes):
        a = _randn16(rng, (m, k), 2.0)
        b = _randn16(rng, (k, n), 2.0)
        ga = (rng.integers(-512, 513, (m, k)) / 128.0).astype(np.float16)
        gb = (rng.integers(-512, 513, (k, n)) / 128.0).astype(np.float16)
        for tag, (x, y) in (("randn", (a, b)), ("grid", (ga, gb))):
            for relu in (True, False):
                want = exact_gemm_bits(x, y, relu)
                _cmp(f"brute {tag} {m}x{n}x{k} relu={relu}", fn(x, y, relu), want, exact, fails)
    return fails


def pin_rounding_ties(fn, exact=True):
    """Sums that land on or next to an fp16 rounding boundary:
    1 + 2^-11 is halfway between 1 and 1 + 2^-10 and must round to 1 (even);
    1 + 3*2^-11 must round up to 1 + 2^-9 (even);
    1 + 2^-11 + 2^-24 is just above halfway and must round up -- an fp32
    accumulator that rounds the sum first would tie and round down;
    65504 + 16 (halfway to the overflow threshold) rounds to +Inf;
    2^-25 (half the smallest subnormal) ties to +0; 3 * 2^-26 rounds up to
    2^-24, also after cancelling terms."""
    fails = []
    cases = [
        ([1.0, 2.0 ** -11], 1.0),
        ([1.0, 3 * 2.0 ** -11], 1.0 + 2.0 ** -9),
        ([1.0, 2.0 ** -11, 2.0 ** -24], 1.0 + 2.0 ** -10),
        ([65504.0, 16.0], np.inf),
        ([65504.0, 15.0], 65504.0),
        ([2.0 ** -25], 0.0),
        ([3 * 2.0 ** -26], 2.0 ** -24),
        ([2.0 ** -14, -(2.0 ** -14), 2.0 ** -25, 2.0 ** -26], 2.0 ** -24),
    ]
    for t, (terms, want) in enumerate(cases):
        # write each term as (fp16 a) * (fp16 b) with exact representations
        ks = len(terms)
        a = np.ones((1, ks), dtype=np.float16)
        b = np.zeros((ks, 1), dtype=np.float16)
        for j, v in enumerate(terms):
            # split v = p * q with both fp16-exact: take q = 2^e so p lies in [1, 2)
            if v == 0:
                continue
            e = int(np.floor(np.log2(abs(v))))
            p = v / 2.0 ** e
            if e < -14:
                a[0, j] = np.float16(2.0 ** (e + 14))
                b[j, 0] = np.float16(p * 2.0 ** -14)
            else:
                a[0, j] = np.float16(p)
                b[j, 0] = np.float16(2.0 ** e)
            assert float(a[0, j]) * float(b[j, 0]) == v, (t, j, v)
        want_bits = np.array([[np.float16(want)]], dtype=np.float16).view(np.uint16)
        _cmp(f"tie case {t} ({terms})", fn(a, b, True), want_bits, exact, fails)
    return fails


def pin_invariants(fn, exact=True, shape=(96, 80, 64), seed=19):
    """ReLU output: no negative value, no -0, no NaN."""
    fails = []
    rng = _rng(seed)
    m, n, k = shape
    a = _randn16(rng, (m, k), 3.0)
    b = _randn16(rng, (k, n), 3.0)
    c = np.asarray(fn(a, b, True), dtype=np.float16)
    if np.isnan(c).any():
        fails.append("invariant: NaN in ReLU output")
    if (c < 0).any():
        fails.append("invariant: negative value in ReLU output")
    if (c.view(np.uint16) == 0x8000).any():
        fails.append("invariant: -0 in ReLU output")
    return fails


def pin_strided(fn, exact=True, m=45, n=70, k=90, pad=(8, 16, 24), seed=23):
    """Padded row strides (ld > cols) give the same result as dense inputs."""
    fails = []
    rng = _rng(seed)
    a = _randn16(rng, (m, k))
    b = _randn16(rng, (k, n))
    ref = np.asarray(fn(a, b, True), dtype=np.float16).view(np.uint16).copy()
    ap = np.full((m, k + pad[0]), np.float16(1000.0), dtype=np.float16)
    bp = np.full((k, n + pad[1]), np.float16(-1000.0), dtype=np.float16)
    ap[:, :k] = a
    bp[:, :n] = b
    got = fn(ap[:, :k], bp[:, :n], True)
    _cmp("strided", got, ref, True, fails, exact)
    return fails


ALL_PINS = [pin_identity, pin_permutation, pin_all_ones, pin_rank1, pin_block_diagonal,
            pin_bruteforce, pin_rounding_ties, pin_invariants, pin_strided]
