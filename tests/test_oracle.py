"""The CPU oracle against what the mathematics fixes (no GPU needed).

The oracle is the plain definition of the fused GEMM + ReLU from "Writing
high-performance kernels in TileLang" (atlascloud.ai blog), section
"Escribamos un GEMM": C = max(A @ B, 0) with fp16 A, B, C.  These tests pin it
to things other than itself: numpy's IEEE fp16 conversions (exhaustively),
exact rational arithmetic, closed forms (identity, permutation, all-ones,
rank-1, block-diagonal), rounding boundaries, invariants and strides, plus a
mutation check that each plausible slip fails at least one pin.
"""
import numpy as np
import pytest
import torch

import pins
from tiled_tensor_core_05_b200 import workloads


def oracle_fn(oracle_mod):
    def fn(a, b, relu):
        return oracle_mod.gemm_relu(a, b) if relu else oracle_mod.gemm(a, b)
    return fn


# ------------------------------------------------------- fp16 conversions ---

def test_decode_exhaustive(oracle_mod):
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle_mod.decode_f16(allbits)
    ref = allbits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zeros survive
    assert np.signbit(ours[0x8000]) and not np.signbit(ours[0x0000])


def test_encode_roundtrip_all_finite(oracle_mod):
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = np.isfinite(allbits.view(np.float16))
    vals = allbits.view(np.float16).astype(np.float64)
    back = oracle_mod.encode_f16(vals[finite])
    assert np.array_equal(back, allbits[finite])
    inf_bits = oracle_mod.encode_f16(np.array([np.inf, -np.inf]))
    assert list(inf_bits) == [0x7C00, 0xFC00]
    assert np.isnan(oracle_mod.encode_f16(np.array([np.nan])).view(np.float16))[0]


def test_encode_midpoints_and_neighbours(oracle_mod):
    """Every midpoint between consecutive fp16 values (a tie), and the doubles
    just either side of it, against numpy's float64 -> float16 conversion."""
    pos = np.arange(0x0000, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    nxt = np.append(pos[1:], 65536.0)  # 65536 stands for the overflow neighbour
    mids = (pos + nxt) / 2.0           # exact in fp64
    pts = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf)])
    pts = np.concatenate([pts, -pts])
    with np.errstate(over="ignore"):
        ref = pts.astype(np.float16).view(np.uint16)
    ours = oracle_mod.encode_f16(pts)
    assert np.array_equal(ours, ref)


def test_encode_random_doubles(oracle_mod):
    rng = np.random.default_rng(5)
    mag = 2.0 ** rng.uniform(-30, 17, 200_000)
    x = mag * rng.choice([-1.0, 1.0], mag.size)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle_mod.encode_f16(x), ref)


# ----------------------------------------------------------------- pins ---

@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(oracle_mod, pin):
    fails = pin(oracle_fn(oracle_mod), exact=True)
    assert not fails, "\n".join(fails)


def test_sampled_equals_full(oracle_mod):
    a, b = workloads.make_inputs(70, 90, 130, seed=3)
    full = oracle_mod.gemm_relu(a, b).view(np.uint16)
    rng = np.random.default_rng(1)
    rows = rng.integers(0, 70, 500)
    cols = rng.integers(0, 90, 500)
    at = oracle_mod.gemm_relu_at(a, b, rows, cols).view(np.uint16)
    assert np.array_equal(at, full[rows, cols])
    plain = oracle_mod.gemm(a, b).view(np.uint16)
    assert np.array_equal(oracle_mod.gemm_at(a, b, rows, cols).view(np.uint16),
                          plain[rows, cols])
    f64 = oracle_mod.gemm_f64_at(a, b, rows, cols)
    with np.errstate(over="ignore"):
        assert np.array_equal(f64.astype(np.float16).view(np.uint16), plain[rows, cols])


def test_thread_count_does_not_change_bits(oracle_mod):
    a, b = workloads.workload_inputs("ragged1000")
    a, b = a[:200], b  # a slice keeps the test quick; same columns and K
    one = oracle_mod.gemm_relu(a, b, nthreads=1).view(np.uint16)
    many = oracle_mod.gemm_relu(a, b, nthreads=max(2, oracle_mod.max_threads())).view(np.uint16)
    assert np.array_equal(one, many)


def test_library_second_opinion_cube256(oracle_mod):
    """torch's fp64 matmul (another summation order) rounded by numpy agrees
    with the oracle on the 256^3 workload up to fp64 ordering effects, which
    can only matter at an fp16 rounding tie."""
    a, b = workloads.workload_inputs("cube256")
    ours = oracle_mod.gemm_relu(a, b)
    ref64 = torch.relu(a.double() @ b.double()).numpy()
    ref = ref64.astype(np.float16)
    diff = ours.view(np.uint16) != ref.view(np.uint16)
    assert diff.sum() <= 2, int(diff.sum())
    if diff.any():
        ulp = np.abs(ours.astype(np.float64) - ref.astype(np.float64))
        assert np.all(ulp[diff] <= np.spacing(np.abs(ref[diff]).astype(np.float16)).astype(np.float64))


def test_invariants_on_workloads(oracle_mod):
    for name in ("cube256", "ragged1000"):
        a, b = workloads.workload_inputs(name)
        if name == "ragged1000":
            a = a[:128]
        c = oracle_mod.gemm_relu(a, b)
        assert not np.isnan(c).any()
        assert (c >= 0).all()
        assert not (c.view(np.uint16) == 0x8000).any()
        # about half the pre-activations of a symmetric product are positive
        frac = float((c > 0).mean())
        assert 0.4 < frac < 0.6, frac


def test_degenerate_sizes(oracle_mod):
    a = np.zeros((0, 5), dtype=np.float16)
    b = np.zeros((5, 3), dtype=np.float16)
    assert oracle_mod.gemm_relu(a, b).shape == (0, 3)
    a = np.zeros((4, 0), dtype=np.float16)
    b = np.zeros((0, 3), dtype=np.float16)
    c = oracle_mod.gemm(a, b)
    assert c.shape == (4, 3) and (c.view(np.uint16) == 0).all()  # empty sum is +0


# -------------------------------------------------------- mutation check ---

def _mutant(kind):
    """A numpy restatement of the computation with one planted mistake."""
    def fn(a, b, relu):
        A = np.asarray(a, dtype=np.float16).astype(np.float64)
        B = np.asarray(b, dtype=np.float16).astype(np.float64)
        if kind == "fp32_accumulate":
            acc = np.zeros((A.shape[0], B.shape[1]), dtype=np.float32)
            for k in range(A.shape[1]):
                acc = (acc + (A[:, k:k + 1] * B[k:k + 1, :]).astype(np.float32)).astype(np.float32)
            s = acc.astype(np.float64)
        elif kind == "drop_last_k":
            s = A[:, :-1] @ B[:-1, :] if A.shape[1] > 1 else np.zeros((A.shape[0], B.shape[1]))
        elif kind == "drop_first_k":
            s = A[:, 1:] @ B[1:, :] if A.shape[1] > 1 else np.zeros((A.shape[0], B.shape[1]))
        elif kind == "sign_flip":
            s = -(A @ B)
        elif kind == "b_column_major":
            K, N = B.shape
            s = A @ B.reshape(-1).reshape(N, K).T
        elif kind == "row_shift":
            s = np.roll(A, 1, axis=0) @ B
        elif kind == "relu_keeps_negative_zero":
            s = A @ B
            if relu:
                s = np.where(s > 0, s, -0.0)
            with np.errstate(over="ignore"):
                return s.astype(np.float16)
        elif kind == "round_half_away":
            s = A @ B
            if relu:
                s = np.maximum(s, 0.0)
            lo = s.astype(np.float16)
            out = lo.copy()
            # where s is exactly halfway between two fp16 values, go away from 0
            nxt = np.nextafter(lo, np.where(s >= 0, np.float16(np.inf), np.float16(-np.inf)))
            prv = np.nextafter(lo, np.where(s >= 0, np.float16(-np.inf), np.float16(np.inf)))
            for cand in (nxt, prv):
                mid = (lo.astype(np.float64) + cand.astype(np.float64)) / 2
                tie = (mid == s) & (np.abs(cand.astype(np.float64)) > np.abs(lo.astype(np.float64)))
                out = np.where(tie, cand, out)
            return out
        elif kind == "ignores_row_stride":
            a_ = np.asarray(a, dtype=np.float16)
            flat = np.lib.stride_tricks.as_strided(a_, shape=a_.shape,
                                                   strides=(a_.shape[1] * 2, 2))
            s = flat.astype(np.float64) @ B
        else:
            raise ValueError(kind)
        if relu:
            s = np.where(s > 0, s, 0.0)
        with np.errstate(over="ignore"):
            return s.astype(np.float16)
    return fn


MUTANTS = ["fp32_accumulate", "drop_last_k", "drop_first_k", "sign_flip", "b_column_major",
           "row_shift", "relu_keeps_negative_zero", "round_half_away", "ignores_row_stride"]


@pytest.mark.parametrize("kind", MUTANTS)
def test_pins_catch_planted_mistakes(kind):
    fn = _mutant(kind)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            if pin(fn, exact=True):
                caught.append(pin.__name__)
        except Exception as e:  # a crash on a pin is also a catch
            caught.append(f"{pin.__name__} ({type(e).__name__})")
    assert caught, f"no pin catches the planted mistake {kind!r}"


def test_clean_numpy_restatement_passes_pins():
    """Control for the mutation check: the same numpy restatement without a
    planted mistake passes every pin except the ones that need exact fp64
    ordering at fp16 ties, which plain numpy also meets here."""
    def fn(a, b, relu):
        A = np.asarray(a, dtype=np.float16).astype(np.float64)
        B = np.asarray(b, dtype=np.float16).astype(np.float64)
        s = A @ B
        if relu:
            s = np.where(s > 0, s, 0.0)
        with np.errstate(over="ignore"):
            return s.astype(np.float16)
    for pin in pins.ALL_PINS:
        fails = pin(fn, exact=True)
        assert not fails, (pin.__name__, fails[:3])


def test_golden_digests(oracle_mod):
    """Inputs and oracle outputs for the small workloads match the digests
    written by tests/golden/make_golden.py (detects drift of the input recipe
    or of the oracle between machines)."""
    import json
    import os
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(__file__), "golden"))
    import make_golden
    with open(os.path.join(os.path.dirname(__file__), "golden", "oracle_digests.json")) as f:
        stored = json.load(f)
    for name in ("cube256", "ragged1000"):
        assert make_golden.digests(name) == stored[name], name
