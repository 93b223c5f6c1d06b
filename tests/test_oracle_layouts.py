"""The oracle's operand layouts (T.gemm's transpose_A / transpose_B of
"Writing high-performance kernels in TileLang", atlascloud.ai blog, section
"Escribamos un GEMM"): storing an operand transposed must give the same bits
as passing its explicit transpose, for every activation, and the general
routine agrees with the plain ones."""
import numpy as np
import pytest

import pins


@pytest.mark.parametrize("ta,tb", [(False, False), (True, False), (False, True), (True, True)])
@pytest.mark.parametrize("act", ["none", "relu", "gelu"])
def test_transposed_storage_same_bits(oracle_mod, ta, tb, act):
    rng = np.random.default_rng(3)
    m, n, k = 37, 53, 71
    a = rng.standard_normal((m, k)).astype(np.float16)
    b = rng.standard_normal((k, n)).astype(np.float16)
    bias = rng.standard_normal(n).astype(np.float16)
    ref = oracle_mod.gemm_bias_act(a, b, bias, act).view(np.uint16)
    a_st = np.ascontiguousarray(a.T) if ta else a
    b_st = np.ascontiguousarray(b.T) if tb else b
    got = oracle_mod.gemm_general(a_st, b_st, bias, act, trans_a=ta, trans_b=tb).view(np.uint16)
    assert np.array_equal(got, ref)


def test_general_matches_exact_bruteforce(oracle_mod):
    rng = np.random.default_rng(4)
    for (m, n, k) in ((1, 1, 1), (3, 5, 7), (9, 4, 33)):
        a = rng.standard_normal((m, k)).astype(np.float16)
        b = rng.standard_normal((k, n)).astype(np.float16)
        want = pins.exact_gemm_bits(a, b, True)
        got = oracle_mod.gemm_general(np.ascontiguousarray(a.T), np.ascontiguousarray(b.T), None,
                                      "relu", trans_a=True, trans_b=True).view(np.uint16)
        assert np.array_equal(got, want)


def test_transposed_strides(oracle_mod):
    """Padded leading dimensions of the transposed storages."""
    rng = np.random.default_rng(5)
    m, n, k = 20, 30, 40
    a = rng.standard_normal((m, k)).astype(np.float16)
    b = rng.standard_normal((k, n)).astype(np.float16)
    a_t = np.full((k, m + 8), np.float16(7), dtype=np.float16)
    a_t[:, :m] = a.T
    b_t = np.full((n, k + 16), np.float16(-7), dtype=np.float16)
    b_t[:, :k] = b.T
    got = oracle_mod.gemm_general(a_t[:, :m], b_t[:, :k], None, "none", True, True)
    assert np.array_equal(got.view(np.uint16), oracle_mod.gemm(a, b).view(np.uint16))
