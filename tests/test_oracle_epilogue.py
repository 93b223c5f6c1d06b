"""The oracle's fused bias + activation epilogue against the mathematics.

act(A @ B + bias) as in "TileLang simplifica la creación de kernels GPU de
alto rendimiento" (posicionamiento-web.ar), section "Fusionar operaciones para
reducir viajes a memoria"; GELU read as the exact x * Phi(x).
"""
import math

import numpy as np
import pytest
import torch

import pins_epilogue as pe


def oracle_fn(oracle_mod):
    def fn(a, b, bias, act):
        return oracle_mod.gemm_bias_act(a, b, bias, act)
    return fn


@pytest.mark.parametrize("pin", pe.EPILOGUE_PINS, ids=lambda p: p.__name__)
def test_epilogue_pin(oracle_mod, pin):
    fails = pin(oracle_fn(oracle_mod), exact=True)
    assert not fails, "\n".join(fails)


def test_plain_paths_agree(oracle_mod):
    rng = np.random.default_rng(1)
    a = rng.standard_normal((50, 70)).astype(np.float16)
    b = rng.standard_normal((70, 90)).astype(np.float16)
    assert np.array_equal(oracle_mod.gemm_bias_act(a, b, None, "none").view(np.uint16),
                          oracle_mod.gemm(a, b).view(np.uint16))
    assert np.array_equal(oracle_mod.gemm_bias_act(a, b, None, "relu").view(np.uint16),
                          oracle_mod.gemm_relu(a, b).view(np.uint16))


def test_gelu_definition(oracle_mod):
    x = np.concatenate([np.linspace(-12, 12, 2001), np.array([0.0, -0.0, 1e-300, -1e-300])])
    ours = oracle_mod.activation_f64(x, "gelu")
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="none").numpy()
    # torch evaluates 0.5 x (1 + erf(x / sqrt 2)), which cancels to 0 in the far
    # negative tail where the oracle's erfc form keeps ~1e-16; both are far
    # below fp16 resolution (6e-8)
    assert np.allclose(ours, ref, rtol=1e-13, atol=1e-15)
    # x Phi(x) - (-x) Phi(-x) = x (Phi(x) + Phi(-x)) = x
    odd = oracle_mod.activation_f64(x, "gelu") - oracle_mod.activation_f64(-x, "gelu")
    assert np.allclose(odd, x, rtol=1e-14, atol=1e-14)
    assert ours[np.argmin(np.abs(x))] == 0.0
    # Phi(10) = 1 - 7.6e-24: GELU(10) is 10 in fp64; GELU(-10) ~ -7.6e-23
    g = oracle_mod.activation_f64(np.array([10.0, -10.0, 1.0]), "gelu")
    assert g[0] == 10.0
    assert -1e-21 < g[1] < 0
    assert abs(g[2] - 0.5 * (1 + math.erf(1 / math.sqrt(2)))) < 1e-15


def _mutant(kind):
    def fn(a, b, bias, act):
        A = np.asarray(a, np.float16).astype(np.float64)
        B = np.asarray(b, np.float16).astype(np.float64)
        s = A @ B
        bb = np.zeros(B.shape[1]) if bias is None else np.asarray(bias, np.float16).astype(np.float64)
        if kind == "bias_after_act":
            x = pe.act64(s, act) + bb[None, :]
        elif kind == "bias_by_row":
            rows = np.resize(bb, s.shape[0])
            x = pe.act64(s + rows[:, None], act)
        elif kind == "tanh_gelu":
            z = s + bb[None, :]
            if act == "gelu":
                x = 0.5 * z * (1 + np.tanh(math.sqrt(2 / math.pi) * (z + 0.044715 * z ** 3)))
            else:
                x = pe.act64(z, act)
        elif kind == "sqrt2_misplaced":
            z = s + bb[None, :]
            if act == "gelu":
                x = 0.5 * z * (1 + np.vectorize(math.erf)(z * math.sqrt(2)))
            else:
                x = pe.act64(z, act)
        else:
            raise ValueError(kind)
        return pe.to_f16_bits(x).view(np.float16)
    return fn


@pytest.mark.parametrize("kind", ["bias_after_act", "bias_by_row", "tanh_gelu",
                                  "sqrt2_misplaced"])
def test_epilogue_pins_catch_planted_mistakes(kind):
    fn = _mutant(kind)
    caught = [p.__name__ for p in pe.EPILOGUE_PINS if p(fn, exact=True)]
    assert caught, kind
