"""CPU oracle for C = ReLU(A @ B) with fp16 inputs and output.

TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the CUDA library and its Python binding) never calls it, and it never calls
the product path: the two share no code.

The computation (see ``gemm_oracle.c``) follows "Writing high-performance
kernels in TileLang" (atlascloud.ai blog), section "Escribamos un GEMM":
row-major fp16 A (M x K) and B (K x N), a sum over k, max(x, 0), fp16 C.  Here
the sum is carried exactly enough in fp64 (ascending k) and rounded once to
fp16 with round-to-nearest-even.

Inputs are numpy ``uint16`` arrays of fp16 bit patterns (``float16`` arrays
and torch CPU ``float16`` tensors are accepted and viewed as bits).  Row
strides are taken from the arrays, so padded (ld > cols) views work.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

__all__ = [
    "gemm_relu", "gemm", "gemm_relu_at", "gemm_at", "gemm_f64_at",
    "gemm_bias_act", "gemm_general", "activation_f64", "decode_f16", "encode_f16",
    "max_threads",
]

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64, p = ctypes.c_int64, ctypes.c_void_p
        lib.oracle_gemm_f16.argtypes = [p, p, p, i64, i64, i64, i64, i64, i64,
                                        ctypes.c_int, ctypes.c_int]
        lib.oracle_gemm_f16.restype = ctypes.c_int
        lib.oracle_gemm_f16_at.argtypes = [p, p, i64, i64, i64, ctypes.c_int, i64,
                                           p, p, p, ctypes.c_int]
        lib.oracle_gemm_f16_at.restype = ctypes.c_int
        lib.oracle_gemm_f64_at.argtypes = [p, p, i64, i64, i64, i64, p, p, p,
                                           ctypes.c_int]
        lib.oracle_gemm_f64_at.restype = ctypes.c_int
        lib.oracle_decode_f16.argtypes = [p, p, i64]
        lib.oracle_decode_f16.restype = None
        lib.oracle_encode_f16.argtypes = [p, p, i64]
        lib.oracle_encode_f16.restype = None
        lib.oracle_gemm_bias_act_f16.argtypes = [p, p, p, p, i64, i64, i64, i64, i64, i64,
                                                 ctypes.c_int, ctypes.c_int]
        lib.oracle_gemm_bias_act_f16.restype = ctypes.c_int
        lib.oracle_gemm_general_f16.argtypes = [p, p, p, p, i64, i64, i64, i64, i64, i64,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int]
        lib.oracle_gemm_general_f16.restype = ctypes.c_int
        lib.oracle_activation_f64.argtypes = [p, p, i64, ctypes.c_int]
        lib.oracle_activation_f64.restype = None
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _bits(x) -> np.ndarray:
    """Return a 2-D uint16 view of fp16 data with unit column stride."""
    if hasattr(x, "detach"):  # torch tensor (CPU)
        import torch
        if x.device.type != "cpu":
            raise ValueError("the oracle takes host (CPU) data only")
        if x.dtype != torch.float16:
            raise TypeError(f"expected float16, got {x.dtype}")
        x = x.detach().contiguous().view(torch.int16).numpy().view(np.uint16)
    x = np.asarray(x)
    if x.dtype == np.float16:
        x = x.view(np.uint16)
    if x.dtype != np.uint16:
        raise TypeError(f"expected fp16 bits (uint16) or float16, got {x.dtype}")
    if x.ndim != 2:
        raise ValueError("expected a 2-D matrix")
    if x.strides[1] != 2 or x.strides[0] % 2 != 0 or x.strides[0] < 0:
        x = np.ascontiguousarray(x)
    return x


def _ld(x: np.ndarray) -> int:
    return max(x.strides[0] // 2, x.shape[1]) if x.shape[0] > 1 else x.shape[1]


def _threads(nthreads):
    return 0 if nthreads is None else int(nthreads)


def _gemm(a, b, relu: bool, nthreads=None) -> np.ndarray:
    a, b = _bits(a), _bits(b)
    M, K = a.shape
    K2, N = b.shape
    if K != K2:
        raise ValueError(f"inner dimensions differ: {a.shape} @ {b.shape}")
    c = np.zeros((M, N), dtype=np.uint16)
    if M == 0 or N == 0:
        return c.view(np.float16)
    rc = _load().oracle_gemm_f16(a.ctypes.data, b.ctypes.data, c.ctypes.data,
                                 M, N, K, _ld(a), _ld(b), N, int(relu),
                                 _threads(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_gemm_f16 failed ({rc})")
    return c.view(np.float16)


def gemm_relu(a, b, nthreads=None) -> np.ndarray:
    """Full ReLU(A @ B) as an (M, N) float16 array."""
    return _gemm(a, b, True, nthreads)


def gemm(a, b, nthreads=None) -> np.ndarray:
    """Full A @ B (no activation) as an (M, N) float16 array."""
    return _gemm(a, b, False, nthreads)


def _at(a, b, rows, cols, relu: bool, nthreads=None) -> np.ndarray:
    a, b = _bits(a), _bits(b)
    M, K = a.shape
    K2, N = b.shape
    if K != K2:
        raise ValueError("inner dimensions differ")
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    if rows.shape != cols.shape or rows.ndim != 1:
        raise ValueError("rows and cols must be 1-D and of equal length")
    if rows.size and (rows.min() < 0 or rows.max() >= M or cols.min() < 0 or cols.max() >= N):
        raise IndexError("sample index out of range")
    out = np.zeros(rows.size, dtype=np.uint16)
    rc = _load().oracle_gemm_f16_at(a.ctypes.data, b.ctypes.data, K, _ld(a), _ld(b),
                                    int(relu), rows.size, rows.ctypes.data,
                                    cols.ctypes.data, out.ctypes.data,
                                    _threads(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_gemm_f16_at failed ({rc})")
    return out.view(np.float16)


def gemm_relu_at(a, b, rows, cols, nthreads=None) -> np.ndarray:
    """ReLU(A @ B)[rows[s], cols[s]] for each sample s, as float16."""
    return _at(a, b, rows, cols, True, nthreads)


def gemm_at(a, b, rows, cols, nthreads=None) -> np.ndarray:
    """(A @ B)[rows[s], cols[s]] for each sample s, as float16."""
    return _at(a, b, rows, cols, False, nthreads)


def gemm_f64_at(a, b, rows, cols, nthreads=None) -> np.ndarray:
    """The fp64 sums (A @ B)[rows[s], cols[s]] before ReLU and rounding."""
    a, b = _bits(a), _bits(b)
    M, K = a.shape
    _, N = b.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    if rows.size and (rows.min() < 0 or rows.max() >= M or cols.min() < 0 or cols.max() >= N):
        raise IndexError("sample index out of range")
    out = np.zeros(rows.size, dtype=np.float64)
    rc = _load().oracle_gemm_f64_at(a.ctypes.data, b.ctypes.data, K, _ld(a), _ld(b),
                                    rows.size, rows.ctypes.data, cols.ctypes.data,
                                    out.ctypes.data, _threads(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_gemm_f64_at failed ({rc})")
    return out


def decode_f16(bits) -> np.ndarray:
    """fp16 bit patterns -> float64, with the oracle's own decoder."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    _load().oracle_decode_f16(bits.ctypes.data, out.ctypes.data, bits.size)
    return out


def encode_f16(values) -> np.ndarray:
    """float64 -> fp16 bit patterns (RNE), with the oracle's own encoder."""
    values = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(values.shape, dtype=np.uint16)
    _load().oracle_encode_f16(values.ctypes.data, out.ctypes.data, values.size)
    return out


ACT_NONE, ACT_RELU, ACT_GELU = 0, 1, 2
_ACTS = {"none": ACT_NONE, "relu": ACT_RELU, "gelu": ACT_GELU}


def gemm_bias_act(a, b, bias=None, act="gelu", nthreads=None) -> np.ndarray:
    """act(A @ B + bias) as an (M, N) float16 array; bias is an fp16 vector of
    length N (or None); act is "none", "relu" or "gelu" (erf form)."""
    a, b = _bits(a), _bits(b)
    M, K = a.shape
    K2, N = b.shape
    if K != K2:
        raise ValueError("inner dimensions differ")
    code = _ACTS[act] if isinstance(act, str) else int(act)
    c = np.zeros((M, N), dtype=np.uint16)
    if M == 0 or N == 0:
        return c.view(np.float16)
    bias_ptr = None
    if bias is not None:
        if hasattr(bias, "detach"):  # torch tensor
            bias = bias.detach().reshape(1, -1)
        else:
            bias = np.asarray(bias).reshape(1, -1)
        bb = np.ascontiguousarray(_bits(bias))
        if bb.shape[1] != N:
            raise ValueError("bias must have N elements")
        bias_ptr = bb.ctypes.data
    rc = _load().oracle_gemm_bias_act_f16(a.ctypes.data, b.ctypes.data, bias_ptr, c.ctypes.data,
                                          M, N, K, _ld(a), _ld(b), N, code, _threads(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_gemm_bias_act_f16 failed ({rc})")
    return c.view(np.float16)


def gemm_general(a, b, bias=None, act="relu", trans_a=False, trans_b=False,
                 nthreads=None) -> np.ndarray:
    """act(op(A) @ op(B) + bias): with trans_a the stored ``a`` is K x M and
    op(A) = a.T; with trans_b the stored ``b`` is N x K and op(B) = b.T."""
    a, b = _bits(a), _bits(b)
    M, K = (a.shape[1], a.shape[0]) if trans_a else a.shape
    K2, N = (b.shape[1], b.shape[0]) if trans_b else b.shape
    if K != K2:
        raise ValueError("inner dimensions differ")
    code = _ACTS[act] if isinstance(act, str) else int(act)
    c = np.zeros((M, N), dtype=np.uint16)
    if M == 0 or N == 0:
        return c.view(np.float16)
    bias_ptr = None
    if bias is not None:
        bias = bias.detach().reshape(1, -1) if hasattr(bias, "detach") else np.asarray(bias).reshape(1, -1)
        bb = np.ascontiguousarray(_bits(bias))
        if bb.shape[1] != N:
            raise ValueError("bias must have N elements")
        bias_ptr = bb.ctypes.data
    rc = _load().oracle_gemm_general_f16(a.ctypes.data, b.ctypes.data, bias_ptr, c.ctypes.data,
                                         M, N, K, _ld(a), _ld(b), N, int(bool(trans_a)),
                                         int(bool(trans_b)), code, _threads(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_gemm_general_f16 failed ({rc})")
    return c.view(np.float16)


def activation_f64(x, act="gelu") -> np.ndarray:
    """The oracle's activation on float64 values (no rounding)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    code = _ACTS[act] if isinstance(act, str) else int(act)
    _load().oracle_activation_f64(x.ctypes.data, out.ctypes.data, x.size, code)
    return out


def max_threads() -> int:
    """Number of OpenMP threads the oracle uses by default."""
    return int(_load().oracle_max_threads())

