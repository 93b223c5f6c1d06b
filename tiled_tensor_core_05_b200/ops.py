"""Python binding of libttc05 (argument marshalling only).

Every function here forwards device pointers, sizes, leading dimensions and
the current CUDA stream of PyTorch to the C ABI of ``include/gemm_f16.h``; all
arithmetic happens in the library's CUDA kernels.  There is no fallback: if
the library is missing or the call fails, a ``RuntimeError`` is raised.

The operation is C = ReLU(A @ B) (``gemm_relu_f16``) or C = A @ B
(``gemm_f16``) on row-major fp16 matrices with fp32 accumulation, as in
"Writing high-performance kernels in TileLang" (atlascloud.ai blog), section
"Escribamos un GEMM"; ``gemm_bias_act_f16`` adds a per-column bias and GELU
("TileLang simplifica la creación de kernels GPU de alto rendimiento",
posicionamiento-web.ar, section "Fusionar operaciones para reducir viajes a
memoria"), ``gemm_general`` the transposed operand layouts, ``gemm_config_run`` an
explicit kernel configuration for offline tuning, and ``gemm_host`` the same
product on CPU (host) tensors, copied in and out by the library.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libttc05.so")

PATH_AUTO, PATH_TILE, PATH_SKINNY, PATH_TILE_PAIR, PATH_TILE_PAIR_TALL = 0, 1, 2, 3, 4
PATH_SKINNY_EVEN = 5
ACT_NONE, ACT_RELU, ACT_GELU = 0, 1, 2
_ACTS = {"none": ACT_NONE, "relu": ACT_RELU, "gelu": ACT_GELU}

_lib = None


class GemmConfig(ctypes.Structure):
    """``gemm_config`` of the C ABI: one kernel configuration (0 = default)."""
    _fields_ = [("kernel", ctypes.c_int32), ("block_n", ctypes.c_int32),
                ("stages", ctypes.c_int32), ("group_rows", ctypes.c_int32),
                ("splits", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {f: int(getattr(self, f)) for f, _ in self._fields_}

    def __repr__(self):
        return "GemmConfig(" + ", ".join(f"{k}={v}" for k, v in self.as_dict().items()) + ")"


class HostPlan(ctypes.Structure):
    """``gemm_host_plan`` of the C ABI: how ``gemm_f16_host`` splits a problem."""
    _fields_ = [("split", ctypes.c_int32), ("panels", ctypes.c_int32),
                ("panel_extent", ctypes.c_int64), ("estimate_bytes", ctypes.c_double)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_}


HOST_SPLIT_ROWS, HOST_SPLIT_COLS = 0, 1

_SIGNATURES = {
    "gemm_relu_f16": ([ctypes.c_void_p] * 3 + [ctypes.c_int64] * 6 + [ctypes.c_void_p],
                      ctypes.c_int),
    "gemm_f16": ([ctypes.c_void_p] * 3 + [ctypes.c_int64] * 6 + [ctypes.c_void_p],
                 ctypes.c_int),
    "gemm_f16_ex": ([ctypes.c_void_p] * 3 + [ctypes.c_int64] * 6 +
                    [ctypes.c_int, ctypes.c_int, ctypes.c_void_p], ctypes.c_int),
    "gemm_bias_act_f16": ([ctypes.c_void_p] * 4 + [ctypes.c_int64] * 6 +
                          [ctypes.c_int, ctypes.c_int, ctypes.c_void_p], ctypes.c_int),
    "gemm_f16_general": ([ctypes.c_void_p] * 4 + [ctypes.c_int64] * 6 +
                         [ctypes.c_int] * 4 + [ctypes.c_void_p], ctypes.c_int),
    "gemm_f16_config": ([ctypes.c_void_p] * 4 + [ctypes.c_int64] * 6 + [ctypes.c_int] * 3 +
                        [ctypes.POINTER(GemmConfig), ctypes.c_void_p], ctypes.c_int),
    "gemm_config_smem_bytes": ([ctypes.POINTER(GemmConfig)], ctypes.c_int),
    "gemm_config_list": ([ctypes.POINTER(GemmConfig), ctypes.c_int], ctypes.c_int),
    "gemm_auto_config": ([ctypes.c_int64] * 3 + [ctypes.c_int, ctypes.POINTER(GemmConfig)],
                         ctypes.c_int),
    "gemm_select_path": ([ctypes.c_int64] * 3, ctypes.c_int),
    "gemm_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "gemm_get_device_status": ([ctypes.c_void_p, ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
    "gemm_selftest_wait_timeout": ([ctypes.c_int64, ctypes.c_void_p,
                                    ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
    "gemm_abi_version": ([], ctypes.c_int),
    "gemm_activation_f32": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                             ctypes.c_void_p], ctypes.c_int),
    "gemm_relu_f16_noalloc": ([ctypes.c_void_p] * 3 + [ctypes.c_int64] * 6 + [ctypes.c_void_p],
                              ctypes.c_int),
    "gemm_read_probe": ([ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p],
                        ctypes.c_int),
    "gemm_f16_host": ([ctypes.c_void_p] * 4 + [ctypes.c_int64] * 6 +
                      [ctypes.c_int, ctypes.c_void_p], ctypes.c_int),
    "gemm_relu_f16_host": ([ctypes.c_void_p] * 3 + [ctypes.c_int64] * 6 + [ctypes.c_void_p],
                           ctypes.c_int),
    "gemm_host_plan_for": ([ctypes.c_int64] * 3 + [ctypes.POINTER(HostPlan)], ctypes.c_int),
    "gemm_f16_host_planned": ([ctypes.c_void_p] * 4 + [ctypes.c_int64] * 6 +
                              [ctypes.c_int, ctypes.POINTER(HostPlan), ctypes.c_void_p],
                              ctypes.c_int),
    "gemm_host_release": ([], ctypes.c_int),
    "gemm_release": ([], ctypes.c_int),
}


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m tiled_tensor_core_05_b200.build` (there is no CPU fallback)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


def status_string(code: int) -> str:
    return lib().gemm_status_string(int(code)).decode()


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"{what} failed: {status_string(rc)} ({rc})")


def _stream_handle(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ld_padded(t: torch.Tensor) -> int:
    """Row stride in elements.  A single-row matrix has no meaningful stride,
    so its columns rounded up to the 8-element rule are passed instead."""
    if t.dim() != 2:
        raise ValueError("expected a 2-D tensor")
    if t.size(1) > 1 and t.stride(1) != 1:
        raise ValueError("columns must be contiguous (stride(1) == 1)")
    if t.size(0) > 1:
        return int(t.stride(0))
    return (int(t.size(1)) + 7) // 8 * 8


def gemm_f16_ex(a: torch.Tensor, b: torch.Tensor, out: torch.Tensor | None = None, *,
                relu: bool = True, path: int = PATH_AUTO, stream=None) -> torch.Tensor:
    """C = ReLU(A @ B) (relu=True) or A @ B on CUDA fp16 tensors.

    ``a`` is (M, K), ``b`` is (K, N), ``out`` (allocated if None) is (M, N);
    all fp16 on the same CUDA device with contiguous columns.  The call is
    asynchronous on ``stream`` (default: the current stream)."""
    if a.dtype != torch.float16 or b.dtype != torch.float16:
        raise TypeError("a and b must be torch.float16")
    if not (a.is_cuda and b.is_cuda):
        raise ValueError("a and b must be CUDA tensors")
    M, K = a.shape
    K2, N = b.shape
    if K != K2:
        raise ValueError(f"shape mismatch {tuple(a.shape)} @ {tuple(b.shape)}")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=a.device)
    if out.dtype != torch.float16 or tuple(out.shape) != (M, N) or out.device != a.device:
        raise ValueError("out must be an fp16 (M, N) tensor on the device of a")
    dev = a.device
    with torch.cuda.device(dev):
        rc = lib().gemm_f16_ex(a.data_ptr(), b.data_ptr(), out.data_ptr(), M, N, K,
                               _ld_padded(a), _ld_padded(b), _ld_padded(out), int(bool(relu)),
                               int(path), _stream_handle(stream, dev))
    _check(rc, "gemm_f16_ex")
    return out


def gemm_bias_act_f16(a: torch.Tensor, b: torch.Tensor, bias: torch.Tensor | None = None,
                      act: str | int = "gelu", out: torch.Tensor | None = None, *,
                      path: int = PATH_AUTO, stream=None) -> torch.Tensor:
    """C = act(A @ B + bias) with a per-column fp16 bias (or None) and act in
    "none" / "relu" / "gelu" (exact GELU), fused into the GEMM epilogue."""
    if a.dtype != torch.float16 or b.dtype != torch.float16:
        raise TypeError("a and b must be torch.float16")
    M, K = a.shape
    K2, N = b.shape
    if K != K2:
        raise ValueError(f"shape mismatch {tuple(a.shape)} @ {tuple(b.shape)}")
    code = _ACTS[act] if isinstance(act, str) else int(act)
    if bias is not None:
        if bias.dtype != torch.float16 or bias.numel() != N or not bias.is_cuda:
            raise ValueError("bias must be a CUDA fp16 tensor with N elements")
        if bias.dim() != 1 and not bias.is_contiguous():
            raise ValueError("bias must be contiguous")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=a.device)
    dev = a.device
    with torch.cuda.device(dev):
        rc = lib().gemm_bias_act_f16(a.data_ptr(), b.data_ptr(),
                                     None if bias is None else bias.data_ptr(), out.data_ptr(),
                                     M, N, K, _ld_padded(a), _ld_padded(b), _ld_padded(out),
                                     code, int(path), _stream_handle(stream, dev))
    _check(rc, "gemm_bias_act_f16")
    return out


def gemm_general(a: torch.Tensor, b: torch.Tensor, bias: torch.Tensor | None = None,
                 act: str | int = "relu", out: torch.Tensor | None = None, *,
                 trans_a: bool = False, trans_b: bool = False, path: int = PATH_AUTO,
                 stream=None) -> torch.Tensor:
    """C = act(op(A) @ op(B) + bias).  With trans_a the stored ``a`` is K x M
    (op(A) = a.T); with trans_b the stored ``b`` is N x K (op(B) = b.T, the
    layout of a linear layer's weight)."""
    if a.dtype != torch.float16 or b.dtype != torch.float16:
        raise TypeError("a and b must be torch.float16")
    M, K = (a.shape[1], a.shape[0]) if trans_a else tuple(a.shape)
    K2, N = (b.shape[1], b.shape[0]) if trans_b else tuple(b.shape)
    if K != K2:
        raise ValueError("inner dimensions differ")
    code = _ACTS[act] if isinstance(act, str) else int(act)
    if bias is not None and (bias.dtype != torch.float16 or bias.numel() != N):
        raise ValueError("bias must be fp16 with N elements")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=a.device)
    dev = a.device
    with torch.cuda.device(dev):
        rc = lib().gemm_f16_general(a.data_ptr(), b.data_ptr(),
                                    None if bias is None else bias.data_ptr(), out.data_ptr(),
                                    M, N, K, _ld_padded(a), _ld_padded(b), _ld_padded(out),
                                    int(bool(trans_a)), int(bool(trans_b)), code, int(path),
                                    _stream_handle(stream, dev))
    _check(rc, "gemm_f16_general")
    return out


def _as_config(cfg) -> GemmConfig:
    if isinstance(cfg, GemmConfig):
        return cfg
    return GemmConfig(**{k: int(v) for k, v in dict(cfg).items()})


def gemm_config_run(a: torch.Tensor, b: torch.Tensor, cfg, bias: torch.Tensor | None = None,
                    act: str | int = "relu", out: torch.Tensor | None = None, *,
                    trans_a: bool = False, trans_b: bool = False,
                    stream=None) -> torch.Tensor:
    """:func:`gemm_general` with an explicit kernel configuration ``cfg`` (a
    :class:`GemmConfig` or a dict of its fields) instead of a path."""
    if a.dtype != torch.float16 or b.dtype != torch.float16:
        raise TypeError("a and b must be torch.float16")
    M, K = (a.shape[1], a.shape[0]) if trans_a else tuple(a.shape)
    K2, N = (b.shape[1], b.shape[0]) if trans_b else tuple(b.shape)
    if K != K2:
        raise ValueError("inner dimensions differ")
    code = _ACTS[act] if isinstance(act, str) else int(act)
    if bias is not None and (bias.dtype != torch.float16 or bias.numel() != N):
        raise ValueError("bias must be fp16 with N elements")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=a.device)
    c = _as_config(cfg)
    dev = a.device
    with torch.cuda.device(dev):
        rc = lib().gemm_f16_config(a.data_ptr(), b.data_ptr(),
                                   None if bias is None else bias.data_ptr(), out.data_ptr(),
                                   M, N, K, _ld_padded(a), _ld_padded(b), _ld_padded(out),
                                   int(bool(trans_a)), int(bool(trans_b)), code,
                                   ctypes.byref(c), _stream_handle(stream, dev))
    _check(rc, f"gemm_f16_config {c!r}")
    return out


def config_smem_bytes(cfg) -> int:
    """Shared memory per CTA that ``cfg`` needs (negative status if it names
    no kernel)."""
    return int(lib().gemm_config_smem_bytes(ctypes.byref(_as_config(cfg))))


def config_list() -> list[GemmConfig]:
    """The compiled kernel configurations (kernel, block_n, stages)."""
    n = int(lib().gemm_config_list(None, 0))
    arr = (GemmConfig * n)()
    lib().gemm_config_list(arr, n)
    return [GemmConfig(**c.as_dict()) for c in arr]


def auto_config(M: int, N: int, K: int, act: str | int = "relu", device=None) -> GemmConfig:
    """The configuration GEMM_PATH_AUTO takes for this problem on the device."""
    code = _ACTS[act] if isinstance(act, str) else int(act)
    out = GemmConfig()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        _check(lib().gemm_auto_config(M, N, K, code, ctypes.byref(out)), "gemm_auto_config")
    return out


def gemm_relu_f16(a, b, out=None, *, stream=None):
    """C = ReLU(A @ B); see :func:`gemm_f16_ex`."""
    return gemm_f16_ex(a, b, out, relu=True, stream=stream)


def gemm_f16(a, b, out=None, *, stream=None):
    """C = A @ B; see :func:`gemm_f16_ex`."""
    return gemm_f16_ex(a, b, out, relu=False, stream=stream)


def activation_f32(x: torch.Tensor, act: str | int = "gelu", stream=None) -> torch.Tensor:
    """The epilogue activation applied elementwise to a CUDA fp32 tensor."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA float32 tensor")
    code = _ACTS[act] if isinstance(act, str) else int(act)
    y = torch.empty_like(x)
    with torch.cuda.device(x.device):
        _check(lib().gemm_activation_f32(x.data_ptr(), y.data_ptr(), x.numel(), code,
                                         _stream_handle(stream, x.device)),
               "gemm_activation_f32")
    return y


def select_path(M: int, N: int, K: int) -> int:
    return int(lib().gemm_select_path(M, N, K))


def device_status(stream=None, device=None) -> int:
    """Synchronise and return (then clear) the device status word (0 = ok)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    st = ctypes.c_int(0)
    with torch.cuda.device(dev):
        _check(lib().gemm_get_device_status(_stream_handle(stream, dev), ctypes.byref(st)),
               "gemm_get_device_status")
    return int(st.value)


def selftest_wait_timeout(timeout_ns: int, stream=None, device=None) -> int:
    """Run the bounded-wait self test; returns the status word it produced."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    st = ctypes.c_int(0)
    with torch.cuda.device(dev):
        _check(lib().gemm_selftest_wait_timeout(int(timeout_ns), _stream_handle(stream, dev),
                                                ctypes.byref(st)),
               "gemm_selftest_wait_timeout")
    return int(st.value)


def read_probe(buf: torch.Tensor, sink: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Stream-read every byte of the contiguous CUDA tensor ``buf`` once (the
    library's read-bandwidth probe); returns the 1-element int32 ``sink``
    holding the XOR of its 32-bit words."""
    if not buf.is_cuda or not buf.is_contiguous():
        raise ValueError("buf must be a contiguous CUDA tensor")
    if sink is None:
        sink = torch.zeros(1, dtype=torch.int32, device=buf.device)
    n = buf.numel() * buf.element_size()
    with torch.cuda.device(buf.device):
        _check(lib().gemm_read_probe(buf.data_ptr(), n, sink.data_ptr(),
                                     _stream_handle(stream, buf.device)), "gemm_read_probe")
    return sink


def _host_ld(t: torch.Tensor) -> int:
    """Row stride in elements of a 2-D CPU fp16 tensor with contiguous columns
    (any stride >= cols; a single row passes its column count)."""
    if t.dim() != 2 or t.dtype != torch.float16 or t.is_cuda:
        raise ValueError("expected a 2-D CPU float16 tensor")
    if t.size(1) > 1 and t.stride(1) != 1:
        raise ValueError("columns must be contiguous (stride(1) == 1)")
    return int(t.stride(0)) if t.size(0) > 1 else int(t.size(1))


def gemm_host(a: torch.Tensor, b: torch.Tensor, bias: torch.Tensor | None = None,
              act: str | int = "relu", out: torch.Tensor | None = None, *, stream=None,
              sync: bool = True, plan: dict | None = None) -> torch.Tensor:
    """C = act(A @ B + bias) on CPU fp16 tensors (``gemm_f16_host``): the
    library copies A, B and bias to the current CUDA device, runs its kernels
    panel by panel while the copies stream, and copies C back into ``out``.
    Page-locked tensors (``pin_memory()``) let the copies overlap; ``out``
    defaults to a new page-locked tensor.  With ``sync=False`` the call only
    enqueues the work on ``stream``: synchronise it before reading ``out``.
    ``plan`` ({"split": 0 or 1, "panel_extent": n}) replaces the library's
    own split (``gemm_f16_host_planned``)."""
    M, K = a.shape
    K2, N = b.shape
    if K != K2:
        raise ValueError("inner dimensions differ")
    code = _ACTS[act] if isinstance(act, str) else int(act)
    if bias is not None and (bias.dtype != torch.float16 or bias.is_cuda or
                             bias.numel() != N or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous CPU fp16 tensor of N elements")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, pin_memory=True)
    if tuple(out.shape) != (M, N):
        raise ValueError("out must be M x N")
    dev = torch.device("cuda", torch.cuda.current_device())
    h = _stream_handle(stream, dev)
    with torch.cuda.device(dev):
        args = (a.data_ptr(), b.data_ptr(), None if bias is None else bias.data_ptr(),
                out.data_ptr(), M, N, K, _host_ld(a), _host_ld(b), _host_ld(out), code)
        if plan is None:
            _check(lib().gemm_f16_host(*args, h), "gemm_f16_host")
        else:
            p = HostPlan(split=int(plan["split"]), panels=0,
                         panel_extent=int(plan["panel_extent"]), estimate_bytes=0.0)
            _check(lib().gemm_f16_host_planned(*args, ctypes.byref(p), h),
                   "gemm_f16_host_planned")
    if sync:
        if stream is None:
            torch.cuda.current_stream(dev).synchronize()
        elif hasattr(stream, "synchronize"):
            stream.synchronize()
        else:  # a raw handle
            torch.cuda.synchronize(dev)
    return out


def host_plan(M: int, N: int, K: int) -> dict:
    """The split ``gemm_f16_host`` takes for an M x N x K problem (pure host)."""
    p = HostPlan()
    _check(lib().gemm_host_plan_for(M, N, K, ctypes.byref(p)), "gemm_host_plan_for")
    return p.as_dict()


def host_release() -> None:
    """Free the device copies and copy streams ``gemm_host`` keeps."""
    _check(lib().gemm_host_release(), "gemm_host_release")


def release() -> None:
    """Free every device buffer the library keeps (small-M workspaces and the
    host-buffer staging), after waiting for the devices that hold them."""
    _check(lib().gemm_release(), "gemm_release")
