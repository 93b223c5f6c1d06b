"""GPU parity of the host-buffer entry points (gemm_f16_host /
gemm_relu_f16_host): CPU fp16 tensors in, CPU fp16 tensor out, the library
copying the operands in and the result out around its kernels, panel by
panel.  Compared element by element with the oracle of the fused GEMM + ReLU
("Writing high-performance kernels in TileLang", atlascloud.ai blog, section
"Escribamos un GEMM") and of the bias + GELU epilogue ("TileLang simplifica la
creación de kernels GPU de alto rendimiento", posicionamiento-web.ar, section
"Fusionar operaciones para reducir viajes a memoria"), with the same
acceptance as the device-pointer entry points.  Cases cover one panel, row
panels and column panels with a ragged last panel, sizes with no 8-element
alignment (the host side has none), padded host strides, pageable and
page-locked memory, K = 0, stream order and the release of the staging.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import check_parity
from tiled_tensor_core_05_b200 import ops, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    ops.lib()
    yield
    torch.cuda.synchronize()
    ops.host_release()
    assert ops.device_status() == 0, "a kernel reported a device-side timeout"


def inputs(M, N, K, seed, scale_b=None):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn((M, K), generator=g).half()
    s = scale_b if scale_b is not None else 1.0 / np.sqrt(max(K, 1))
    b = (torch.randn((K, N), generator=g) * s).half()
    return a, b


def host(x, pinned):
    return x.pin_memory() if pinned else x.clone()


@pytest.mark.parametrize("shape", [(256, 256, 256), (1000, 1000, 1000), (37, 1003, 515),
                                   (1, 9, 3), (130, 70, 1)],
                         ids=["cube256", "ragged1000", "odd", "tiny", "k1"])
@pytest.mark.parametrize("pinned", [True, False], ids=["pinned", "pageable"])
@pytest.mark.parametrize("relu", [True, False])
def test_host_small_full(oracle_mod, shape, pinned, relu):
    M, N, K = shape
    a, b = inputs(M, N, K, seed=M + N + K)
    out = torch.full((M, N), float("nan"), dtype=torch.float16)
    out = out.pin_memory() if pinned else out
    ops.gemm_host(host(a, pinned), host(b, pinned), None, "relu" if relu else "none", out)
    ref = oracle_mod.gemm_relu(a, b) if relu else oracle_mod.gemm(a, b)
    check_parity(out.numpy(), ref, relu, f"host {shape}")


@pytest.mark.parametrize("shape", [(20000, 2048, 1000), (2048, 24000, 520), (40, 70000, 1000)],
                         ids=["row-panels", "col-panels", "col-panels-small-M"])
def test_host_panels_full(oracle_mod, shape):
    """Several panels with a ragged last one, compared in full."""
    M, N, K = shape
    plan = ops.host_plan(M, N, K)
    assert plan["panels"] >= 3
    assert (plan["panels"] - 1) * plan["panel_extent"] < (M if plan["split"] == 0 else N)
    a, b = inputs(M, N, K, seed=11)
    out = ops.gemm_host(a.pin_memory(), b.pin_memory())
    check_parity(out.numpy(), oracle_mod.gemm_relu(a, b), True, f"host panels {shape}")


@pytest.mark.parametrize("shape", [(1000, 1000, 1000), (20000, 2048, 1000), (2048, 24000, 520)],
                         ids=["one-panel", "row-panels", "col-panels"])
def test_host_bias_gelu(oracle_mod, shape):
    M, N, K = shape
    a, b = inputs(M, N, K, seed=21)
    bias = (torch.randn(N, generator=torch.Generator().manual_seed(22)) * 0.5).half()
    out = ops.gemm_host(a.pin_memory(), b.pin_memory(), bias.pin_memory(), "gelu")
    ref = oracle_mod.gemm_bias_act(a, b, bias, "gelu")
    check_parity(out.numpy(), ref, False, f"host bias+gelu {shape}")


def test_host_padded_strides(oracle_mod):
    """Row strides larger than the rows, and not multiples of 8 elements."""
    M, N, K = 300, 200, 150
    a, b = inputs(M, N, K, seed=31)
    abuf = torch.zeros((M, K + 5), dtype=torch.float16).pin_memory()
    bbuf = torch.zeros((K, N + 3), dtype=torch.float16).pin_memory()
    cbuf = torch.full((M, N + 11), 7.0, dtype=torch.float16).pin_memory()
    abuf[:, :K] = a
    bbuf[:, :N] = b
    ops.gemm_host(abuf[:, :K], bbuf[:, :N], out=cbuf[:, :N])
    check_parity(cbuf[:, :N].numpy(), oracle_mod.gemm_relu(a, b), True, "host padded")
    assert (cbuf[:, N:] == 7.0).all(), "wrote outside the M x N window of C"


def test_host_one_panel_matches_device_bits():
    """With one panel the host entry point runs the device path's kernel on the
    same operands: the same bits."""
    a, b = workloads.workload_inputs("ragged1000")
    assert ops.host_plan(1000, 1000, 1000)["panels"] == 1
    got = ops.gemm_host(a.pin_memory(), b.pin_memory())
    dev = ops.gemm_relu_f16(a.cuda(), b.cuda()).cpu()
    assert torch.equal(got.view(torch.int16), dev.view(torch.int16))


def test_host_k_zero():
    M, N = 33, 40
    a = torch.empty((M, 0), dtype=torch.float16)
    b = torch.empty((0, N), dtype=torch.float16)
    bias = torch.linspace(-2, 2, N).half()
    out = ops.gemm_host(a, b, bias, "relu")
    assert torch.equal(out, torch.relu(bias.float()).half().expand(M, N))
    out = ops.gemm_host(a, b, None, "none")
    assert (out.view(torch.int16) == 0).all()


def test_host_stream_order_and_reuse(oracle_mod):
    """Three calls enqueued on a side stream without synchronising in between
    (the staging buffers are reused, and grown for the second): each output
    is right once the stream is synchronised."""
    shapes = [(512, 384, 256), (2048, 1024, 768), (100, 60, 40)]
    s = torch.cuda.Stream()
    cases = []
    for i, (M, N, K) in enumerate(shapes):
        a, b = inputs(M, N, K, seed=40 + i)
        out = torch.empty((M, N), dtype=torch.float16).pin_memory()
        ops.gemm_host(a.pin_memory(), b.pin_memory(), out=out, stream=s, sync=False)
        cases.append((a, b, out))
    s.synchronize()
    for a, b, out in cases:
        check_parity(out.numpy(), oracle_mod.gemm_relu(a, b), True, "host stream order")


def test_host_release_then_reuse(oracle_mod):
    a, b = inputs(300, 260, 140, seed=51)
    ops.gemm_host(a, b)
    ops.host_release()
    out = ops.gemm_host(a.pin_memory(), b.pin_memory())
    check_parity(out.numpy(), oracle_mod.gemm_relu(a, b), True, "host after release")


def test_host_rejects_device_memory():
    a = torch.zeros((64, 64), dtype=torch.float16, device="cuda")
    c = torch.zeros((64, 64), dtype=torch.float16)
    h = int(torch.cuda.current_stream().cuda_stream)
    rc = ops.lib().gemm_relu_f16_host(a.data_ptr(), c.data_ptr(), c.data_ptr(), 64, 64, 64,
                                      64, 64, 64, h)
    assert rc == -1
    rc = ops.lib().gemm_relu_f16_host(c.data_ptr(), c.data_ptr(), a.data_ptr(), 64, 64, 64,
                                      64, 64, 64, h)
    assert rc == -1
    null = ctypes.c_void_p(0)
    assert ops.lib().gemm_relu_f16_host(null, c.data_ptr(), c.data_ptr(), 64, 64, 64, 64, 64,
                                        64, h) == -1


@pytest.mark.parametrize("plan", [{"split": 0, "panel_extent": 1}, {"split": 0, "panel_extent": 700},
                                  {"split": 1, "panel_extent": 8}, {"split": 1, "panel_extent": 1000},
                                  {"split": 1, "panel_extent": 4096}],
                         ids=["rows1", "rows700", "cols8", "cols1000", "cols-whole"])
def test_host_planned(oracle_mod, plan):
    """The caller's plan instead of the library's: one-row panels, panels of
    8 columns (the narrowest the device rows allow), ragged last panels."""
    M, N, K = (12, 96, 200) if plan["panel_extent"] in (1, 8) else (1500, 3000, 300)
    a, b = inputs(M, N, K, seed=61)
    bias = (torch.randn(N, generator=torch.Generator().manual_seed(62)) * 0.5).half()
    out = ops.gemm_host(a.pin_memory(), b.pin_memory(), bias.pin_memory(), "gelu", plan=plan)
    check_parity(out.numpy(), oracle_mod.gemm_bias_act(a, b, bias, "gelu"), False,
                 f"host planned {plan}")


def test_host_release_after_the_callers_stream_is_destroyed(oracle_mod):
    """The staging of a stream the caller has since destroyed is freed (and a
    later call on a new stream works) without the library touching the dead
    handle."""
    from cuda.bindings import runtime as rt
    err, s = rt.cudaStreamCreateWithFlags(1)  # cudaStreamNonBlocking
    assert err == rt.cudaError_t.cudaSuccess
    handle = int(s)
    a, b = inputs(200, 300, 100, seed=71)
    out = torch.empty((200, 300), dtype=torch.float16).pin_memory()
    ops.gemm_host(a.pin_memory(), b.pin_memory(), out=out, stream=handle, sync=False)
    assert rt.cudaStreamSynchronize(s)[0] == rt.cudaError_t.cudaSuccess
    assert rt.cudaStreamDestroy(s)[0] == rt.cudaError_t.cudaSuccess
    check_parity(out.numpy(), oracle_mod.gemm_relu(a, b), True, "host on a raw stream")
    ops.host_release()
    out2 = ops.gemm_host(a.pin_memory(), b.pin_memory())
    check_parity(out2.numpy(), oracle_mod.gemm_relu(a, b), True, "host after the stream died")
