"""GPU parity of the fused bias + activation epilogue, act(A @ B + bias).

Against the CPU oracle (fp64 sum + bias, exact GELU via erfc, RNE fp16) on
all three kernels, with the acceptance tolerance |c - ref| <= 1e-2 + 1e-2 |ref|
("TileLang simplifica la creación de kernels GPU de alto rendimiento",
posicionamiento-web.ar, section "Fusionar operaciones para reducir viajes a
memoria", for the epilogue; the tolerance of "Writing high-performance kernels
in TileLang", atlascloud.ai blog, section "Escribamos un GEMM").
"""
import numpy as np
import pytest
import torch

import pins_epilogue as pe
from gpu_util import GuardedOut, check_parity, dev_to_np, round8, to_dev
from tiled_tensor_core_05_b200 import ops, workloads

pytestmark = pytest.mark.gpu

PATHS = {"tile": ops.PATH_TILE, "pair": ops.PATH_TILE_PAIR, "tall": ops.PATH_TILE_PAIR_TALL,
         "skinny": ops.PATH_SKINNY}


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    ops.lib()
    yield
    torch.cuda.synchronize()
    assert ops.device_status() == 0


def run(a_cpu, b_cpu, bias_cpu, act, path):
    M, K = a_cpu.shape
    N = b_cpu.shape[1]
    a = to_dev(a_cpu, round8(K), rows_pad=1)
    b = to_dev(b_cpu, round8(N), rows_pad=1)
    bias = None
    if bias_cpu is not None:
        buf = torch.full((round8(N) + 8,), float("nan"), dtype=torch.float16, device="cuda")
        buf[:N] = torch.as_tensor(np.asarray(bias_cpu, dtype=np.float16)).cuda()
        bias = buf[:N]
    g = GuardedOut(M, N)
    ops.gemm_bias_act_f16(a, b, bias, act, g.view, path=path)
    torch.cuda.synchronize()
    out = dev_to_np(g.view).copy()
    assert g.untouched(), "wrote outside the output window"
    return out


def gpu_fn(path):
    def fn(a, b, bias, act):
        a = torch.from_numpy(np.ascontiguousarray(np.asarray(a, np.float16)))
        b = torch.from_numpy(np.ascontiguousarray(np.asarray(b, np.float16)))
        p = ops.PATH_TILE if (path == ops.PATH_SKINNY and a.shape[0] > 64) else path
        return run(a, b, bias, act, p)
    return fn


@pytest.mark.parametrize("pin", pe.EPILOGUE_PINS, ids=lambda p: p.__name__)
@pytest.mark.parametrize("path", list(PATHS.values()), ids=list(PATHS.keys()))
def test_epilogue_pins_on_gpu(pin, path):
    fails = pin(gpu_fn(path), exact=False)
    assert not fails, "\n".join(fails[:5])


CASES = [(300, 500, 700), (64, 1000, 1000), (32, 777, 4099), (513, 257, 130), (1, 65, 70)]


@pytest.mark.parametrize("m,n,k", CASES)
@pytest.mark.parametrize("act", ["none", "relu", "gelu"])
@pytest.mark.parametrize("with_bias", [True, False], ids=["bias", "nobias"])
def test_bias_act_parity(oracle_mod, m, n, k, act, with_bias):
    a, b = workloads.make_inputs(m, n, k, seed=m + n + k)
    rng = np.random.default_rng(m * n)
    bias = (rng.standard_normal(n) * 2).astype(np.float16) if with_bias else None
    ref = oracle_mod.gemm_bias_act(a, b, bias, act)
    for name, path in PATHS.items():
        if path == ops.PATH_SKINNY and m > 64:
            continue
        c = run(a, b, bias, act, path)
        check_parity(c, ref, act == "relu", f"{name} {act} {m}x{n}x{k}")


def test_k_zero_gives_activation_of_bias():
    n = 40  # a contiguous C needs ldc % 8 == 0
    a = torch.empty((5, 0), dtype=torch.float16, device="cuda")
    b = torch.empty((0, n), dtype=torch.float16, device="cuda")
    bias_h = (np.random.default_rng(0).standard_normal(n) * 3).astype(np.float16)
    bias = torch.from_numpy(bias_h).cuda()
    for act in ("none", "relu", "gelu"):
        out = ops.gemm_bias_act_f16(a, b, bias, act)
        torch.cuda.synchronize()
        want = pe.to_f16_bits(pe.act64(bias_h.astype(np.float64), act)).view(np.float16)
        got = dev_to_np(out)
        check_parity(got, np.broadcast_to(want, got.shape), act == "relu", f"K=0 {act}")


@pytest.mark.slow
def test_mlp_up_gelu_sampled(oracle_mod):
    """The MLP up-projection with a bias and GELU, sampled against the oracle."""
    w = workloads.WORKLOADS["mlp_up"]
    a_cpu, b_cpu = workloads.workload_inputs("mlp_up")
    rng = np.random.default_rng(7)
    bias_h = (rng.standard_normal(w.N) * 0.5).astype(np.float16)
    c = ops.gemm_bias_act_f16(a_cpu.cuda(), b_cpu.cuda(), torch.from_numpy(bias_h).cuda(), "gelu")
    torch.cuda.synchronize()
    c_np = dev_to_np(c)
    # 512 whole rows spread over M, from the oracle's fused bias + GELU
    rows_full = np.unique(np.round(np.linspace(0, w.M - 1, 512)).astype(np.int64))
    ref_rows = oracle_mod.gemm_bias_act(a_cpu[torch.from_numpy(rows_full)], b_cpu, bias_h,
                                        "gelu")
    check_parity(c_np[rows_full], ref_rows, False, "mlp_up gelu 512 whole rows")
    # random elements, built from the oracle's fp64 sums, its own GELU and
    # its own fp16 encoder
    rows = rng.integers(0, w.M, 2048)
    cols = rng.integers(0, w.N, 2048)
    s = oracle_mod.gemm_f64_at(a_cpu, b_cpu, rows, cols) + bias_h.astype(np.float64)[cols]
    ref = oracle_mod.encode_f16(oracle_mod.activation_f64(s, "gelu")).view(np.float16)
    check_parity(c_np[rows, cols], ref, False, "mlp_up gelu sampled")


def test_bias_must_be_aligned():
    a = torch.zeros((16, 16), dtype=torch.float16, device="cuda")
    b = torch.zeros((16, 16), dtype=torch.float16, device="cuda")
    bias = torch.zeros(17, dtype=torch.float16, device="cuda")[1:]
    with pytest.raises(RuntimeError, match="aligned"):
        ops.gemm_bias_act_f16(a, b, bias, "gelu")


def test_gelu_activation_accuracy():
    """The epilogue's GELU (Phi from Abramowitz & Stegun 7.1.26) against fp64
    and against CUDA's erfc-based GELU in fp32: |Phi error| within 1e-6."""
    x64 = torch.linspace(-12, 12, 200001, dtype=torch.float64)
    x = x64.float().cuda()
    y = ops.activation_f32(x, "gelu").double().cpu()
    xf = x.double().cpu()
    ref = xf * 0.5 * torch.special.erfc(-xf / np.sqrt(2.0))
    err = (y - ref).abs()
    assert float((err / xf.abs().clamp(min=1.0)).max()) < 1e-6
    cuda_ref = torch.nn.functional.gelu(x, approximate="none").double().cpu()
    assert float((y - cuda_ref).abs().max()) < 2e-6 * 12
    zero = ops.activation_f32(torch.zeros(4).cuda(), "gelu").cpu()
    assert (zero == 0).all()
    relu = ops.activation_f32(torch.tensor([-1.0, -0.0, 0.0, 2.5, float("nan")]).cuda(), "relu")
    assert relu.cpu().tolist()[:4] == [0.0, 0.0, 0.0, 2.5] and relu.cpu()[4].item() == 0.0
    assert not torch.signbit(relu.cpu()[1])
