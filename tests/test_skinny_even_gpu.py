"""The even small-M schedule (GEMM_PATH_SKINNY_EVEN) against the oracle.

One CTA per SM owns q whole 64-column units of B for the full K; the r
leftover units are split along K over the CTAs and summed by whichever slice
arrives last.  The shapes here are built from the device's SM count P so that
every regime is reached: q = 1..4, no leftover, one leftover unit split into
many slices, many leftover units of one slice each, a ragged last unit (N not
a multiple of 64), a ragged last k-block, M from 1 to 64 (both MMA widths),
the transposed storages, and each epilogue (ReLU, none, bias + GELU).  Every
result is compared element by element with the oracle, with canary bands
around C, and repeated calls must give the same bits (the arrival counters
are left at zero by each call).
"""
import numpy as np
import pytest
import torch

from gpu_util import GuardedOut, check_parity, dev_to_np, to_dev
from tiled_tensor_core_05_b200 import ops, workloads

pytestmark = pytest.mark.gpu
EVEN = ops.PATH_SKINNY_EVEN


def sms() -> int:
    return torch.cuda.get_device_properties(0).multi_processor_count


def cols(q: int, r: int, short: int = 0) -> int:
    """N with q whole units per SM and r leftover units, the last unit
    `short` columns short of 64 (a multiple of 8, so that ld = N is legal)."""
    return 64 * (q * sms() + r) - short


@pytest.mark.parametrize("m", [1, 32, 33, 64])
@pytest.mark.parametrize("q,r,short", [(1, 0, 0), (1, 7, 24), (2, 1, 0), (2, -2, 8), (3, 4, 0),
                                       (3, 4, 40), (3, 0, 56), (4, 2, 56)],
                         ids=["q1", "q1-r7-ragged", "q2-r1", "q2-rP-2", "q3-r4", "q3-r4-ragged",
                              "q3-ragged", "q4-r2-ragged"])
def test_even_relu_against_oracle(oracle_mod, m, q, r, short):
    if r < 0:
        r += sms()  # P - 2 leftover units: one slice each
    n, k = cols(q, r, short), 1000  # 16 k-blocks, the last one 40 deep
    a, b = workloads.make_inputs(m, n, k, seed=100 + 7 * q + r + m, a_scale=1.0 / k ** 0.5)
    ref = oracle_mod.gemm_relu(a, b)
    out = GuardedOut(m, n)
    ops.gemm_f16_ex(to_dev(a), to_dev(b), out.view, relu=True, path=EVEN)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    check_parity(dev_to_np(out.view), ref, True, f"even m={m} n={n} k={k}")
    assert out.untouched(), "write outside C"


def test_even_decode_in_full_and_deterministic(oracle_mod):
    """The decode workload (448 units on 148 SMs: q = 3, 4 leftover units in
    37 slices of 3-4 k-blocks), every element, three calls with equal bits."""
    w = workloads.WORKLOADS["decode"]
    a_cpu, b_cpu = workloads.workload_inputs("decode")
    a, b = a_cpu.cuda(), b_cpu.cuda()
    outs = []
    for _ in range(3):
        c = torch.empty((w.M, w.N), dtype=torch.float16, device="cuda")
        ops.gemm_f16_ex(a, b, c, relu=True, path=EVEN)
        outs.append(c)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    for c in outs[1:]:
        assert torch.equal(c.view(torch.int16), outs[0].view(torch.int16)), "not deterministic"
    ref = oracle_mod.gemm_relu(a_cpu, b_cpu)
    check_parity(dev_to_np(outs[0]), ref, True, "decode, even schedule, in full")


@pytest.mark.parametrize("act", ["none", "relu", "gelu"])
def test_even_bias_and_activations(oracle_mod, act):
    m, n, k = 20, cols(3, 5, 16), 2088
    a, b = workloads.make_inputs(m, n, k, seed=77, a_scale=1.0 / k ** 0.5)
    bias = (np.random.default_rng(5).standard_normal(n) * 0.5).astype(np.float16)
    ref = oracle_mod.gemm_bias_act(a, b, bias, act)
    c = ops.gemm_bias_act_f16(a.cuda(), b.cuda(), torch.from_numpy(bias).cuda(), act, path=EVEN)
    torch.cuda.synchronize()
    check_parity(dev_to_np(c), ref, act == "relu", f"even bias {act}")


@pytest.mark.parametrize("trans_a,trans_b", [(False, True), (True, False), (True, True)])
def test_even_transposed_storage(oracle_mod, trans_a, trans_b):
    m, n, k = 32, cols(2, 3, 8), 1536
    a, b = workloads.make_inputs(m, n, k, seed=78, a_scale=1.0 / k ** 0.5)
    ref = oracle_mod.gemm_relu(a, b)
    a_st = a.T.contiguous() if trans_a else a
    b_st = b.T.contiguous() if trans_b else b
    c = ops.gemm_general(to_dev(a_st), to_dev(b_st), None, "relu", trans_a=trans_a,
                         trans_b=trans_b, path=EVEN)
    torch.cuda.synchronize()
    check_parity(dev_to_np(c), ref, True, f"even trans_a={trans_a} trans_b={trans_b}")


@pytest.mark.parametrize("stages", [4, 5, 6])
def test_even_every_compiled_depth(oracle_mod, stages):
    m, n, k = 32, cols(3, 4), 704  # 11 k-blocks; row strides multiples of 8
    a, b = workloads.make_inputs(m, n, k, seed=79, a_scale=1.0 / k ** 0.5)
    ref = oracle_mod.gemm_relu(a, b)
    c = ops.gemm_config_run(a.cuda(), b.cuda(), {"kernel": EVEN, "stages": stages}, None, "relu")
    torch.cuda.synchronize()
    check_parity(dev_to_np(c), ref, True, f"even stages={stages}")


def test_even_rejects_shapes_it_does_not_cover():
    a = torch.zeros((32, 64), dtype=torch.float16, device="cuda")
    few = torch.zeros((64, 64 * (sms() - 1)), dtype=torch.float16, device="cuda")  # q = 0
    with pytest.raises(RuntimeError):
        ops.gemm_f16_ex(a, few, relu=True, path=EVEN)
    tall = torch.zeros((65, 64), dtype=torch.float16, device="cuda")  # M > 64
    b = torch.zeros((64, 64 * sms() * 2), dtype=torch.float16, device="cuda")
    with pytest.raises(RuntimeError):
        ops.gemm_f16_ex(tall, b, relu=True, path=EVEN)
    with pytest.raises(RuntimeError):  # the width is fixed by the shape
        ops.gemm_config_run(a, b, {"kernel": EVEN, "block_n": 64}, None, "relu")
    torch.cuda.synchronize()
    assert ops.device_status() == 0
