"""GPU parity of the operand layouts (T.gemm's transpose_A / transpose_B of
"Writing high-performance kernels in TileLang", atlascloud.ai blog, section
"Escribamos un GEMM"): A stored K x M and/or B stored N x K, on the three
kernels, against the oracle within |c - ref| <= 1e-2 + 1e-2 |ref|."""
import numpy as np
import pytest
import torch

from gpu_util import GuardedOut, check_parity, dev_to_np, round8, to_dev
from tiled_tensor_core_05_b200 import ops, workloads

pytestmark = pytest.mark.gpu

PATHS = {"tile": ops.PATH_TILE, "pair": ops.PATH_TILE_PAIR, "tall": ops.PATH_TILE_PAIR_TALL,
         "skinny": ops.PATH_SKINNY}
LAYOUTS = [(False, False), (True, False), (False, True), (True, True)]


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()
    assert ops.device_status() == 0


def run(a_st, b_st, bias, act, ta, tb, path, m, n):
    a = to_dev(a_st, round8(a_st.shape[1]) + 8, rows_pad=1)
    b = to_dev(b_st, round8(b_st.shape[1]), rows_pad=1)
    bias_d = None if bias is None else torch.from_numpy(bias).cuda()
    g = GuardedOut(m, n)
    ops.gemm_general(a, b, bias_d, act, g.view, trans_a=ta, trans_b=tb, path=path)
    torch.cuda.synchronize()
    out = dev_to_np(g.view).copy()
    assert g.untouched()
    return out


@pytest.mark.parametrize("ta,tb", LAYOUTS, ids=lambda v: str(int(v)))
@pytest.mark.parametrize("m,n,k", [(200, 300, 150), (33, 1000, 700), (513, 257, 129),
                                   (64, 64, 64), (7, 65, 1000), (1, 7, 3)])
def test_layouts_parity(oracle_mod, ta, tb, m, n, k):
    a, b = workloads.make_inputs(m, n, k, seed=7 * m + n + k)
    rng = np.random.default_rng(m + 3 * n)
    bias = (rng.standard_normal(n)).astype(np.float16)
    a_st = a.T.contiguous() if ta else a
    b_st = b.T.contiguous() if tb else b
    for act in ("relu", "gelu"):
        ref = oracle_mod.gemm_general(a, b, bias, act)
        for name, path in PATHS.items():
            if path == ops.PATH_SKINNY and m > 64:
                continue
            c = run(a_st, b_st, bias, act, ta, tb, path, m, n)
            check_parity(c, ref, act == "relu", f"{name} ta={ta} tb={tb} {act} {m}x{n}x{k}")


@pytest.mark.slow
def test_decode_weights_stored_n_by_k(oracle_mod):
    """The decode shape with B stored N x K (linear-layer weights)."""
    w = workloads.WORKLOADS["decode"]
    a, b = workloads.workload_inputs("decode")
    bt = b.T.contiguous()
    c = ops.gemm_general(a.cuda(), bt.cuda(), None, "relu", trans_b=True)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    rows = rng.integers(0, w.M, 2048)
    cols = rng.integers(0, w.N, 2048)
    ref = oracle_mod.gemm_relu_at(a, b, rows, cols)
    check_parity(dev_to_np(c)[rows, cols], ref, True, "decode B^T sampled")
