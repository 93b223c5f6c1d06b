"""The column-sharded product on the GPU with the library's kernels, every
rank of a `world` emulated in turn in one process (no rank waits for another;
each writes its own columns of one output), against the oracle within
|c - ref| <= 1e-2 + 1e-2 |ref|."""
import numpy as np
import pytest
import torch

from gpu_util import check_parity, dev_to_np
from tiled_tensor_core_05_b200 import shard, workloads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 3, 8])
@pytest.mark.parametrize("m,n,k,act", [(32, 4096, 2048, "relu"), (48, 3000, 1024, "gelu"),
                                       (300, 2560, 512, "relu")])
def test_sharded_columns(oracle_mod, world, m, n, k, act):
    a, b = workloads.make_inputs(m, n, k, seed=70 + world, a_scale=1.0 / k ** 0.5)
    rng = np.random.default_rng(world)
    bias = rng.standard_normal(n).astype(np.float16)
    a_d, b_d = a.cuda(), b.cuda()
    bias_d = torch.from_numpy(bias).cuda()
    out = torch.full((m, n), float("nan"), dtype=torch.float16, device="cuda")
    for r in range(world):
        blk = shard.gemm_sharded(a_d, b_d, bias=bias_d, act=act, out=out, rank=r, world=world)
        n0, n1 = shard.column_range(n, world, r)
        assert blk.shape == (m, n1 - n0)
    torch.cuda.synchronize()
    ref = oracle_mod.gemm_general(a, b, bias, act)
    check_parity(dev_to_np(out), ref, act == "relu", f"sharded {world} {m}x{n}x{k} {act}")
