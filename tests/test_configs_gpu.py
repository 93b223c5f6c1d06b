"""GPU parity of every compiled kernel configuration (tile shape x ring depth,
plus raster panels and k-slices) through gemm_f16_config, against the oracle
within |c - ref| <= 1e-2 + 1e-2 |ref| (the check of "Writing high-performance
kernels in TileLang", atlascloud.ai blog, section "Escribamos un GEMM").  The
offline sweep ranks only configurations from this set, so each one it can
report is covered here."""
import numpy as np
import pytest
import torch

from gpu_util import GuardedOut, check_parity, dev_to_np, round8, to_dev
from tiled_tensor_core_05_b200 import ops, workloads

pytestmark = pytest.mark.gpu

CONFIG_ERR = -8


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()
    assert ops.device_status() == 0


def _run(a, b, cfg, bias=None, act="relu", ta=False, tb=False, m=None, n=None):
    a_d = to_dev(a, round8(a.shape[1]) + 8, rows_pad=1)
    b_d = to_dev(b, round8(b.shape[1]), rows_pad=1)
    bias_d = None if bias is None else torch.from_numpy(bias).cuda()
    g = GuardedOut(m, n)
    ops.gemm_config_run(a_d, b_d, cfg, bias_d, act, g.view, trans_a=ta, trans_b=tb)
    torch.cuda.synchronize()
    out = dev_to_np(g.view).copy()
    assert g.untouched(), f"write outside C for {cfg!r}"
    return out


def _ids(c):
    return f"k{c.kernel}-n{c.block_n}-s{c.stages}"


BUILT = ops.config_list()
TILE_KERNELS = (ops.PATH_TILE, ops.PATH_TILE_PAIR, ops.PATH_TILE_PAIR_TALL)
TILE_BUILT = [c for c in BUILT if c.kernel in TILE_KERNELS]
SKINNY_BUILT = [c for c in BUILT if c.kernel == ops.PATH_SKINNY]
# the even small-M schedule's configurations (their width is fixed by the
# shape) are covered, depth by depth, in test_skinny_even_gpu.py
assert all(c.kernel in TILE_KERNELS + (ops.PATH_SKINNY, ops.PATH_SKINNY_EVEN) for c in BUILT)


@pytest.mark.parametrize("cfg", TILE_BUILT, ids=_ids)
def test_tile_configs(oracle_mod, cfg):
    # ragged in every dimension, several tiles of the widest shape, and more
    # k-blocks than the deepest ring
    m, n, k = 777, 600, 1000
    a, b = workloads.make_inputs(m, n, k, seed=41)
    rng = np.random.default_rng(41)
    bias = rng.standard_normal(n).astype(np.float16)
    for act, bb in (("relu", None), ("none", None), ("gelu", bias)):
        ref = oracle_mod.gemm_general(a, b, bb, act)
        c = _run(a, b, cfg.as_dict(), bb, act, m=m, n=n)
        check_parity(c, ref, act == "relu", f"{cfg!r} {act}")


@pytest.mark.parametrize("cfg", TILE_BUILT, ids=_ids)
def test_tile_configs_transposed(oracle_mod, cfg):
    m, n, k = 300, 520, 264
    a, b = workloads.make_inputs(m, n, k, seed=42)
    ref = oracle_mod.gemm_general(a, b, None, "relu")
    c = _run(a.T.contiguous(), b.T.contiguous(), cfg.as_dict(), None, "relu", True, True,
             m=m, n=n)
    check_parity(c, ref, True, f"{cfg!r} transposed")


@pytest.mark.parametrize("group_rows", [1, 128, 256, 512, 1024, 100000,
                                        -1, -256, -512, -768, -100000])
@pytest.mark.parametrize("kernel", [ops.PATH_TILE, ops.PATH_TILE_PAIR, ops.PATH_TILE_PAIR_TALL])
def test_raster_panels(oracle_mod, kernel, group_rows):
    m, n, k = 1300, 1100, 200
    a, b = workloads.make_inputs(m, n, k, seed=43)
    ref = oracle_mod.gemm_relu(a.numpy(), b.numpy())
    cfg = {"kernel": kernel, "group_rows": group_rows}
    c = _run(a, b, cfg, m=m, n=n)
    check_parity(c, ref, True, f"{cfg}")


@pytest.mark.parametrize("kernel,m,n", [(ops.PATH_TILE_PAIR_TALL, 6556, 3278),
                                         (ops.PATH_TILE_PAIR, 4000, 3000)])
@pytest.mark.parametrize("group_rows", [0, 1024, -768])
def test_waves_sweep_k_both_ways(oracle_mod, kernel, m, n, group_rows):
    """Enough tiles for two to three waves of pairs, so that every pair also
    runs units whose k-blocks are loaded from the top down (starting on the
    partial last k-block of K = 200), in panels walked alternately forwards
    and backwards (an odd panel count, the last one partial)."""
    k = 200
    a, b = workloads.make_inputs(m, n, k, seed=47)
    ref = oracle_mod.gemm_relu(a.numpy(), b.numpy())
    cfg = {"kernel": kernel, "group_rows": group_rows}
    c = _run(a, b, cfg, m=m, n=n)
    check_parity(c, ref, True, f"{cfg} {m}x{n}x{k}")


@pytest.mark.parametrize("kernel", [ops.PATH_TILE_PAIR_TALL, ops.PATH_TILE_PAIR])
def test_waves_both_ways_transposed_bias_gelu(oracle_mod, kernel):
    """The same two-way K sweeps with both operands stored transposed (K x M
    and N x K) and the bias + GELU epilogue, over two to three waves."""
    m, n, k = 4000, 3000, 328
    a, b = workloads.make_inputs(m, n, k, seed=48)
    rng = np.random.default_rng(48)
    bias = rng.standard_normal(n).astype(np.float16)
    ref = oracle_mod.gemm_general(a, b, bias, "gelu")
    c = _run(a.T.contiguous(), b.T.contiguous(), {"kernel": kernel}, bias, "gelu", True, True,
             m=m, n=n)
    check_parity(c, ref, False, f"kernel {kernel} transposed bias + gelu {m}x{n}x{k}")


@pytest.mark.parametrize("cfg", SKINNY_BUILT, ids=_ids)
@pytest.mark.parametrize("m", [1, 20, 33, 64])
def test_skinny_configs(oracle_mod, cfg, m):
    n, k = 1000, 2000  # 4 column tiles, 32 k-blocks
    a, b = workloads.make_inputs(m, n, k, seed=44 + m)
    rng = np.random.default_rng(m)
    bias = rng.standard_normal(n).astype(np.float16)
    ref = oracle_mod.gemm_relu(a.numpy(), b.numpy())
    ref_g = oracle_mod.gemm_general(a, b, bias, "gelu")
    tiles = -(-n // cfg.block_n)
    for splits in (0, 1, 2, 3, 7, 18, 32):
        if splits > 1 and splits * tiles > torch.cuda.get_device_properties(0).multi_processor_count:
            continue  # more (tile, slice) items than the split-K workspace holds
        d = dict(cfg.as_dict(), splits=splits)
        c = _run(a, b, d, m=m, n=n)
        check_parity(c, ref, True, f"{d} m={m}")
    c = _run(a, b, dict(cfg.as_dict(), splits=5), bias, "gelu", m=m, n=n)
    check_parity(c, ref_g, False, f"{cfg!r} gelu m={m}")


def test_skinny_splits_are_deterministic_and_agree():
    m, n, k = 32, 512, 4096
    a, b = workloads.make_inputs(m, n, k, seed=45)
    outs = {}
    for s in (1, 2, 4, 8, 16, 64):
        cfg = {"kernel": ops.PATH_SKINNY, "block_n": 256, "splits": s}
        outs[s] = _run(a, b, cfg, m=m, n=n)
        again = _run(a, b, cfg, m=m, n=n)
        assert (outs[s].view(np.uint16) == again.view(np.uint16)).all(), s
    # different slice counts sum in different orders: equal within fp32 rounding
    for s, o in outs.items():
        assert np.allclose(o.astype(np.float32), outs[1].astype(np.float32), rtol=2e-3,
                           atol=2e-3), s


def test_auto_tile_by_activation():
    """With GELU (the longest epilogue) AUTO keeps the double-buffered 256-row
    pair tile up to K = 6144; with ReLU or none it takes the 512-row tile from
    K = 4096."""
    assert ops.auto_config(8192, 14336, 4096, "gelu").kernel == ops.PATH_TILE_PAIR
    assert ops.auto_config(8192, 14336, 6144, "gelu").kernel == ops.PATH_TILE_PAIR_TALL
    for act in ("relu", "none"):
        assert ops.auto_config(8192, 14336, 4096, act).kernel == ops.PATH_TILE_PAIR_TALL
        assert ops.auto_config(8192, 14336, 4095, act).kernel == ops.PATH_TILE_PAIR


@pytest.mark.parametrize("m,n,k,act", [(8192, 1024, 512, "relu"), (1000, 1000, 1000, "relu"),
                                       (40, 3000, 704, "relu"), (4096, 2048, 256, "gelu"),
                                       (200, 104, 64, "none")])
def test_auto_config_is_what_auto_runs(m, n, k, act):
    """The configuration gemm_auto_config reports gives the same bits as
    GEMM_PATH_AUTO (every kernel is deterministic)."""
    a, b = workloads.make_inputs(m, n, k, seed=46)
    a_d, b_d = a.cuda(), b.cuda()
    cfg = ops.auto_config(m, n, k, act)
    assert cfg.kernel in (ops.PATH_TILE, ops.PATH_TILE_PAIR, ops.PATH_TILE_PAIR_TALL,
                          ops.PATH_SKINNY)
    assert cfg.stages > 0 and cfg.block_n > 0
    c1 = ops.gemm_general(a_d, b_d, None, act)
    c2 = ops.gemm_config_run(a_d, b_d, cfg, None, act)
    torch.cuda.synchronize()
    assert torch.equal(c1.view(torch.int16), c2.view(torch.int16))


def _raw(cfg, m=256, n=256, k=128, bias=False, act=ops.ACT_RELU):
    a = torch.randn(m, k, device="cuda").half()
    b = torch.randn(k, n, device="cuda").half()
    c = torch.full((m, n), 7.0, device="cuda", dtype=torch.float16)
    bb = torch.zeros(n, device="cuda", dtype=torch.float16) if bias else None
    conf = None if cfg is None else ops._as_config(cfg)
    import ctypes
    rc = ops.lib().gemm_f16_config(a.data_ptr(), b.data_ptr(),
                                   None if bb is None else bb.data_ptr(), c.data_ptr(), m, n, k,
                                   k, n, n, 0, 0, act,
                                   None if conf is None else ctypes.byref(conf),
                                   torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return rc, bool((c == 7.0).all())


@pytest.mark.parametrize("cfg,m", [
    ({"kernel": 0}, 256),                                  # AUTO is not a kernel
    ({"kernel": 9}, 256),
    ({"kernel": ops.PATH_TILE, "block_n": 32}, 256),
    ({"kernel": ops.PATH_TILE, "stages": 2}, 256),         # not built
    ({"kernel": ops.PATH_TILE, "block_n": 256, "stages": 5}, 256),  # over the budget
    ({"kernel": ops.PATH_TILE_PAIR, "stages": 7}, 256),
    ({"kernel": ops.PATH_TILE_PAIR_TALL, "block_n": 128}, 256),
    ({"kernel": ops.PATH_TILE, "splits": 2}, 256),         # splits: small-M kernel only
    ({"kernel": ops.PATH_SKINNY}, 65),                     # M > 64
    ({"kernel": ops.PATH_SKINNY, "group_rows": 512}, 32),
    ({"kernel": ops.PATH_SKINNY, "splits": 3}, 32),        # 3 > 2 k-blocks
    ({"kernel": ops.PATH_SKINNY, "block_n": 256, "stages": 6}, 32),  # over the budget
    ({"kernel": ops.PATH_SKINNY, "block_n": 128, "stages": 7}, 32),  # past the depth cap
    ({"kernel": ops.PATH_SKINNY, "block_n": 64}, 32),
    ({"kernel": ops.PATH_TILE, "stages": -1}, 256),
])
def test_config_errors_launch_nothing(cfg, m):
    rc, untouched = _raw(cfg, m=m)
    assert rc == CONFIG_ERR, (cfg, rc)
    assert untouched


def test_null_config_is_an_argument_error():
    rc, untouched = _raw(None)
    assert rc == -1 and untouched


def test_skinny_splits_beyond_the_workspace():
    # 512 column tiles: any split would need more (tile, slice) items than SMs
    m, n, k = 16, 512 * 256, 256
    rc, untouched = _raw({"kernel": ops.PATH_SKINNY, "splits": 2}, m=m, n=n, k=k)
    assert rc == CONFIG_ERR and untouched
