"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Every case draws seeded inputs from ``workloads``, runs ``gemm_relu_f16`` /
``gemm_f16`` on the GPU and compares element by element with the oracle of
the fused GEMM + ReLU ("Writing high-performance kernels in TileLang",
atlascloud.ai blog, section "Escribamos un GEMM"), within the acceptance
tolerance |c - ref| <= 1e-2 + 1e-2 |ref| plus the sign/zero pattern.  Sizes
the oracle finishes in seconds are compared in full; the full-size workloads
are compared on sampled outputs (whole rows, whole columns and random
elements) and checked for invariants everywhere.
"""
import numpy as np
import pytest
import torch

import pins
from gpu_util import GuardedOut, check_parity, dev_to_np, round8, to_dev
from tiled_tensor_core_05_b200 import ops, workloads

pytestmark = pytest.mark.gpu

TILE, SKINNY, PAIR, TALL = ops.PATH_TILE, ops.PATH_SKINNY, ops.PATH_TILE_PAIR, ops.PATH_TILE_PAIR_TALL


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    major, minor = torch.cuda.get_device_capability(0)
    assert (major, minor) == (10, 0), f"needs sm_100 (B200), got sm_{major}{minor}"
    torch.cuda.set_device(0)
    ops.lib()
    yield
    torch.cuda.synchronize()
    assert ops.device_status() == 0, "a kernel reported a device-side timeout"


def run(a_cpu, b_cpu, relu=True, path=ops.PATH_AUTO, lda=None, ldb=None, ldc=None,
        guard=True):
    """Run the CUDA path on CPU fp16 inputs; returns the (M, N) result as numpy."""
    M, K = a_cpu.shape
    N = b_cpu.shape[1]
    a = to_dev(a_cpu, lda if lda is not None else round8(K), rows_pad=1)
    b = to_dev(b_cpu, ldb if ldb is not None else round8(N), rows_pad=1)
    g = GuardedOut(M, N, ld=ldc)
    ops.gemm_f16_ex(a, b, g.view, relu=relu, path=path)
    torch.cuda.synchronize()
    out = dev_to_np(g.view).copy()
    if guard:
        assert g.untouched(), "kernel wrote outside the M x N output window"
    return out


# ------------------------------------------------ small workloads, in full ---

@pytest.mark.parametrize("name", ["cube256", "cube1024", "ragged1000"])
@pytest.mark.parametrize("relu", [True, False])
@pytest.mark.parametrize("path", [ops.PATH_AUTO, TILE, PAIR, TALL],
                         ids=["auto", "tile", "pair", "tall"])
def test_workload_full(oracle_mod, name, relu, path):
    a, b = workloads.workload_inputs(name)
    ref = oracle_mod.gemm_relu(a, b) if relu else oracle_mod.gemm(a, b)
    c = run(a, b, relu=relu, path=path)
    check_parity(c, ref, relu, name)


@pytest.mark.parametrize("name", ["cube256", "ragged1000"])
def test_workload_full_skinny_path(oracle_mod, name):
    """The small-M kernel on the first 64 / 32 rows of the small workloads."""
    a, b = workloads.workload_inputs(name)
    for m in (64, 32, 1):
        ref = oracle_mod.gemm_relu(a[:m], b)
        c = run(a[:m].contiguous(), b, relu=True, path=SKINNY)
        check_parity(c, ref, True, f"{name}[:{m}] small-M")


# ------------------------------------------------ ragged shape grid, both paths ---

EDGE = [1, 7, 63, 64, 65, 127, 128, 129, 200, 257]
GRID = [(m, n, k) for m in EDGE for n in EDGE for k in EDGE
        if (m * 31 + n * 17 + k * 7) % 23 == 0]  # a deterministic ~1/23 sample


@pytest.mark.parametrize("m,n,k", GRID)
@pytest.mark.parametrize("path", [TILE, PAIR, TALL], ids=["tile", "pair", "tall"])
def test_ragged_grid_tile(oracle_mod, m, n, k, path):
    a, b = workloads.make_inputs(m, n, k, seed=1000 + m + 7 * n + 13 * k)
    ref = oracle_mod.gemm_relu(a, b)
    check_parity(run(a, b, path=path), ref, True, f"path {path} {m}x{n}x{k}")


@pytest.mark.parametrize("m,n,k", [(600, 1100, 700), (513, 257, 1030), (2048, 2048, 512),
                                   (4000, 300, 96)])
def test_pair_kernel_multi_tile(oracle_mod, m, n, k):
    """Several pair tiles per CTA pair, ragged in every dimension."""
    a, b = workloads.make_inputs(m, n, k, seed=3000 + m + n + k)
    for relu in (True, False):
        ref = oracle_mod.gemm_relu(a, b) if relu else oracle_mod.gemm(a, b)
        for path in (PAIR, TALL):
            check_parity(run(a, b, relu=relu, path=path), ref, relu, f"{path} {m}x{n}x{k}")


@pytest.mark.parametrize("m,n,k", [(4600, 2300, 520), (8192, 14336, 256), (300, 1000, 130),
                                   (100, 500, 64)])
def test_tall_tile_last_wave_halves(oracle_mod, m, n, k):
    """The 512-row pair tile splits the tiles of a sparse last wave into two
    256-row halves: whole tiles followed by halves (81 and 896 tiles on 74
    pairs), halves only (one wave of 2 or 1 tiles), a ragged last row of
    tiles, and a half entirely below M (100 rows).  Compared in full."""
    a, b = workloads.make_inputs(m, n, k, seed=5000 + m + n + k)
    for relu in (True, False):
        ref = oracle_mod.gemm_relu(a, b) if relu else oracle_mod.gemm(a, b)
        check_parity(run(a, b, relu=relu, path=TALL), ref, relu, f"tall {m}x{n}x{k}")


@pytest.mark.parametrize("m,n,k", [(8192, 14336, 256), (2000, 3000, 300), (4600, 2300, 520),
                                   (300, 1000, 130), (100, 200, 64)])
def test_pair_tile_sparse_last_wave(oracle_mod, m, n, k):
    """The 256-row pair tile on shapes whose last wave holds few tiles (1792
    tiles on 74 pairs, 96, 8, 1), with ragged rows and columns (the last
    column tile of 3000 is 184 columns wide).  Compared in full."""
    a, b = workloads.make_inputs(m, n, k, seed=6000 + m + n + k)
    for relu in (True, False):
        ref = oracle_mod.gemm_relu(a, b) if relu else oracle_mod.gemm(a, b)
        check_parity(run(a, b, relu=relu, path=PAIR), ref, relu, f"pair {m}x{n}x{k}")


def test_pair_tile_transposed_b_and_gelu(oracle_mod):
    """The 256-row pair tile with B stored N x K and bias + GELU on a ragged
    shape (96 tiles, the last column tile 184 columns wide)."""
    m, n, k = 2000, 3000, 304  # row strides of A and of B stored N x K: multiples of 8
    a, b = workloads.make_inputs(m, n, k, seed=6100)
    bias = (np.random.default_rng(61).standard_normal(n) * 0.5).astype(np.float16)
    ref = oracle_mod.gemm_general(a, b, bias, "gelu")
    c = ops.gemm_general(a.cuda(), b.T.contiguous().cuda(), torch.from_numpy(bias).cuda(), "gelu",
                         trans_b=True, path=PAIR)
    torch.cuda.synchronize()
    check_parity(dev_to_np(c), ref, False, "pair, B stored N x K, bias + GELU")
    assert ops.device_status() == 0


@pytest.mark.parametrize("m,n,k", [(m, n, k) for (m, n, k) in GRID if m <= 64] +
                         [(32, 129, 257), (64, 1000, 1000), (7, 4096, 65), (64, 2048, 4099),
                          (32, 256, 8192), (5, 600, 3000), (33, 520, 12000), (1, 64, 70000)])
def test_ragged_grid_skinny(oracle_mod, m, n, k):
    a, b = workloads.make_inputs(m, n, k, seed=2000 + m + 7 * n + 13 * k)
    for relu in (True, False):
        ref = oracle_mod.gemm_relu(a, b) if relu else oracle_mod.gemm(a, b)
        check_parity(run(a, b, relu=relu, path=SKINNY), ref, relu, f"small-M {m}x{n}x{k}")


@pytest.mark.parametrize("path", [TILE, SKINNY, PAIR, TALL])
def test_padded_leading_dimensions(oracle_mod, path):
    m, n, k = 45, 300, 190
    a, b = workloads.make_inputs(m, n, k, seed=5)
    ref = oracle_mod.gemm_relu(a, b)
    c = run(a, b, path=path, lda=k + 26, ldb=n + 20, ldc=n + 36)
    check_parity(c, ref, True, "padded ld")


# ---------------------------------------------------------- pins on the GPU ---

def gpu_fn_for(path):
    def fn(a, b, relu):
        a = torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.float16)))
        b = torch.from_numpy(np.ascontiguousarray(np.asarray(b, dtype=np.float16)))
        if path == SKINNY and a.shape[0] > 64:
            p = TILE
        else:
            p = path
        return run(a, b, relu=relu, path=p)
    return fn


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
@pytest.mark.parametrize("path", [TILE, SKINNY, PAIR, TALL],
                         ids=["tile", "skinny", "pair", "tall"])
def test_pins_on_gpu(pin, path):
    fails = pin(gpu_fn_for(path), exact=False)
    assert not fails, "\n".join(fails[:5])


# ------------------------------------------------ full-size workloads, sampled ---

def sample_points(M, N, rng, n_random=4096, rows=(0,), cols=(0,)):
    rr = [rng.integers(0, M, n_random)]
    cc = [rng.integers(0, N, n_random)]
    for r in rows:
        rr.append(np.full(N, r))
        cc.append(np.arange(N))
    for c in cols:
        rr.append(np.arange(M))
        cc.append(np.full(M, c))
    return np.concatenate(rr).astype(np.int64), np.concatenate(cc).astype(np.int64)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["cube8192", "mlp_up", "decode"])
def test_workload_fullsize_sampled(oracle_mod, name):
    w = workloads.WORKLOADS[name]
    a_cpu, b_cpu = workloads.workload_inputs(name)
    a, b = a_cpu.cuda(), b_cpu.cuda()
    c = torch.empty((w.M, w.N), dtype=torch.float16, device="cuda")
    ops.gemm_relu_f16(a, b, c)          # the launch configuration the benchmark times
    torch.cuda.synchronize()
    c2 = torch.empty_like(c)
    ops.gemm_relu_f16(a, b, c2)
    torch.cuda.synchronize()
    assert torch.equal(c.view(torch.int16), c2.view(torch.int16)), "not deterministic"
    # invariants at every element
    assert not torch.isnan(c).any()
    assert (c >= 0).all()
    assert not (c.view(torch.int16) == -32768).any()
    c_np = dev_to_np(c)
    # whole rows against the oracle: all of them for the small-M workload (C
    # is 32 x 28672), 512 spread over M (first and last included, every
    # 128-row tile sampled) for the large ones
    if w.M <= 64:
        rows_full = np.arange(w.M)
    else:
        rows_full = np.unique(np.round(np.linspace(0, w.M - 1, 512)).astype(np.int64))
        assert len(rows_full) == 512
    ref_rows = oracle_mod.gemm_relu(a_cpu[torch.from_numpy(rows_full)], b_cpu)
    check_parity(c_np[rows_full], ref_rows, True, f"{name} {len(rows_full)} whole rows")
    # and whole columns (first and last: ragged tile edges of the grid) plus
    # 4096 random elements
    rng = np.random.default_rng(w.seed)
    rows, cols = sample_points(w.M, w.N, rng, rows=(), cols=(0, w.N - 1))
    ref = oracle_mod.gemm_relu_at(a_cpu, b_cpu, rows, cols)
    check_parity(c_np[rows, cols], ref, True, f"{name} sampled")
    frac = float((c > 0).float().mean())
    assert 0.45 < frac < 0.55, frac


# --------------------------------------------------------- large extents ---

@pytest.mark.slow
@pytest.mark.parametrize("m,n,k,path", [
    (3, 1 << 21, 16, SKINNY),       # 8192 column tiles of the small-M kernel
    (64, 256, 1 << 20, SKINNY),     # one column tile, 16384 k-blocks in 4 slices
    (70001, 72, 64, ops.PATH_AUTO),  # 274 pair row tiles, ragged M and N
    (70001, 72, 64, TILE),          # 547 single-SM row tiles
    (128, 128, 1 << 20, TILE),      # one tile, 16384 k-blocks
    (128, 128, 1 << 20, PAIR),      # one pair tile (half of its rows past M)
], ids=["skinny-wideN", "skinny-deepK", "auto-tallM", "tile-tallM", "tile-deepK",
        "pair-deepK"])
def test_large_extents(oracle_mod, m, n, k, path):
    """Extents far beyond the workloads in one dimension: 64-bit offsets in
    the epilogues, long k loops, long split-K slices and many tiles; A scaled
    by 1/sqrt(K) so the sums stay of order 1 (fp32 accumulation keeps them
    inside the tolerance at any K)."""
    a_cpu, b_cpu = workloads.make_inputs(m, n, k, seed=k % 1000 + m, a_scale=1.0 / k ** 0.5)
    a, b = a_cpu.cuda(), b_cpu.cuda()
    c = torch.empty((m, n), dtype=torch.float16, device="cuda")
    ops.gemm_f16_ex(a, b, c, relu=True, path=path)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    assert not torch.isnan(c).any() and (c >= 0).all()
    rng = np.random.default_rng(m + n)
    rows, cols = sample_points(m, n, rng, n_random=2048, rows=(0, m - 1), cols=(0, n - 1))
    if len(rows) > 200_000:  # a whole row of the 2M-column case is plenty
        keep = np.concatenate([np.arange(2048), 2048 + rng.choice(len(rows) - 2048, 100_000,
                                                                    replace=False)])
        rows, cols = rows[keep], cols[keep]
    ref = oracle_mod.gemm_relu_at(a_cpu, b_cpu, rows, cols)
    got = dev_to_np(c)[rows, cols]
    check_parity(got, ref, True, f"{m}x{n}x{k} path {path}")


# ------------------------------------------------------------ special cases ---

@pytest.mark.parametrize("path", [ops.PATH_AUTO, TILE, PAIR, TALL])
def test_k_zero_writes_zeros(path):
    a = torch.empty((5, 0), dtype=torch.float16, device="cuda")
    b = torch.empty((0, 9), dtype=torch.float16, device="cuda")
    g = GuardedOut(5, 9)
    ops.gemm_f16_ex(a, b, g.view, relu=False, path=path)
    torch.cuda.synchronize()
    assert (g.view.view(torch.int16) == 0).all()
    assert g.untouched()


def test_empty_output_is_noop():
    a = torch.zeros((0, 16), dtype=torch.float16, device="cuda")
    b = torch.zeros((16, 8), dtype=torch.float16, device="cuda")
    out = torch.empty((0, 8), dtype=torch.float16, device="cuda")
    ops.gemm_relu_f16(a, b, out)


def test_deterministic_bits_both_paths():
    a, b = workloads.make_inputs(64, 3000, 2500, seed=9)
    ad, bd = to_dev(a, round8(2500)), to_dev(b)
    for path in (TILE, SKINNY, PAIR, TALL):
        outs = []
        for _ in range(3):
            outs.append(ops.gemm_f16_ex(ad, bd, relu=True, path=path).view(torch.int16).cpu())
        assert all(torch.equal(outs[0], o) for o in outs[1:]), path


def test_back_to_back_calls_on_two_streams(oracle_mod):
    """Two streams, each with its own small-M workspace, interleaved."""
    a, b = workloads.make_inputs(32, 5000, 3000, seed=21)
    ref = oracle_mod.gemm_relu(a, b)
    ad, bd = a.cuda(), b.cuda()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for i in range(6):
        s = s1 if i % 2 == 0 else s2
        with torch.cuda.stream(s):
            outs.append(ops.gemm_relu_f16(ad, bd))
    torch.cuda.synchronize()
    for o in outs:
        check_parity(dev_to_np(o), ref, True, "two streams")


# ------------------------------------------------------------ error handling ---

def test_misaligned_pointer_rejected():
    a = torch.zeros((16, 24), dtype=torch.float16, device="cuda")
    b = torch.zeros((16, 16), dtype=torch.float16, device="cuda")
    with pytest.raises(RuntimeError, match="aligned"):
        ops.gemm_relu_f16(a[:, 1:17], b)


def test_unaligned_leading_dimension_rejected():
    a = torch.zeros((16, 20), dtype=torch.float16, device="cuda")[:, :16]
    b = torch.zeros((16, 16), dtype=torch.float16, device="cuda")
    with pytest.raises(RuntimeError, match="multiple of 8"):
        ops.gemm_relu_f16(a, b)


def test_host_pointer_rejected():
    lib = ops.lib()
    a = torch.zeros((16, 16), dtype=torch.float16, device="cuda")
    host = torch.zeros((16, 16), dtype=torch.float16)
    rc = lib.gemm_relu_f16(host.data_ptr(), a.data_ptr(), a.data_ptr(), 16, 16, 16, 16, 16, 16,
                           None)
    assert rc == -1


def test_extent_beyond_allocation_rejected():
    lib = ops.lib()
    a = torch.zeros((16, 16), dtype=torch.float16, device="cuda")
    big = 1 << 20
    rc = lib.gemm_relu_f16(a.data_ptr(), a.data_ptr(), a.data_ptr(), big, 16, 16, 16, 16, 16,
                           None)
    assert rc == -1


def test_skinny_path_refuses_large_m():
    a = torch.zeros((65, 16), dtype=torch.float16, device="cuda")
    b = torch.zeros((16, 16), dtype=torch.float16, device="cuda")
    with pytest.raises(RuntimeError, match="invalid argument"):
        ops.gemm_f16_ex(a, b, path=SKINNY)


# ------------------------------------------------------ failure detection ---

def test_bounded_wait_times_out_and_context_survives(oracle_mod):
    """A wait on an mbarrier that nothing arrives on gives up after its limit,
    records the timeout in the status word, and the context stays usable."""
    st = ops.selftest_wait_timeout(50_000_000)  # 50 ms
    assert st != 0 and (st & 0xF000) == 0x1000 and ((st >> 4) & 0xF) == 4, hex(st)
    assert ops.device_status() == 0  # cleared by the read
    a, b = workloads.workload_inputs("cube256")
    check_parity(run(a, b), oracle_mod.gemm_relu(a, b), True, "after timeout")
    assert ops.device_status() == 0


def test_release_frees_the_workspaces_and_later_calls_work(oracle_mod):
    """gemm_release frees the small-M workspace of every (device, stream) that
    has one; the next small-M call allocates a fresh one and is still right."""
    a_cpu, b_cpu = workloads.make_inputs(32, 1000, 1000, seed=3)
    a, b = a_cpu.cuda(), b_cpu.cuda()
    ref = oracle_mod.gemm_relu(a_cpu, b_cpu)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):  # a workspace for this stream
        c = ops.gemm_relu_f16(a, b)
    torch.cuda.synchronize()
    check_parity(dev_to_np(c), ref, True, "before release")
    free0 = torch.cuda.mem_get_info()[0]
    ops.release()
    free1 = torch.cuda.mem_get_info()[0]
    assert free1 - free0 >= 9 << 20, (free0, free1)  # at least that stream's 9.7 MB
    for s in (side, torch.cuda.current_stream()):
        with torch.cuda.stream(s):
            c = ops.gemm_relu_f16(a, b)
        torch.cuda.synchronize()
        check_parity(dev_to_np(c), ref, True, "after release")
    assert ops.device_status() == 0
