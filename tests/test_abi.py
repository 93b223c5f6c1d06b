"""The C-ABI library loads and exports every entry point the header declares;
host-only entry points behave as documented (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gemm_f16.h")


@pytest.fixture(scope="module")
def lib():
    from tiled_tensor_core_05_b200 import build, ops
    build.build()
    return ops.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"GEMM_API\s+[\w\s\*]+?\b(gemm_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"gemm_relu_f16", "gemm_f16", "gemm_f16_ex", "gemm_status_string",
            "gemm_get_device_status", "gemm_selftest_wait_timeout"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_only_the_api_is_exported():
    import subprocess
    from tiled_tensor_core_05_b200 import ops
    out = subprocess.run(["nm", "-D", "--defined-only", ops.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted(line.split()[-1] for line in out.splitlines()
                      if line.split() and line.split()[-2] in ("T", "W"))
    assert set(exported) == set(declared_functions()), exported


def test_status_strings(lib):
    from tiled_tensor_core_05_b200 import ops
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8):
        s = ops.status_string(code)
        assert s and s != "unknown status", code
    assert ops.status_string(12345) == "unknown status"


def test_path_selection(lib):
    from tiled_tensor_core_05_b200 import ops
    # the even schedule is taken only when asked for (it streams B more slowly)
    assert ops.select_path(32, 28672, 8192) == ops.PATH_SKINNY
    assert ops.select_path(32, 14336, 4096) == ops.PATH_SKINNY
    assert ops.select_path(64, 100, 100) == ops.PATH_SKINNY
    assert ops.select_path(65, 100, 100) == ops.PATH_TILE
    assert ops.select_path(1024, 1024, 1024) == ops.PATH_TILE
    assert ops.select_path(8192, 8192, 8192) == ops.PATH_TILE_PAIR_TALL
    # with ReLU the 512-row tile from K = 4096; below, the double-buffered
    # 256-row tile (its epilogue hidden) wins
    assert ops.select_path(8192, 14336, 4096) == ops.PATH_TILE_PAIR_TALL
    assert ops.select_path(5120, 5120, 4096) == ops.PATH_TILE_PAIR_TALL
    assert ops.select_path(8192, 8192, 3072) == ops.PATH_TILE_PAIR
    assert ops.select_path(8192, 8192, 4095) == ops.PATH_TILE_PAIR
    assert ops.select_path(8192, 8192, 4096) == ops.PATH_TILE_PAIR_TALL
    # 20 x 20 tiles of 256: 400 / 74 = 5.4 waves (90 %); 10 x 20 of 512: 2.7 (90 %)
    assert ops.select_path(5120, 5120, 8192) == ops.PATH_TILE_PAIR_TALL
    # 9 x 9 = 81 tiles (55 % of two waves) against 5 x 9 = 45 (61 % of one)
    assert ops.select_path(2304, 2304, 8192) == ops.PATH_TILE_PAIR_TALL
    # 12 x 13 = 156 (70 %) against 6 x 13 = 78 (53 %): keep 256-row tiles
    assert ops.select_path(3072, 3328, 8192) == ops.PATH_TILE_PAIR


def test_abi_version(lib):
    assert lib.gemm_abi_version() >= 10300


def test_argument_errors_are_reported_before_any_device_work(lib):
    # Negative sizes and bad flags are rejected on the host, without touching a GPU.
    null = ctypes.c_void_p(0)
    assert lib.gemm_f16_ex(null, null, null, -1, 4, 4, 8, 8, 8, 1, 0, None) == -1
    assert lib.gemm_f16_ex(null, null, null, 4, 4, 4, 8, 8, 8, 2, 0, None) == -1
    assert lib.gemm_f16_ex(null, null, null, 4, 4, 4, 8, 8, 8, 1, 7, None) == -1
    assert lib.gemm_f16_ex(null, null, null, 1 << 31, 4, 4, 8, 8, 8, 1, 0, None) == -1
    # empty output: a no-op, whatever the pointers
    assert lib.gemm_relu_f16(null, null, null, 0, 5, 5, 8, 8, 8, None) == 0
    assert lib.gemm_f16(null, null, null, 5, 0, 5, 8, 8, 8, None) == 0


def test_host_entry_argument_errors_before_any_device_work(lib):
    null = ctypes.c_void_p(0)
    buf = (ctypes.c_uint16 * 64)()
    assert lib.gemm_f16_host(null, null, null, null, -1, 4, 4, 4, 4, 4, 1, None) == -1
    assert lib.gemm_f16_host(buf, buf, null, buf, 2, 2, 2, 2, 2, 2, 9, None) == -1  # activation
    assert lib.gemm_relu_f16_host(null, null, null, 0, 5, 5, 5, 5, 5, None) == 0    # empty
    assert lib.gemm_relu_f16_host(null, null, null, 5, 0, 5, 5, 5, 5, None) == 0
    assert lib.gemm_relu_f16_host(null, buf, buf, 2, 2, 2, 2, 2, 2, None) == -1      # null A
    assert lib.gemm_relu_f16_host(buf, buf, buf, 2, 4, 4, 3, 4, 4, None) == -1       # lda < K
    assert lib.gemm_relu_f16_host(buf, buf, buf, 2, 4, 4, 4, 4, 3, None) == -1       # ldc < N
    assert lib.gemm_relu_f16_host(buf, buf, buf, 1 << 31, 4, 4, 4, 4, 4, None) == -1


PLAN_SHAPES = [(M, N, K) for M in (1, 32, 300, 1000, 4096, 8192, 20000)
               for N in (1, 256, 1000, 14336, 28672) for K in (0, 64, 1000, 8192)]


def test_host_plan_invariants(lib):
    """The host-buffer plan: whole 512-row / 256-column panels (column panels
    at least 2048 wide), 1 to 16 of
    them covering the split dimension exactly, an estimate that follows its
    formula, never above the serial copy and never below either direction's
    bytes."""
    from tiled_tensor_core_05_b200 import ops
    for M, N, K in PLAN_SHAPES:
        p = ops.host_plan(M, N, K)
        by_rows = p["split"] == ops.HOST_SPLIT_ROWS
        dim, unit = (M, 512) if by_rows else (N, 256)
        P, ext = p["panels"], p["panel_extent"]
        assert 1 <= P <= 16, (M, N, K, p)
        assert ext % unit == 0 or ext == dim, (M, N, K, p)
        assert by_rows or ext >= 2048 or ext == dim, (M, N, K, p)
        assert (P - 1) * ext < dim <= P * ext, (M, N, K, p)
        a, b, c = 2.0 * M * K, 2.0 * K * N, 2.0 * M * N
        first, streamed = (b, a) if by_rows else (a, b)
        est = max(first + streamed + c / P, first + streamed / P + c)
        assert p["estimate_bytes"] == pytest.approx(est, rel=1e-12), (M, N, K, p)
        assert max(a + b, c) <= est * (1 + 1e-12) and est <= (a + b + c) * (1 + 1e-12)


def test_host_plan_on_the_workloads(lib):
    from tiled_tensor_core_05_b200 import ops
    # the cube: B whole, A and C in 8 panels of 1024 rows (the split is a tie)
    p = ops.host_plan(8192, 8192, 8192)
    assert (p["split"], p["panels"], p["panel_extent"]) == (ops.HOST_SPLIT_ROWS, 8, 1024)
    assert p["estimate_bytes"] == 2 * 8192 * 8192 * 2 + 8192 * 8192 * 2 / 8
    # the MLP up-projection: C (224 MiB) dominates; A (64 MiB) whole first,
    # then 2048-column panels (the narrowest column panel)
    p = ops.host_plan(8192, 14336, 4096)
    assert (p["split"], p["panels"], p["panel_extent"]) == (ops.HOST_SPLIT_COLS, 7, 2048)
    # decode: B is nearly everything; streamed in column panels behind A
    p = ops.host_plan(32, 28672, 8192)
    assert (p["split"], p["panels"], p["panel_extent"]) == (ops.HOST_SPLIT_COLS, 14, 2048)
    # small problems: one panel
    assert ops.host_plan(1000, 1000, 1000)["panels"] == 1
    assert ops.host_plan(1, 1, 0)["panels"] == 1
    for bad in ((0, 4, 4), (4, 0, 4), (4, 4, -1)):
        with pytest.raises(RuntimeError):
            ops.host_plan(*bad)


def test_host_planned_rejects_bad_plans_before_device_work(lib):
    from tiled_tensor_core_05_b200 import ops
    buf = (ctypes.c_uint16 * 64)()
    null = ctypes.c_void_p(0)

    def call(split, extent, M=4, N=100):
        p = ops.HostPlan(split=split, panels=0, panel_extent=extent, estimate_bytes=0.0)
        return lib.gemm_f16_host_planned(buf, buf, null, buf, M, N, 4, 4, N, N, 1,
                                         ctypes.byref(p), None)
    assert call(2, 8) == -8                 # no such split
    assert call(0, 0) == -8                 # empty panels
    assert call(1, 12) == -8                # column panels must keep 16-byte device rows
    assert call(0, 1, M=17) == -8           # 17 panels
    assert lib.gemm_f16_host_planned(buf, buf, null, buf, 4, 4, 4, 4, 4, 4, 1, None, None) == -1
