"""Host side of the offline configuration sweep: the candidate space, its
pruning by the shared-memory budget, and agreement between the budget and the
set of compiled kernels (no GPU needed)."""
import pytest

from tiled_tensor_core_05_b200 import ops, tune

BUDGET = 232448


@pytest.fixture(scope="module")
def lib():
    from tiled_tensor_core_05_b200 import build
    build.build()
    return ops.lib()


def test_built_configs_are_exactly_those_within_the_budget(lib):
    built = {(c.kernel, c.block_n, c.stages) for c in ops.config_list()}
    kinds = tune.TILE_KINDS + [(ops.PATH_SKINNY, w) for w in tune.SKINNY_WIDTHS] + \
        [(ops.PATH_SKINNY_EVEN, w) for w in tune.EVEN_WIDTHS]
    expect = set()
    for kernel, bn in kinds:
        for st in range(3, 17):
            if ops.config_smem_bytes({"kernel": kernel, "block_n": bn, "stages": st}) > BUDGET:
                continue
            if kernel == ops.PATH_SKINNY and st > 6:  # the small-M ring's depth cap
                continue
            if kernel == ops.PATH_SKINNY_EVEN and st not in tune.EVEN_STAGES:
                continue
            expect.add((kernel, bn, st))
    assert built == expect
    # the defaults are among them
    for kernel, bn, st in ((1, 64, 4), (1, 128, 6), (1, 256, 4), (3, 256, 6), (4, 256, 4),
                           (2, 256, 4), (2, 128, 6)):
        assert (kernel, bn, st) in built


def test_smem_formula(lib):
    # ring + 4 warps x 2 staging boxes of 32 x 64 fp16 + barriers + slack
    def tile(stage, st):
        return 1024 + st * stage + 4 * 2 * 32 * 64 * 2 + (2 * st + 5) * 8 + 16
    assert ops.config_smem_bytes({"kernel": 1, "block_n": 128, "stages": 6}) == tile(32768, 6)
    assert ops.config_smem_bytes({"kernel": 1, "block_n": 256, "stages": 4}) == tile(49152, 4)
    assert ops.config_smem_bytes({"kernel": 3, "stages": 6}) == tile(32768, 6)
    assert ops.config_smem_bytes({"kernel": 4, "stages": 4}) == tile(49152, 4)
    assert ops.config_smem_bytes({"kernel": 2, "block_n": 256, "stages": 5}) == \
        1024 + 5 * 40960 + 13 * 8 + 16
    assert ops.config_smem_bytes({"kernel": 2, "block_n": 128, "stages": 6}) == \
        1024 + 6 * 24576 + 15 * 8 + 16
    # the even small-M schedule: max(q, 2) slabs of 8 KiB of B + 8 KiB of A per stage
    assert ops.config_smem_bytes({"kernel": 5, "block_n": 192, "stages": 6}) == \
        1024 + 6 * (3 * 8192 + 8192) + 16 * 8 + 16
    assert ops.config_smem_bytes({"kernel": 5, "block_n": 64, "stages": 4}) == \
        1024 + 4 * (2 * 8192 + 8192) + 12 * 8 + 16
    assert ops.config_smem_bytes({"kernel": 5, "block_n": 96, "stages": 4}) == -8
    assert ops.config_smem_bytes({"kernel": 2, "block_n": 64, "stages": 4}) == -8
    assert ops.config_smem_bytes({"kernel": 2, "stages": 4}) == -8  # width must be given
    # defaults when stages = 0; AUTO and bad widths name no kernel
    assert ops.config_smem_bytes({"kernel": 3}) == tile(32768, 6)
    assert ops.config_smem_bytes({"kernel": 0}) == -8
    assert ops.config_smem_bytes({"kernel": 1, "block_n": 0}) == -8
    assert ops.config_smem_bytes({"kernel": 1, "block_n": 32}) == -8
    assert ops.config_smem_bytes({"kernel": 1, "block_n": 64, "stages": 8}) == tile(24576, 8)
    assert ops.config_smem_bytes({"kernel": 4, "block_n": 128}) == -8


def test_status_string_for_config_errors(lib):
    assert "configuration" in ops.status_string(-8)


def test_candidates_cube(lib):
    kept, pruned = tune.candidates(8192, 8192, 8192, 148, ops.config_smem_bytes)
    built = {(c.kernel, c.block_n, c.stages) for c in ops.config_list()}
    # every kept candidate has a compiled kernel; every pruned one is over budget
    assert all((c["kernel"], c["block_n"], c["stages"]) in built for c in kept)
    assert all("shared memory" in why for _, why in pruned)
    assert len({tuple(sorted(c.items())) for c in kept}) == len(kept)
    # panels: 1, 2, 4, ... tile-rows up to the whole column (64 rows of 128)
    panels = sorted({c["group_rows"] for c in kept
                     if c["kernel"] == ops.PATH_TILE and c["block_n"] == 128})
    assert panels == [128 * g for g in (1, 2, 4, 8, 16, 32, 64)]
    tall = sorted({c["group_rows"] for c in kept if c["kernel"] == ops.PATH_TILE_PAIR_TALL})
    assert tall == [512 * g for g in (1, 2, 4, 8, 16)]
    assert not any(c["kernel"] == ops.PATH_SKINNY for c in kept)


def test_candidates_small_m(lib):
    built = {(c.kernel, c.block_n, c.stages) for c in ops.config_list()}
    kept, pruned = tune.candidates(32, 4096, 8192, 148, ops.config_smem_bytes, built=built)
    sk = [c for c in kept if c["kernel"] == ops.PATH_SKINNY and c["block_n"] == 256]
    # 16 column tiles of 256: up to 9 slices fit 148 items; 128 k-blocks
    assert sorted({c["splits"] for c in sk}) == [0, 1, 2, 3, 4, 6, 8]
    assert {c["stages"] for c in sk} == {3, 4, 5}
    sk128 = [c for c in kept if c["kernel"] == ops.PATH_SKINNY and c["block_n"] == 128]
    # 32 column tiles of 128: up to 4 slices
    assert sorted({c["splits"] for c in sk128}) == [0, 1, 2, 3, 4]
    assert {c["stages"] for c in sk128} == {3, 4, 5, 6}
    assert any("depth cap" in why for _, why in pruned)
    # tile kernels have a single tile-row: one panel each
    assert all(c["group_rows"] == tune.TILE_ROWS[c["kernel"]] for c in kept
               if c["kernel"] != ops.PATH_SKINNY)
    # decode: 112 column tiles leave no room for a second slice
    kept, _ = tune.candidates(32, 28672, 8192, 148, ops.config_smem_bytes)
    assert sorted({c["splits"] for c in kept if c["kernel"] == ops.PATH_SKINNY}) == [0, 1]


def test_describe():
    assert tune.describe({"kernel": 4, "block_n": 256, "stages": 4, "group_rows": 2048,
                          "splits": 0}) == "pair-tall 512x256 st4 panel=2048"
    assert tune.describe({"kernel": 2, "block_n": 256, "stages": 5, "group_rows": 0,
                          "splits": 0}) == "skinny 256 st5 splits=auto"


def test_host_plan_candidates():
    from tiled_tensor_core_05_b200 import ops, tune
    c = tune.host_plan_candidates(8192, 8192)
    assert {"split": ops.HOST_SPLIT_ROWS, "panel_extent": 512} in c
    assert {"split": ops.HOST_SPLIT_COLS, "panel_extent": 8192} in c
    assert len(c) == len({(p["split"], p["panel_extent"]) for p in c})
    for M, N in ((8192, 14336), (32, 28672), (1000, 1003), (7, 9)):
        for p in tune.host_plan_candidates(M, N):
            dim = M if p["split"] == ops.HOST_SPLIT_ROWS else N
            assert 1 <= p["panel_extent"] <= dim
            assert -(-dim // p["panel_extent"]) <= 16
            if p["split"] == ops.HOST_SPLIT_COLS and p["panel_extent"] < dim:
                assert p["panel_extent"] % 8 == 0
    # decode: 1024-column panels would be 28 of them; rows collapse to one panel
    d = tune.host_plan_candidates(32, 28672)
    assert {"split": ops.HOST_SPLIT_COLS, "panel_extent": 1024} not in d
    assert [p for p in d if p["split"] == ops.HOST_SPLIT_ROWS] == [
        {"split": ops.HOST_SPLIT_ROWS, "panel_extent": 32}]


def test_candidates_decode_include_the_even_schedule(lib):
    kept, _ = tune.candidates(32, 28672, 8192, 148, ops.config_smem_bytes)
    even = [c for c in kept if c["kernel"] == ops.PATH_SKINNY_EVEN]
    # 448 units of 64 columns on 148 SMs: 3 whole units per CTA
    assert {c["block_n"] for c in even} == {192}
    within = {st for st in tune.STAGE_RANGE
              if ops.config_smem_bytes({"kernel": 5, "block_n": 192, "stages": st}) <= BUDGET}
    assert {c["stages"] for c in even} == within
    kept, _ = tune.candidates(32, 4096, 8192, 148, ops.config_smem_bytes)
    assert not [c for c in kept if c["kernel"] == ops.PATH_SKINNY_EVEN]  # 64 units < 148
