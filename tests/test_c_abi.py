"""The boundary as a C consumer sees it: `tests/c_abi_check.c` includes
include/gemm_f16.h as strict C99 (-pedantic -Wall -Wextra -Werror), references
every entry point, links against the built library and runs the host-only
calls, here without a GPU."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi_check.c")
HEADER = os.path.join(ROOT, "include", "gemm_f16.h")


@pytest.fixture(scope="module")
def program(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    from tiled_tensor_core_05_b200 import build, ops
    build.build()
    out = str(tmp_path_factory.mktemp("cabi") / "c_abi_check")
    libdir = os.path.dirname(ops.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"), SRC, "-o", out, ops.LIB_PATH,
                    f"-Wl,-rpath,{libdir}"], check=True, capture_output=True, text=True)
    return out


def test_every_declared_entry_point_is_referenced():
    declared = set(re.findall(r"GEMM_API\s+[\w\s\*]+?\b(gemm_\w+)\s*\(", open(HEADER).read()))
    used = set(re.findall(r"\(any_fn\)(gemm_\w+)", open(SRC).read()))
    assert declared == used, (declared - used, used - declared)


def test_c_program_links_and_runs(program):
    from tiled_tensor_core_05_b200 import ops
    r = subprocess.run([program], check=True, capture_output=True, text=True)
    lines = dict(line.split(" ", 1) for line in r.stdout.strip().splitlines())
    declared = set(re.findall(r"GEMM_API\s+[\w\s\*]+?\b(gemm_\w+)\s*\(", open(HEADER).read()))
    assert lines["entry_points"] == f"{len(declared)} missing 0"
    assert int(lines["abi"]) >= 10300
    assert lines["path_cube"] == f"{ops.PATH_TILE_PAIR_TALL} path_decode {ops.PATH_SKINNY}"
    assert lines["plan"] == "rc 0 split 0 panels 8 extent 1024"
    smem, configs = lines["smem"].split(" configs ")
    assert 0 < int(smem) <= 232448 and int(configs) == len(ops.config_list())
    assert lines["bad_size"] == "-1 empty 0"
    assert lines["status"].startswith("pointer not 16-byte aligned")
