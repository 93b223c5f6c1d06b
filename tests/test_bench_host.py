"""Host-side logic of bench.py that needs no GPU: the unit of each workload,
the roofline arithmetic and the traffic lookup, the clock summary, and the
JSON line of the reference arm (the CPU oracle) on a small workload."""
import io
import json
import os
import sys
import time
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from tiled_tensor_core_05_b200 import workloads  # noqa: E402
from tiled_tensor_core_05_b200.clocks import ClockSampler  # noqa: E402


@pytest.fixture(scope="module")
def lib():
    from tiled_tensor_core_05_b200 import build, ops
    build.build()
    return ops.lib()


def test_units_follow_the_shape():
    for name, w in workloads.WORKLOADS.items():
        assert bench.hbm_bound(w) == (w.M <= 64), name


def test_roofline_arithmetic(lib):
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    w = workloads.WORKLOADS["cube8192"]
    r = bench.roofline_entry("cube8192", 1.0, peaks, "measured", long_run=False)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(w.flops / 1e-3 / 1e12, rel=1e-4)
    assert r["frac"] == pytest.approx(r["achieved"] / 1600.0, rel=1e-3)
    assert r["kernel"] == "tile_pair_gemm_kernel"
    r = bench.roofline_entry("cube8192", 1.0, peaks, "measured", long_run=True)
    assert r["peak"] == 1400.0
    d = workloads.WORKLOADS["decode"]
    r = bench.roofline_entry("decode", 0.1, peaks, "measured", long_run=False)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(d.bytes_min / 1e-4 / 1e9, rel=1e-4)
    assert d.bytes_min == 472121344
    assert r["kernel"] == "skinny_gemm_kernel"


def test_traffic_is_reported_only_for_the_captured_source(lib, tmp_path, monkeypatch):
    entry = bench.traffic_for("cube8192", "tile_pair_gemm_kernel")
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    rec = table["tile_pair_gemm_kernel/cube8192"]
    if rec["kernel_src_sha"] == bench.kernel_source_hash("tile_pair_gemm_kernel"):
        assert entry == rec["dram_bytes_per_launch"]
    else:
        assert entry is None
    # a changed source (another hash) hides the figure
    monkeypatch.setattr(bench, "kernel_source_hash", lambda k: "0" * 16)
    assert bench.traffic_for("cube8192", "tile_pair_gemm_kernel") is None
    assert bench.traffic_for("cube256", "tile_gemm_kernel") is None  # never captured


def test_traffic_is_keyed_by_variant(tmp_path, monkeypatch):
    """A variant's line reads its own capture, never the plain ReLU one."""
    table = {"k/w": {"kernel_src_sha": "s", "dram_bytes_per_launch": 1},
             "k/w/bias_gelu": {"kernel_src_sha": "s", "dram_bytes_per_launch": 2}}
    os.makedirs(tmp_path / "profiles")
    with open(tmp_path / "profiles" / "traffic.json", "w") as f:
        json.dump(table, f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda k: "s")
    assert bench.traffic_for("w", "k") == 1
    assert bench.traffic_for("w", "k", "relu") == 1
    assert bench.traffic_for("w", "k", "bias_gelu") == 2
    assert bench.traffic_for("w", "k", "wT") is None


def _sampler(samples, marks):
    s = ClockSampler.__new__(ClockSampler)
    s.samples, s.marks, s.ok, s.max_mhz = samples, marks, True, 1965
    s.bits = [(name, 1 << i) for i, (name, _) in enumerate(ClockSampler.REASONS)]
    return s


def test_clock_summary_window_and_reasons():
    t = 100.0
    # (time, MHz, reason bits, W): power cap (bit 3) inside the window only
    samples = [(t + 0.001 * i, 1965 if i < 10 else 1300, (1 << 3) if i >= 10 else 0, 500.0)
               for i in range(30)]
    s = _sampler(samples, {"warm0": t, "t0": t + 0.0095, "t1": t + 0.0295})
    out = s.summary()
    assert out["sm_mhz"] == 1300 and out["samples"] == 20
    assert out["reasons"] == ["sw_power_cap"]
    # a timed region too short for three samples falls back to warm-up + timed
    s = _sampler(samples, {"warm0": t, "t0": t + 0.0155, "t1": t + 0.0165})
    out = s.summary()
    assert out["samples"] == 17 and "warm-up" in out["note"]


def test_clock_summary_without_nvml():
    s = ClockSampler.__new__(ClockSampler)
    s.ok, s.err = False, "no NVML here"
    out = s.summary()
    assert out["sm_mhz"] is None and "NVML unavailable" in out["note"]


def test_reference_arm_line(monkeypatch):
    class Args:
        workload, steps, warmup, gpus = "cube256", 2, 1, 1
    monkeypatch.setenv("RANK", "0")
    buf = io.StringIO()
    t0 = time.time()
    with redirect_stdout(buf):
        assert bench.run_reference(Args) == 0
    assert time.time() - t0 < 60
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["config"]["workload"] == "cube256" and line["gpu_launches"] == 0
    assert line["higher_is_better"] is True and line["dtype"] == "f64"


def test_parity_summary():
    import numpy as np
    ref = np.array([[0.0, 1.0, 2.0], [0.5, 0.0, 100.0]], dtype=np.float16)
    s = bench.parity_summary(ref.copy(), ref)
    assert s["pass"] and s["out_of_tolerance"] == 0 and s["max_abs_err"] == 0.0
    assert s["elements"] == 6
    got = ref.copy()
    got[1, 2] = 100.5             # 0.5 off at |ref| = 100: within 1e-2 + 1e-2 * 100
    s = bench.parity_summary(got, ref)
    assert s["pass"] and s["max_abs_err"] == 0.5 and abs(s["max_rel_err"] - 0.005) < 1e-12
    got[0, 1] = 1.5               # 0.5 off at 1.0: out of tolerance
    s = bench.parity_summary(got, ref)
    assert not s["pass"] and s["out_of_tolerance"] == 1
    got = ref.copy()
    got[1, 0] = 0.0               # a positive reference value clamped away
    s = bench.parity_summary(got, ref)
    assert not s["pass"] and s["sign_mismatches"] == 1
    got = ref.copy()
    got[0, 0] = np.nan
    assert not bench.parity_summary(got, ref)["pass"]


def test_parity_summary_gelu_signs():
    """GELU output may be negative: only the sign pattern where |ref| > 1e-2
    and the tolerance count, not got >= 0."""
    import numpy as np
    ref = np.array([-0.17, -0.005, 0.0, 0.8], dtype=np.float16)
    s = bench.parity_summary(ref.copy(), ref, relu=False)
    assert s["pass"]
    assert not bench.parity_summary(ref.copy(), ref, relu=True)["pass"]  # negatives
    got = ref.copy()
    got[0] = 0.0                  # -0.17 lost its sign (and is 0.17 off)
    s = bench.parity_summary(got, ref, relu=False)
    assert not s["pass"] and s["sign_mismatches"] == 1


@pytest.mark.parametrize("M,n", [(32, 512), (1000, 512), (8192, 256), (8192, 512), (2, 2)])
def test_parity_rows_cover_every_tile_row(M, n):
    rows = bench.parity_rows(M, n)
    assert rows == sorted(set(rows)) and rows[0] == 0 and rows[-1] == M - 1
    assert len(rows) == min(M, n)
    # every 128-row tile (the smallest tile height of the kernels) is sampled
    # when there are at least as many samples as tiles
    if n >= -(-M // 128):
        assert {r // 128 for r in rows} == set(range(-(-M // 128)))


def _fake_res(name, variant, ms):
    return {"w": workloads.WORKLOADS[name], "variant": variant, "launch_ms": ms}


def test_per_workload_records_fit_the_drivers_tail():
    """The short per-workload table ends the bench line and must fit, whole,
    in the last 1500 characters that the driver keeps of it."""
    peaks = {"hbm_gbs": 6532.5, "bf16_tflops": 1672.3, "bf16_tflops_sustained": 1370.4}
    res = [_fake_res("cube8192", "relu", 0.73226), _fake_res("mlp_up", "relu", 0.65612),
           _fake_res("decode", "relu", 0.07163), _fake_res("cube1024", "relu", 0.00915),
           _fake_res("ragged1000", "relu", 0.00913), _fake_res("cube256", "relu", 0.00716),
           _fake_res("mlp_up", "bias_gelu", 0.71361), _fake_res("decode", "wT", 0.07597)]
    recs = [bench.compact_record(r, peaks, "measured") for r in res]
    for rec, r in zip(recs, res):
        rec["traffic"] = 1004495616
        rec["frac_probe"] = 0.9347
        rec["parity"] = bench.parity_text({"pass": True, "out_of_tolerance": 0,
                                           "sign_mismatches": 0, "rows": 512}, r["w"].M)
    text = json.dumps({"configs": recs}, separators=(",", ":"))
    assert len(text) < 1450, len(text)
    assert recs[2]["unit"] == "GB/s" and recs[0]["unit"] == "TFLOP/s"
    assert recs[0]["value"] == pytest.approx(1501.5, abs=0.1)
    assert recs[1]["parity"] == "pass 512/8192 rows"
    bad = bench.parity_text({"pass": False, "out_of_tolerance": 3, "sign_mismatches": 1,
                             "rows": 32}, 32)
    assert bad.startswith("FAIL 3 out, 1 sign")


def test_oracle_check_catches_a_planted_error():
    """The cpu_baseline leg's comparison against the oracle, on the host: the
    oracle's own rows pass, a row with one flipped element fails."""
    import numpy as np
    import torch

    import oracle
    w = workloads.WORKLOADS["cube256"]
    a, b = workloads.workload_inputs("cube256")
    rows = bench.parity_rows(w.M, 64)
    good = torch.from_numpy(np.ascontiguousarray(oracle.gemm_relu(a[rows], b)))
    res = {"w": w, "variant": "relu", "check": {"rows": rows, "c_rows": good, "bias": None}}
    s = bench.oracle_check(res)
    assert s["pass"] and s["rows"] == 64 and s["elements"] == 64 * 256
    bad = good.clone()
    i = int(torch.argmax(bad[3].float()))
    bad[3, i] = 0.0  # a positive value zeroed
    res["check"]["c_rows"] = bad
    s = bench.oracle_check(res)
    assert not s["pass"] and s["out_of_tolerance"] >= 1
