"""Benchmark of the fused fp16 GEMM + ReLU (C = ReLU(A @ B)) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload cube8192|mlp_up|decode|...] [--no-secondary]

One step is one call of ``gemm_relu_f16`` (through the C ABI) over one set of
synthetic, seeded inputs already resident in HBM.  The default workload is the
compute-bound 8192^3 cube (A, B ~ N(0,1)/sqrt(K), seed 2); the MLP
up-projection and the decode-shaped skinny product are reported alongside as
``other_workloads``.  Timing: W untimed warm-up steps, then K steps between a
barrier + synchronize on both sides, timed with CUDA events on the launching
stream; the job time is the max over ranks.  With N > 1 (torchrun, one rank
per GPU) every rank runs its own independent replica of the problem (weak
scaling, no collective on the data path).

``e2e`` is the same metric through the host-buffer entry point
``gemm_relu_f16_host``: page-locked host A and B in, C back in host memory,
every step, with the library's copies pipelined against its kernels.

``--impl reference`` times the CPU oracle (the plain fp64 definition of the
operation) on a bounded sample of the same workload on the host cores; under
torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from tiled_tensor_core_05_b200.clocks import ClockSampler, gpu_id_for  # noqa: E402

METRIC = "fused GEMM+ReLU TFLOP/s and % of B200 dense fp16 peak (GB/s % HBM for skinny)"
NOMINAL_FP16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# source files that define each timed kernel (the `traffic` figure of a
# committed ncu capture is reported only while these are unchanged)
KERNEL_SOURCES = {
    "tile_pair_gemm_kernel": ["tiled_tensor_core_05_b200/csrc/gemm_tile.cu",
                              "tiled_tensor_core_05_b200/csrc/sm100.cuh"],
    "tile_gemm_kernel": ["tiled_tensor_core_05_b200/csrc/gemm_tile.cu",
                         "tiled_tensor_core_05_b200/csrc/sm100.cuh"],
    "skinny_gemm_kernel": ["tiled_tensor_core_05_b200/csrc/gemm_skinny.cu",
                           "tiled_tensor_core_05_b200/csrc/skinny_common.cuh",
                           "tiled_tensor_core_05_b200/csrc/sm100.cuh"],
    "skinny_even_kernel": ["tiled_tensor_core_05_b200/csrc/gemm_skinny_even.cu",
                           "tiled_tensor_core_05_b200/csrc/skinny_common.cuh",
                           "tiled_tensor_core_05_b200/csrc/sm100.cuh"],
}


# ------------------------------------------------------------------ utils ---

def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(workload: str, kernel: str, variant: str = "relu"):
    """DRAM bytes (read + write) per launch from a committed ncu capture of
    `kernel` on `workload` (and `variant`, other than the plain ReLU one), if
    it was taken on the current sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            table = json.load(f)
    except (OSError, ValueError):
        return None
    key = f"{kernel}/{workload}" + ("" if variant == "relu" else f"/{variant}")
    e = table.get(key)
    if not e or e.get("kernel_src_sha") != kernel_source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


def max_over_ranks(value: float, dist=None) -> float:
    """The max of `value` over all ranks (the job's time is the slowest
    rank's).  Uses a CUDA tensor under NCCL and a CPU tensor otherwise."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, job_ms: float) -> float:
    """Whole-job throughput: every rank processes `units_per_rank` units (one
    independent replica each), the job takes the slowest rank's `job_ms`."""
    return world * units_per_rank / (job_ms * 1e-3)


# ----------------------------------------------------------- measurements ---

def time_launches(fn, steps: int, warmup: int, stream, dist=None, sampler=None,
                  per_launch=False):
    """Warm up, then time exactly `steps` back-to-back calls between two CUDA
    events on `stream` (barrier + synchronize on both sides).  Returns
    (total_ms of the timed region, max over ranks; ms per launch).  One step
    launches one kernel, so the kernel's average duration over the timed region
    is total / steps (gaps between launches included: a conservative figure).
    With per_launch=True, `steps` more calls are timed afterwards each between
    its own pair of events, and their mean is returned instead."""
    import torch
    if sampler:
        sampler.mark("warm0")
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.mark("t0")
    ev0.record(stream)
    for _ in range(steps):
        fn()
    ev1.record(stream)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark("t1")
    if dist is not None:
        dist.barrier()
    total = max_over_ranks(ev0.elapsed_time(ev1), dist)
    per_ms = total / steps
    if per_launch:
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for i in range(steps):
            starts[i].record(stream)
            fn()
            ends[i].record(stream)
        torch.cuda.synchronize()
        per = [a.elapsed_time(b) for a, b in zip(starts, ends)]
        per_ms = sum(per) / len(per)
    return total, per_ms


def parity_rows(M: int, max_rows: int) -> list:
    """Rows of an M-row result to compare with the oracle: all of them when
    there are at most `max_rows`, else `max_rows` rows spread evenly over M
    (first and last included), so that every tile row of every kernel's
    tiling is sampled."""
    if M <= max_rows:
        return list(range(M))
    step = (M - 1) / (max_rows - 1)
    return sorted({int(round(i * step)) for i in range(max_rows)})


def measure_workload(name, steps, warmup, dist=None, sampler=None, e2e=True,
                     comparator=False, variant="relu", path=0, check_rows=0, min_ms=0.0):
    """Time one workload.  variant: "relu" (gemm_relu_f16, the measured path),
    "bias_gelu" (gemm_bias_act_f16 with a per-column bias and GELU) or "wT"
    (gemm_f16_general with B stored N x K, ReLU).  With `check_rows` > 0 the
    result's rows (all, or that many spread over M) are kept for the oracle
    check.  With `min_ms` > 0 (single-process context runs only) a timed
    region shorter than that is timed again with enough launches to fill it,
    so that short kernels are measured over many launches."""
    import torch

    from tiled_tensor_core_05_b200 import ops, workloads
    w = workloads.WORKLOADS[name]
    a_cpu, b_cpu = workloads.workload_inputs(name)
    a, b = a_cpu.cuda(), b_cpu.cuda()
    c = torch.empty((w.M, w.N), dtype=torch.float16, device="cuda")
    stream = torch.cuda.current_stream()
    lib = ops.lib()
    h = int(stream.cuda_stream)
    bias = None
    if variant == "relu" and path == 0:
        fn, args = lib.gemm_relu_f16, (a.data_ptr(), b.data_ptr(), c.data_ptr(), w.M, w.N, w.K,
                                       w.K, w.N, w.N, h)
    elif variant == "relu":  # an explicitly chosen kernel
        fn, args = lib.gemm_f16_ex, (a.data_ptr(), b.data_ptr(), c.data_ptr(), w.M, w.N, w.K,
                                     w.K, w.N, w.N, 1, path, h)
    elif variant == "bias_gelu":
        g = torch.Generator(device="cpu")
        g.manual_seed(w.seed + 100)
        bias = (torch.randn(w.N, generator=g) * 0.5).half().cuda()
        fn, args = lib.gemm_bias_act_f16, (a.data_ptr(), b.data_ptr(), bias.data_ptr(),
                                           c.data_ptr(), w.M, w.N, w.K, w.K, w.N, w.N,
                                           ops.ACT_GELU, path, h)
    elif variant == "wT":
        b = b.t().contiguous()  # stored N x K
        b_cpu = b_cpu.t().contiguous()
        fn, args = lib.gemm_f16_general, (a.data_ptr(), b.data_ptr(), None, c.data_ptr(), w.M,
                                          w.N, w.K, w.K, w.K, w.N, 0, 1, ops.ACT_RELU,
                                          path, h)
    else:
        raise ValueError(variant)

    def step():
        rc = fn(*args)
        if rc != 0:
            raise RuntimeError(f"{variant} call failed: {ops.status_string(rc)}")

    total_ms, launch_ms = time_launches(step, steps, warmup, stream, dist, sampler)
    if dist is None and min_ms > 0 and total_ms < min_ms:
        n = min(2000, int(min_ms / max(launch_ms, 1e-4)) + 1)
        total_ms, launch_ms = time_launches(step, n, warmup, stream, None, None)
    st = ops.device_status()
    if st != 0:
        raise RuntimeError(f"device reported status {st:#x}")
    # `step` holds raw pointers: keep the tensors alive as long as it is
    res = {"total_ms": total_ms, "launch_ms": launch_ms, "w": w, "step": step,
           "tensors": (a, b, c, bias), "variant": variant, "name": name}
    if check_rows:
        # rows of the measured call's result, kept on the host for the oracle
        # check of the cpu_baseline leg
        rows = parity_rows(w.M, check_rows)
        res["check"] = {"rows": rows, "c_rows": c[torch.as_tensor(rows, device=c.device)].cpu(),
                        "bias": None if bias is None else bias.cpu()}
    if comparator:
        # context only, never on the measured path: cuBLAS through torch on
        # the same inputs, timed the same way right after our kernel
        if variant == "bias_gelu":
            def torch_step():
                torch.nn.functional.gelu(torch.addmm(bias, a, b, out=c))
        elif variant == "wT":
            def torch_step():
                torch.relu_(torch.matmul(a, b.t(), out=c))
        else:
            def torch_step():
                torch.relu_(torch.matmul(a, b, out=c))
        t_total, _ = time_launches(torch_step, steps, warmup, stream, None, None,
                                   per_launch=False)
        t_ms = t_total / steps
        res["torch_launch_ms"] = t_ms
    if e2e and variant in ("relu", "bias_gelu"):
        # end to end through the C ABI's host-buffer entry point: page-locked
        # host A and B in, the kernels, C back in host memory, every step (the
        # library pipelines the copies with the kernels panel by panel)
        a_h = a_cpu.pin_memory()
        b_h = b_cpu.pin_memory()
        c_h = torch.empty((w.M, w.N), dtype=torch.float16).pin_memory()
        bias_h = None if bias is None else bias.cpu().pin_memory()
        if bias_h is None:
            hfn, hargs = lib.gemm_relu_f16_host, (a_h.data_ptr(), b_h.data_ptr(), c_h.data_ptr(),
                                                  w.M, w.N, w.K, w.K, w.N, w.N, h)
        else:
            hfn, hargs = lib.gemm_f16_host, (a_h.data_ptr(), b_h.data_ptr(), bias_h.data_ptr(),
                                             c_h.data_ptr(), w.M, w.N, w.K, w.K, w.N, w.N,
                                             ops.ACT_GELU, h)

        def e2e_step():
            rc = hfn(*hargs)
            if rc != 0:
                raise RuntimeError(f"host-buffer call failed: {ops.status_string(rc)}")

        e_steps = max(3, min(steps, 10))
        e_total, _ = time_launches(e2e_step, e_steps, 1, stream, dist, None, per_launch=False)
        res["e2e_ms"] = e_total / e_steps
        res["h2d"] = (a.numel() + b.numel() + (0 if bias is None else bias.numel())) * 2
        res["d2h"] = c.numel() * 2
        # the host result against the device result of the measured call:
        # the panels may run other kernels, so the same tolerance as parity
        step()
        torch.cuda.synchronize()
        dev = c.cpu()
        res["e2e_bits_equal"] = bool(torch.equal(c_h.view(torch.int16), dev.view(torch.int16)))
        if not res["e2e_bits_equal"]:
            d, r = c_h.float(), dev.float()
            if not bool(((d - r).abs() <= 1e-2 + 1e-2 * r.abs()).all()):
                raise RuntimeError("end-to-end result differs from the device result")
        res["e2e_plan"] = ops.host_plan(w.M, w.N, w.K)
    del a, b, c
    torch.cuda.empty_cache()
    return res


def hbm_bound(w) -> bool:
    """Small-M products stream B once and are measured in GB/s; the rest are
    tensor-pipe bound and measured in TFLOP/s."""
    return w.M <= 64


def kernel_for(w) -> str:
    from tiled_tensor_core_05_b200 import ops
    return {ops.PATH_SKINNY: "skinny_gemm_kernel", ops.PATH_TILE: "tile_gemm_kernel",
            ops.PATH_TILE_PAIR: "tile_pair_gemm_kernel",
            ops.PATH_TILE_PAIR_TALL: "tile_pair_gemm_kernel",
            ops.PATH_SKINNY_EVEN: "skinny_even_kernel"}[ops.select_path(w.M, w.N, w.K)]


def roofline_entry(name, launch_ms, peaks, peak_src, long_run: bool, variant: str = "relu"):
    from tiled_tensor_core_05_b200 import workloads
    w = workloads.WORKLOADS[name]
    kernel = kernel_for(w)
    if hbm_bound(w):
        # HBM bound: algorithmic bytes = A, B read once, C written once
        achieved = w.bytes_min / (launch_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic_for(name, kernel, variant),
                "kernel": kernel, "algorithmic_bytes_per_launch": w.bytes_min,
                "peak_source": f"{peak_src} hbm_gbs (copy bandwidth)"}
    achieved = w.flops / (launch_ms * 1e-3) / 1e12
    key = "bf16_tflops_sustained" if long_run else "bf16_tflops"
    peak = peaks.get(key, peaks["bf16_tflops"])
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": traffic_for(name, kernel, variant),
            "kernel": kernel, "algorithmic_flops_per_launch": w.flops,
            "peak_source": f"{peak_src} {key} (cuBLAS bf16; fp16 has the same nominal rate)"}


def oracle_seconds_per_row(oracle, a, b) -> float:
    """Host time per row of C for the oracle, measured on a block of rows
    large enough to occupy every thread it uses (it parallelises over rows)."""
    oracle.gemm_relu(a[:1], b)  # thread pool and page faults out of the way
    rows = min(int(a.shape[0]), 2 * oracle.max_threads())
    t0 = time.perf_counter()
    oracle.gemm_relu(a[:rows], b)
    return max(time.perf_counter() - t0, 1e-6) / rows


def launch_stats(step, n: int = 50):
    """Median and best of `n` launches, each between its own pair of CUDA
    events on the launching stream (outside the timed region; context)."""
    import torch
    stream = torch.cuda.current_stream()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    torch.cuda.synchronize()
    for i in range(n):
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    per = sorted(a.elapsed_time(b) for a, b in zip(starts, ends))
    return {"launches": n, "median_ms": round(statistics.median(per), 5),
            "best_ms": round(per[0], 5),
            "note": "each launch between its own events, after the timed region; for a "
                    "kernel shorter than the host's time per call the GPU waits for the "
                    "launch inside the events, so the figure is the host's rate"}


def sustained_run(step, launch_ms: float, seconds: float, gpu_uuid: str):
    """Back-to-back launches for about `seconds` (after the timed region), with
    the SM clock and throttle reasons sampled meanwhile: the rate under the
    power cap rather than in a burst."""
    import torch
    n = max(10, int(seconds * 1e3 / max(launch_ms, 1e-3)))
    sampler = ClockSampler(gpu_uuid)
    sampler.wait_first()
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    sampler.mark("t0")
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    sampler.mark("t1")
    sampler.stop()
    total = e0.elapsed_time(e1)
    return {"launches": n, "seconds": round(total / 1e3, 2), "ms_per_launch": round(total / n, 5),
            "clocks": sampler.summary()}


def stream_read_probe(gib: float = 2.0, steps: int = 20):
    """Achievable HBM streaming-read bandwidth on this GPU: the library's
    read probe (every byte of a buffer larger than L2 read once) timed with
    CUDA events.  Context for the small-M kernel, which reads B once."""
    import torch
    from tiled_tensor_core_05_b200 import ops
    n = int(gib * 2 ** 30) // 4
    buf = torch.ones(n, dtype=torch.int32, device="cuda")
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(3):
        ops.read_probe(buf, sink)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        ops.read_probe(buf, sink)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    nbytes = n * 4
    del buf
    return {"what": "gemm_read_probe: every byte of a %.0f GiB buffer read once with 16-byte "
                    "streaming loads (context for the small-M roofline)" % gib,
            "bytes": nbytes, "ms_per_launch": round(ms, 4),
            "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1)}


def parity_summary(got, ref, relu: bool = True) -> dict:
    """Element-by-element comparison of fp16 results with the acceptance rule
    of the tests: |got - ref| <= 1e-2 + 1e-2 |ref|, and wherever |ref| > 1e-2
    the sign of got equals the sign of ref (for ReLU output: got > 0)."""
    import numpy as np
    g = np.asarray(got, dtype=np.float16).astype(np.float64)
    r = np.asarray(ref, dtype=np.float16).astype(np.float64)
    with np.errstate(invalid="ignore"):
        err = np.where(g == r, 0.0, np.abs(g - r))  # equal infinities count as equal
    bad = ~(err <= 1e-2 + 1e-2 * np.abs(r))  # NaN counts as out of tolerance
    big = np.abs(r) > 1e-2
    sign_bad = int(np.count_nonzero(big & (np.sign(g) != np.sign(r))))
    if relu:
        sign_bad += int(np.count_nonzero(g < 0))
    rel = err[big] / np.abs(r[big])
    return {"elements": int(r.size), "max_abs_err": float(np.nanmax(err)) if r.size else 0.0,
            "max_rel_err": float(rel.max()) if rel.size else 0.0,
            "out_of_tolerance": int(np.count_nonzero(bad)), "sign_mismatches": sign_bad,
            "pass": bool(not bad.any() and sign_bad == 0)}


def cpu_baseline(name, budget_s=10.0, gpu_c=None):
    """The oracle timed on a bounded sample (leading rows) of the workload.
    With `gpu_c` (the measured call's result, on the device) the sample's
    rows are also compared with the oracle's (`parity`)."""
    import oracle
    from tiled_tensor_core_05_b200 import workloads
    w = workloads.WORKLOADS[name]
    a, b = workloads.workload_inputs(name)
    rows = int(max(1, min(w.M, budget_s / oracle_seconds_per_row(oracle, a, b))))
    t0 = time.perf_counter()
    ref = oracle.gemm_relu(a[:rows], b)
    dt = time.perf_counter() - t0
    flops = 2.0 * rows * w.N * w.K
    if hbm_bound(w):
        value = (2.0 * (rows * w.K + w.K * w.N + rows * w.N)) / dt / 1e9
        unit = "GB/s"
    else:
        value = flops / dt / 1e12
        unit = "TFLOP/s"
    out = {"value": value, "unit": unit, "cores": oracle.max_threads(), "kind": "oracle",
           "sample": f"first {rows} of {w.M} rows of C ({rows}x{w.N}x{w.K}), {dt:.1f} s",
           "seconds": round(dt, 2)}
    if gpu_c is not None:
        out["parity"] = dict(parity_summary(gpu_c[:rows].cpu().numpy(), ref),
                             rows=f"0-{rows - 1} of {w.M}")
    return out


def oracle_check(res) -> dict:
    """Part of the cpu_baseline leg: the oracle's rows of one measured
    workload (all rows, or a spread sample; see parity_rows) against the rows
    of the measured call's result kept by measure_workload."""
    import numpy as np

    import oracle
    from tiled_tensor_core_05_b200 import workloads
    chk = res["check"]
    w = res["w"]
    a, b = workloads.workload_inputs(w.name)
    a_rows = a[torch_index(chk["rows"])]
    if res["variant"] == "bias_gelu":
        ref = oracle.gemm_bias_act(a_rows, b, chk["bias"], "gelu")
        relu = False
    else:  # "relu" and "wT" (B stored N x K: the same product)
        ref = oracle.gemm_relu(a_rows, b)
        relu = True
    s = parity_summary(np.asarray(chk["c_rows"].numpy()), ref, relu)
    s["rows"] = len(chk["rows"])
    return s


def torch_index(rows):
    import torch
    return torch.as_tensor(rows, dtype=torch.long)


def compact_record(res, peaks, peak_src) -> dict:
    """One short line of the per-workload table that ends the bench line."""
    w = res["w"]
    ms = res["launch_ms"]
    roof = roofline_entry(w.name, ms, peaks, peak_src, False, res["variant"])
    # keys: op = the variant; frac = of the measured peak; pct_nom = % of the
    # nominal 2.25 PFLOP/s or 8 TB/s; traffic = ncu DRAM bytes per launch
    rec = {"workload": w.name, "op": res["variant"], "ms": round(ms, 4),
           "value": roof["achieved"], "unit": roof["unit"], "frac": roof["frac"],
           "pct_nom": round(100 * roof["achieved"] / (
               NOMINAL_HBM_GBS if roof["unit"] == "GB/s" else NOMINAL_FP16_TFLOPS), 1),
           "traffic": roof["traffic"]}
    return rec


def parity_text(s: dict, M: int) -> str:
    """'pass 256/8192 rows' (or 'FAIL ...' with the counts)."""
    head = "pass" if s["pass"] else f"FAIL {s['out_of_tolerance']} out, {s['sign_mismatches']} sign"
    return f"{head} {s['rows']}/{M} rows"


# ------------------------------------------------------------------ arms ---

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from tiled_tensor_core_05_b200 import workloads
    w = workloads.WORKLOADS[args.workload]
    a, b = workloads.workload_inputs(args.workload)
    # size one step to about a second of host work
    rows = int(max(1, min(w.M, 1.0 / oracle_seconds_per_row(oracle, a, b))))
    for _ in range(args.warmup):
        oracle.gemm_relu(a[:rows], b)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.gemm_relu(a[:rows], b)
    dt = (time.perf_counter() - t0) / args.steps
    if hbm_bound(w):
        value, unit = 2.0 * (rows * w.K + w.K * w.N + rows * w.N) / dt / 1e9, "GB/s"
    else:
        value, unit = 2.0 * rows * w.N * w.K / dt / 1e12, "TFLOP/s"
    sample = f"first {rows} of {w.M} rows of C per step ({rows}x{w.N}x{w.K})"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w),
            "cpu_baseline": {"value": value, "unit": unit, "cores": oracle.max_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w):
    mib = (w.M * w.K + w.K * w.N) * 2 / 2 ** 20
    if mib * 2 ** 20 > 126e6:
        l2 = "A+B = %.0f MiB > 126 MB L2: inputs larger than L2, no flush" % mib
    else:
        l2 = "A+B = %.2f MiB fits in L2: L2-warm timing (latency-bound case)" % mib
    return {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "seed": w.seed,
            "a_scale": w.a_scale, "b_scale": w.b_scale, "layout": "row-major, ld = cols",
            "l2": l2, "parallelism": "replicas (one independent problem per GPU)"}


def sharded_decode(dist, world, rank, steps, warmup, gather=True):
    """The column-sharded small-M product across the ranks (one process per
    GPU): every rank holds A and its own block of whole 256-column tiles of
    B, computes its block of C = ReLU(A @ B) and, with `gather`, all-gathers
    the blocks so that every rank holds the whole C.  Total work is fixed
    (strong scaling): the job rate is the whole problem's algorithmic bytes
    over the max-over-ranks time per step.  Returns (record, C on the device,
    or None without `gather`)."""
    import torch

    from tiled_tensor_core_05_b200 import shard, workloads
    w = workloads.WORKLOADS["decode"]
    a_cpu, b_cpu = workloads.workload_inputs("decode")
    n0, n1 = shard.column_range(w.N, world, rank)
    a = a_cpu.cuda()
    b_blk = b_cpu[:, n0:n1].contiguous().cuda()
    del b_cpu
    out = torch.empty((w.M, w.N), dtype=torch.float16, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        shard.gemm_sharded(a, b_blk, n_total=w.N, out=out, rank=rank, world=world,
                           gather=gather)

    total_ms, _ = time_launches(step, steps, warmup, stream, dist)
    return shard_record(w, world, rank, total_ms / steps, gather), (out if gather else None)


def shard_record(w, world: int, rank: int, ms: float, gather: bool) -> dict:
    """The sharded leg's record: the whole problem's algorithmic bytes (A, B
    and C once) over the max-over-ranks time per step `ms` (strong scaling:
    the problem does not grow with the rank count)."""
    from tiled_tensor_core_05_b200 import shard
    n0, n1 = shard.column_range(w.N, world, rank)
    return {"workload": w.name, "n_gpus": world, "scaling": "strong", "gather": gather,
            "ms": round(ms, 5), "value": round(w.bytes_min / (ms * 1e-3) / 1e9, 1),
            "unit": "GB/s", "columns_per_rank": n1 - n0}


def run_ours(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    from tiled_tensor_core_05_b200 import ops
    ops.lib()
    peaks, peak_src = load_peaks()
    single = rank == 0 and world == 1
    check = single and not args.no_cpu_baseline
    sampler = ClockSampler(gpu_id_for(local))
    sampler.wait_first()
    main = measure_workload(args.workload, args.steps, args.warmup, dist, sampler,
                            e2e=not args.no_e2e, comparator=not args.no_comparator,
                            path=args.path, variant=args.variant,
                            check_rows=256 if check else 0)
    sampler.stop()
    clocks = sampler.summary()
    w = main["w"]
    long_run = main["total_ms"] > 2000.0
    ms = main["total_ms"] / args.steps
    if hbm_bound(w):
        value, unit = job_rate(w.bytes_min, world, ms) / 1e9, "GB/s"
    else:
        value, unit = job_rate(w.flops, world, ms) / 1e12, "TFLOP/s"
    line = {"metric": METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic (seeded torch.randn on the CPU, cast to fp16)",
            "config": workload_config(w), "gpu_launches": args.steps}
    if hbm_bound(w):
        line["pct_of_nominal_hbm"] = round(100 * value / world / NOMINAL_HBM_GBS, 2)
    else:
        line["pct_of_dense_fp16_peak"] = round(100 * value / world / NOMINAL_FP16_TFLOPS, 2)
    line["roofline"] = roofline_entry(args.workload, main["launch_ms"], peaks, peak_src,
                                      long_run, args.variant)
    if "e2e_ms" in main:
        e_ms = main["e2e_ms"]
        ev = (w.flops / (e_ms * 1e-3) / 1e12) if unit == "TFLOP/s" else \
            (w.bytes_min / (e_ms * 1e-3) / 1e9)
        line["e2e"] = {"value": round(world * ev, 2), "unit": unit,
                       "h2d_bytes_per_step": main["h2d"], "d2h_bytes_per_step": main["d2h"],
                       "ms_per_step": round(e_ms, 4),
                       "call": "gemm_relu_f16_host" if args.variant == "relu" else "gemm_f16_host",
                       "plan": main["e2e_plan"], "bits_equal_device": main["e2e_bits_equal"]}
    line["clocks"] = clocks
    context = {}
    if "torch_launch_ms" in main:
        context["torch_matmul_act_ms"] = round(main["torch_launch_ms"], 5)
    # the sharded small-M product (row f4) at every rank count: each rank
    # streams its 1/N of B; every rank takes the same steps and collectives
    if not args.no_shard:
        srec, s_out = sharded_decode(dist, world, rank, max(args.steps, 20),
                                     max(args.warmup, 3), gather=world > 1)
        if s_out is not None and check:
            srec["check"] = {"rows": list(range(s_out.shape[0])), "c_rows": s_out.cpu(),
                             "bias": None}
        del s_out
        torch.cuda.empty_cache()
    else:
        srec = None
    # context passes (other workloads, probe, per-launch and sustained runs)
    # only in single-GPU runs: under torchrun the other ranks would wait for
    # rank 0 at the closing barrier meanwhile
    others = []
    if single and not args.no_secondary:
        for name, variant in (("mlp_up", "relu"), ("decode", "relu"), ("cube1024", "relu"),
                              ("ragged1000", "relu"), ("cube256", "relu"),
                              ("mlp_up", "bias_gelu"), ("decode", "wT")):
            if name == args.workload and variant == args.variant:
                continue
            r = measure_workload(name, max(args.steps, 20), max(args.warmup, 3), None, None,
                                 e2e=False, comparator=not args.no_comparator, variant=variant,
                                 check_rows=512 if check else 0, min_ms=20.0)
            r.pop("step")
            r.pop("tensors")
            others.append(r)
            torch.cuda.empty_cache()
        probe = stream_read_probe()
        context["read_probe_gbs"] = probe["gbs"]
    if single and args.sustained_seconds > 0:
        ls = launch_stats(main["step"])
        context["launch_median_ms"] = ls["median_ms"]
        context["launch_best_ms"] = ls["best_ms"]
        sus = sustained_run(main["step"], main["launch_ms"], args.sustained_seconds,
                            gpu_id_for(local))
        rate = (w.bytes_min / (sus["ms_per_launch"] * 1e-3) / 1e9 if unit == "GB/s"
                else w.flops / (sus["ms_per_launch"] * 1e-3) / 1e12)
        sc = sus["clocks"]
        context["sustained"] = {"seconds": sus["seconds"], "ms": sus["ms_per_launch"],
                                "value": round(rate, 2), "unit": unit,
                                "sm_mhz": sc.get("sm_mhz"), "reasons": sc.get("reasons")}
    # the first record is the main workload's
    records = [compact_record(r, peaks, peak_src) for r in [main] + others]
    if "read_probe_gbs" in context:
        for rec in records:
            if rec["unit"] == "GB/s":
                rec["frac_probe"] = round(rec["value"] / context["read_probe_gbs"], 4)
    if check:
        # the cpu_baseline leg: the oracle timed on a sample of the main
        # workload, and every measured result compared with the oracle
        line["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_budget,
                                            main["tensors"][2]
                                            if args.variant in ("relu", "wT") else None)
        for rec, r in zip(records, [main] + others):
            rec["parity"] = parity_text(oracle_check(r), r["w"].M)
        if srec is not None and "check" in srec:
            from tiled_tensor_core_05_b200 import workloads
            srec["parity"] = parity_text(oracle_check(dict(srec, variant="relu",
                                                           w=workloads.WORKLOADS["decode"])),
                                         32)
    if srec is not None:
        srec.pop("check", None)
        context["sharded_decode"] = srec
    line["context"] = context
    line["configs"] = records  # last: the short per-workload table
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line, separators=(",", ":")), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="cube8192")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-shard", action="store_true",
                    help="skip the column-sharded decode leg (each rank 1/N of B)")
    ap.add_argument("--sustained-seconds", type=float, default=2.0,
                    help="length of the back-to-back context run after the timed region "
                         "(0: skip it and the per-launch statistics)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--path", type=int, default=0,
                    help="kernel for the main workload: 0 = chosen by shape (gemm_relu_f16), "
                         "1 tile, 2 small-M, 3 CTA pair, 4 CTA pair with 512-row tiles")
    ap.add_argument("--variant", default="relu", choices=["relu", "bias_gelu", "wT"],
                    help="operation of the main workload (default: the fused ReLU GEMM)")
    ap.add_argument("--no-comparator", action="store_true",
                    help="skip timing torch.matmul + relu as a context comparator")
    ap.add_argument("--cpu-budget", type=float, default=10.0,
                    help="seconds of oracle work for the cpu_baseline sample")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.steps < 1:
        ap.error("--steps must be >= 1")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
