"""Offline sweep of kernel configurations (tile shape, ring depth, CTA pairing,
raster panel, split-K) for the fused fp16 GEMM + activation.

    python -m tiled_tensor_core_05_b200.tune [--workloads cube8192,mlp_up,...]
                                             [--steps 30] [--out table.md] [--json out.json]
    python -m tiled_tensor_core_05_b200.tune --host [--workloads cube8192,mlp_up,decode]

With --host the sweep is over the host-buffer entry point's panel plans
(gemm_f16_host_planned: row or column panels of several widths, and the plan
gemm_host_plan_for picks), with the host link's copy rates measured beside
them (host-to-device alone, device-to-host alone, both at once).

The tuning workflow of "TileLang simplifica la creación de kernels GPU de alto
rendimiento" (posicionamiento-web.ar) and "TileLang explicado: kernels de IA
escritos por mosaicos" (easyairoute.com), in their sections on tuning tile
sizes, pipeline stages and L2 ordering for each GPU and validating every
candidate before trusting its time, done once, offline: the library never
times or picks among configurations at run time.  Its GEMM_PATH_AUTO rules and
defaults are set from the table this script writes.

For each workload:
  1. the candidate space: every tile shape (128 x 64, 128 x 128 and 128 x 256 on one SM,
     256 x 256 and 512 x 256 on a CTA pair, the 128- and 256-column small-M
     kernel when M <= 64) x ring depths 3..8 x raster panels (1, 2, 4, ...
     tile-rows, up to all of them) or k-slices;
  2. pruning: depths whose shared memory (gemm_config_smem_bytes) exceeds the
     227 KiB a CTA can opt into, small-M ring depths beyond the compiled cap of
     6, duplicate panels (a panel of more tile-rows than the problem has is
     the whole column), k-slice counts the split-K workspace or K cannot hold;
  3. validation of each survivor against torch's fp32 product, activated, with
     the pages' check |c - ref| <= 1e-2 + 1e-2 |ref| plus c > 0 wherever
     ref > 1e-2 (ReLU); a candidate that fails is reported and never ranked;
  4. timing: `steps` back-to-back launches between two CUDA events after 3
     warm-up launches (operands larger than L2 for the large workloads; the
     small ones run L2-warm);
  5. the leaders (and the AUTO configuration) re-timed in interleaved rounds
     (a fresh random order each round), because the power-capped SM clock
     drifts by more than the differences between neighbouring candidates; the
     median of the rounds is ranked, the spread of the rounds and the median
     SM clock (NVML, sampled during each block) are reported beside it, and
     ms x MHz (thousands of SM cycles) separates a faster kernel from a
     higher clock.
"""
from __future__ import annotations

import argparse
import json
import math
import random
import statistics
import sys
import time

from . import ops
from .workloads import WORKLOADS, Workload, make_inputs

SMEM_BUDGET = 232448  # bytes of dynamic shared memory a CTA may opt into (sm_100)
STAGE_RANGE = range(3, 9)
TILE_KINDS = [(ops.PATH_TILE, 64), (ops.PATH_TILE, 128), (ops.PATH_TILE, 256),
              (ops.PATH_TILE_PAIR, 256), (ops.PATH_TILE_PAIR_TALL, 256)]
TILE_ROWS = {ops.PATH_TILE: 128, ops.PATH_TILE_PAIR: 256, ops.PATH_TILE_PAIR_TALL: 512}
KERNEL_NAMES = {ops.PATH_TILE: "tile", ops.PATH_SKINNY: "skinny",
                ops.PATH_TILE_PAIR: "pair", ops.PATH_TILE_PAIR_TALL: "pair-tall",
                ops.PATH_SKINNY_EVEN: "skinny-even"}
SKINNY_WIDTHS = (128, 256)
EVEN_WIDTHS = (64, 128, 192, 256)  # 64 q columns per CTA, q whole 64-column units
EVEN_STAGES = range(4, 7)          # the compiled depths of the even small-M schedule

def describe(cfg: dict) -> str:
    k = cfg["kernel"]
    if k == ops.PATH_SKINNY:
        s = cfg["splits"]
        return f"skinny {cfg['block_n']} st{cfg['stages']} splits={'auto' if s == 0 else s}"
    if k == ops.PATH_SKINNY_EVEN:
        return f"skinny-even {cfg['block_n']} st{cfg['stages']}"
    rows = TILE_ROWS[k]
    return (f"{KERNEL_NAMES[k]} {rows}x{cfg['block_n']} st{cfg['stages']} "
            f"panel={cfg['group_rows']}")


def candidates(M: int, N: int, K: int, sm_count: int, smem_fn, budget: int = SMEM_BUDGET,
               built=None):
    """(kept, pruned): kept is a list of config dicts; pruned a list of
    (config dict, reason).  `smem_fn(cfg) -> bytes` is the library's formula;
    `built` (a set of (kernel, block_n, stages)) prunes what is not compiled."""
    kept, pruned = [], []
    kinds = list(TILE_KINDS)
    if M <= 64:
        kinds += [(ops.PATH_SKINNY, w) for w in SKINNY_WIDTHS]
        # the even schedule's width is fixed by the shape: 64 q, q whole
        # 64-column units per SM (none when there are fewer units than SMs)
        q = -(-N // 64) // sm_count
        if 1 <= q <= 4:
            kinds.append((ops.PATH_SKINNY_EVEN, 64 * q))
    for kernel, bn in kinds:
        for st in STAGE_RANGE:
            base = {"kernel": kernel, "block_n": bn, "stages": st, "group_rows": 0,
                    "splits": 0}
            smem = smem_fn(base)
            if smem > budget:
                pruned.append((base, f"shared memory {smem} > {budget}"))
                continue
            if built is not None and (kernel, bn, st) not in built:
                pruned.append((base, "not compiled (depth cap)"))
                continue
            if kernel == ops.PATH_SKINNY:
                tiles = -(-N // bn)
                kb = -(-K // 64)
                seen = set()
                for s in (0, 1, 2, 3, 4, 6, 8, 12, 16, 24, 32):
                    if s > kb or (s > 1 and s * tiles > sm_count):
                        pruned.append(({**base, "splits": s}, "k-slices do not fit"))
                        continue
                    if s in seen:
                        continue
                    seen.add(s)
                    kept.append({**base, "splits": s})
            elif kernel == ops.PATH_SKINNY_EVEN:
                kept.append(base)
            else:
                rows = TILE_ROWS[kernel]
                tile_rows = -(-M // rows)
                seen = set()
                g = 1
                while True:
                    eff = min(g, tile_rows)
                    if eff not in seen:
                        seen.add(eff)
                        kept.append({**base, "group_rows": eff * rows})
                    if g >= tile_rows:
                        break
                    g *= 2
    return kept, pruned


# ------------------------------------------------------------ measurement ---

def _reference(a, b, bias, act):
    import torch
    ref = torch.matmul(a.float(), b.float())
    if bias is not None:
        ref += bias.float()[None, :]
    if act == "relu":
        ref.clamp_(min=0.0)
    elif act == "gelu":
        ref = torch.nn.functional.gelu(ref)
    return ref


def check(c, ref, act) -> tuple[bool, float]:
    """The pages' tolerance (and, after ReLU, the sign/zero pattern)."""
    import torch
    cf = c.float()
    err = (cf - ref).abs()
    ok = bool(torch.all(err <= 1e-2 + 1e-2 * ref.abs()).item())
    ok = ok and bool(torch.isfinite(cf).all().item())
    if act == "relu":
        ok = ok and bool(torch.all(cf[ref > 1e-2] > 0).item())
    return ok, float(err.max().item())


_BLOCK = [0]


def time_config(run, steps: int, stream, sampler=None):
    """(ms per launch, median SM MHz during the block or None)."""
    import torch
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    _BLOCK[0] += 1
    tag = str(_BLOCK[0])
    if sampler is not None:
        sampler.mark("s" + tag)
    e0.record(stream)
    for _ in range(steps):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    mhz = None
    if sampler is not None and sampler.ok:
        sampler.mark("e" + tag)
        mhz = sampler.summary("s" + tag, "e" + tag).get("sm_mhz")
    return e0.elapsed_time(e1) / steps, mhz


def sweep_workload(w: Workload, act: str, use_bias: bool, steps: int, rounds: int,
                   leaders: int, log=print, sampler=None, seed: int = 0,
                   round_steps: int | None = None, cool_s: float = 0.0,
                   only: list[dict] | None = None) -> dict:
    """Validate and time the candidates of `w` (or only the configurations in
    `only`, with the AUTO one added), then re-time the leaders in `rounds`
    shuffled rounds of `round_steps` launches (default `steps`), idling
    `cool_s` seconds before each block."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device())
    sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
    a_h, b_h = make_inputs(w.M, w.N, w.K, w.seed, w.a_scale, w.b_scale)
    a, b = a_h.to(dev), b_h.to(dev)
    bias = None
    if use_bias:
        g = torch.Generator(device="cpu")
        g.manual_seed(w.seed + 1000)
        bias = (torch.randn(w.N, generator=g) * 0.5).to(torch.float16).to(dev)
    c = torch.empty((w.M, w.N), dtype=torch.float16, device=dev)
    ref = _reference(a, b, bias, act)
    stream = torch.cuda.current_stream(dev)
    auto = ops.auto_config(w.M, w.N, w.K, act).as_dict()
    built = {(c.kernel, c.block_n, c.stages) for c in ops.config_list()}
    kept, pruned = candidates(w.M, w.N, w.K, sm_count, ops.config_smem_bytes, built=built)
    if only is not None:
        full = {"kernel": 0, "block_n": 0, "stages": 0, "group_rows": 0, "splits": 0}
        kept, pruned = [{**full, **c} for c in only], []
    if not any(cfg == auto for cfg in kept):
        kept.append(auto)
    results = []
    t_start = time.time()
    for cfg in kept:
        def run(cfg=cfg):
            ops.gemm_config_run(a, b, cfg, bias, act, c)
        c.fill_(float("nan"))
        run()
        torch.cuda.synchronize()
        ok, err = check(c, ref, act)
        status = ops.device_status()
        entry = {"config": cfg, "desc": describe(cfg), "smem": ops.config_smem_bytes(cfg),
                 "parity": ok and status == 0, "max_abs_err": err}
        if entry["parity"]:
            entry["first_ms"], entry["first_mhz"] = time_config(run, steps, stream, sampler)
        results.append(entry)
    ranked = sorted((r for r in results if r["parity"]), key=lambda r: r["first_ms"])
    top = ranked[:leaders]
    auto_entry = next(r for r in results if r["config"] == auto)
    if auto_entry not in top and auto_entry["parity"]:
        top.append(auto_entry)
    for r in top:
        r["round_ms"], r["round_mhz"] = [], []
    rng = random.Random(seed)
    for _ in range(rounds):
        order = list(top)
        rng.shuffle(order)
        for r in order:
            def run(cfg=r["config"]):
                ops.gemm_config_run(a, b, cfg, bias, act, c)
            if cool_s > 0:
                time.sleep(cool_s)
            ms, mhz = time_config(run, round_steps or steps, stream, sampler)
            r["round_ms"].append(ms)
            r["round_mhz"].append(mhz)
    for r in top:
        r["ms"] = statistics.median(r["round_ms"])
        r["spread_ms"] = [min(r["round_ms"]), max(r["round_ms"])]
        mhz = [x for x in r["round_mhz"] if x]
        r["mhz"] = statistics.median(mhz) if mhz else None
        kc = [m * f for m, f in zip(r["round_ms"], r["round_mhz"]) if f]
        r["kcycles"] = statistics.median(kc) if kc else None
    top.sort(key=lambda r: r["ms"])
    log(f"{w.name} act={act} bias={use_bias}: {len(kept)} candidates, {len(pruned)} pruned, "
        f"{sum(not r['parity'] for r in results)} failed parity, {time.time() - t_start:.1f} s")
    return {"workload": w.name, "shape": [w.M, w.N, w.K], "act": act, "bias": use_bias,
            "sm_count": sm_count, "auto": auto, "results": results, "leaders": top,
            "pruned": [(cfg, why) for cfg, why in pruned]}


# ----------------------------------------------------------------- report ---

# ------------------------------------------------------- host-buffer plans ---

HOST_ROW_EXTENTS = (512, 1024, 2048, 4096)
HOST_COL_EXTENTS = (1024, 2048, 4096, 8192)


def host_plan_candidates(M: int, N: int, max_panels: int = 16) -> list[dict]:
    """Row and column panel plans gemm_f16_host_planned accepts for an M x N
    output: at most `max_panels` panels, column panels whole multiples of 8
    columns; the single-panel plan of each split included."""
    out, seen = [], set()
    for split, dim, extents in ((ops.HOST_SPLIT_ROWS, M, HOST_ROW_EXTENTS + (M,)),
                                (ops.HOST_SPLIT_COLS, N, HOST_COL_EXTENTS + (N,))):
        for ext in extents:
            ext = min(ext, dim)
            if ext < 1 or -(-dim // ext) > max_panels or (split, ext) in seen:
                continue
            if split == ops.HOST_SPLIT_COLS and ext < dim and ext % 8:
                continue
            seen.add((split, ext))
            out.append({"split": split, "panel_extent": ext})
    return out


def _events_ms(fn, reps: int, streams=()) -> float:
    """Median over `reps` of one call of `fn` between CUDA events on the
    current stream (side `streams` joined back in before the end event)."""
    import torch
    cur = torch.cuda.current_stream()
    times = []
    for _ in range(reps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(cur)
        for st in streams:
            st.wait_event(e0)
        fn()
        for st in streams:
            ev = torch.cuda.Event()
            ev.record(st)
            cur.wait_event(ev)
        e1.record(cur)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def sweep_host(w: Workload, steps: int, rounds: int, seed: int = 0, log=print) -> dict:
    """Time every host-buffer plan for workload `w` (ReLU), after checking its
    result against the device path's, and the host link's copy rates."""
    import torch
    a, b = make_inputs(w.M, w.N, w.K, w.seed, w.a_scale, w.b_scale)
    a_h, b_h = a.pin_memory(), b.pin_memory()
    c_h = torch.empty((w.M, w.N), dtype=torch.float16).pin_memory()
    dev = ops.gemm_relu_f16(a.cuda(), b.cuda())
    in_bytes = (a.numel() + b.numel()) * 2
    out_bytes = c_h.numel() * 2
    # the link: the same bytes as one call, in one direction or both at once
    h_in = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
    d_in = torch.empty(in_bytes, dtype=torch.uint8, device="cuda")
    d_out = torch.empty(out_bytes, dtype=torch.uint8, device="cuda")
    h_out = torch.empty(out_bytes, dtype=torch.uint8).pin_memory()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()

    def h2d():
        with torch.cuda.stream(s1):
            d_in.copy_(h_in, non_blocking=True)

    def d2h():
        with torch.cuda.stream(s2):
            h_out.copy_(d_out, non_blocking=True)

    def both():
        h2d()
        d2h()
    link = {"h2d_ms": _events_ms(h2d, 5, (s1,)), "d2h_ms": _events_ms(d2h, 5, (s2,)),
            "both_ms": _events_ms(both, 5, (s1, s2))}
    link["h2d_gbs"] = in_bytes / link["h2d_ms"] / 1e6
    link["d2h_gbs"] = out_bytes / link["d2h_ms"] / 1e6
    del h_in, d_in, d_out, h_out
    plans = [None] + host_plan_candidates(w.M, w.N)
    auto = ops.host_plan(w.M, w.N, w.K)
    results = []
    for plan in plans:
        c_h.fill_(float("nan"))
        ops.gemm_host(a_h, b_h, None, "relu", c_h, plan=plan)
        ok, err = check(c_h.cuda(), dev.float(), "relu")
        results.append({"plan": plan or {"split": auto["split"],
                                         "panel_extent": auto["panel_extent"]},
                        "auto": plan is None, "valid": ok, "max_abs_err": err, "ms": []})
    rng = random.Random(seed)
    order = [i for i, r in enumerate(results) if r["valid"]]
    for _ in range(rounds):
        rng.shuffle(order)
        for i in order:
            plan = plans[i]
            results[i]["ms"].append(_events_ms(
                lambda: ops.gemm_host(a_h, b_h, None, "relu", c_h, sync=False, plan=plan),
                steps))
    for r in results:
        r["median_ms"] = statistics.median(r["ms"]) if r["ms"] else None
    serial = {}
    da, db = a.cuda(), b.cuda()
    dc = torch.empty_like(dev)

    def serial_call():
        da.copy_(a_h, non_blocking=True)
        db.copy_(b_h, non_blocking=True)
        ops.gemm_relu_f16(da, db, dc)
        c_h.copy_(dc, non_blocking=True)
    serial["ms"] = _events_ms(serial_call, steps)
    log(f"{w.name}: link {link}, serial {serial['ms']:.3f} ms")
    return {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "in_bytes": in_bytes,
            "out_bytes": out_bytes, "link": link, "serial_ms": serial["ms"], "auto": auto,
            "plans": results}


def host_markdown(reports: list[dict], command: str, device: str) -> str:
    lines = [f"# Host-buffer plan sweep ({device})", "", f"Command: `{command}`", ""]
    for r in reports:
        k = r["link"]
        lines += [f"## {r['workload']} ({r['M']} x {r['N']} x {r['K']}, ReLU)", "",
                  f"Link: {r['in_bytes'] / 2**20:.0f} MiB host-to-device alone "
                  f"{k['h2d_ms']:.3f} ms ({k['h2d_gbs']:.1f} GB/s); "
                  f"{r['out_bytes'] / 2**20:.0f} MiB device-to-host alone {k['d2h_ms']:.3f} ms "
                  f"({k['d2h_gbs']:.1f} GB/s); both at once {k['both_ms']:.3f} ms.  "
                  f"Serial copies and kernel on one stream: {r['serial_ms']:.3f} ms.", "",
                  "| plan | panels | valid | median ms | rounds min-max | TFLOP/s |",
                  "|---|---|---|---|---|---|"]
        flops = 2.0 * r["M"] * r["N"] * r["K"]
        rows = sorted(r["plans"], key=lambda p: p["median_ms"] or float("inf"))
        for p in rows:
            pl = p["plan"]
            dim = r["M"] if pl["split"] == ops.HOST_SPLIT_ROWS else r["N"]
            name = ("rows" if pl["split"] == ops.HOST_SPLIT_ROWS else "cols") + \
                f" {pl['panel_extent']}" + (" (AUTO)" if p["auto"] else "")
            if p["median_ms"] is None:
                lines.append(f"| {name} | {-(-dim // pl['panel_extent'])} | no | - | - | - |")
                continue
            lines.append(f"| {name} | {-(-dim // pl['panel_extent'])} | yes | "
                         f"{p['median_ms']:.3f} | {min(p['ms']):.3f}-{max(p['ms']):.3f} | "
                         f"{flops / (p['median_ms'] * 1e-3) / 1e12:.1f} |")
        lines.append("")
    return "\n".join(lines)


def _rate(w_shape, ms, skinny_like: bool):
    M, N, K = w_shape
    if skinny_like:
        return f"{2 * (M * K + K * N + M * N) / (ms * 1e-3) / 1e9:.0f} GB/s"
    return f"{2 * M * N * K / (ms * 1e-3) / 1e12:.0f} TFLOP/s"


def to_markdown(reports: list[dict], command: str, device: str) -> str:
    out = [f"# Kernel configuration sweep ({device})", "",
           f"Command: `{command}`", "",
           "Every candidate was validated against torch's fp32 product with the pages' "
           "tolerance before it was timed; `first` is one block of back-to-back launches, "
           "`median` the median of interleaved re-timing rounds of the leaders (and of the "
           "AUTO configuration).", ""]
    for rep in reports:
        M, N, K = rep["shape"]
        skinny_like = M <= 64
        fails = [r for r in rep["results"] if not r["parity"]]
        out += [f"## {rep['workload']} ({M} x {N} x {K}, act={rep['act']}"
                f"{', bias' if rep['bias'] else ''})", "",
                f"{len(rep['results'])} candidates timed, {len(rep['pruned'])} pruned "
                f"(shared memory / k-slices), {len(fails)} failed validation.  "
                f"AUTO: `{describe(rep['auto'])}`.", "",
                "| rank | configuration | smem KiB | median ms | rounds min-max | rate | "
                "SM MHz | ms x MHz | vs AUTO |",
                "|---|---|---|---|---|---|---|---|---|"]
        auto_ms = next((r["ms"] for r in rep["leaders"] if r["config"] == rep["auto"]), None)
        for i, r in enumerate(rep["leaders"]):
            rel = f"{(auto_ms / r['ms'] - 1) * 100:+.1f} %" if auto_ms else "-"
            tag = " (AUTO)" if r["config"] == rep["auto"] else ""
            mhz = f"{r['mhz']:.0f}" if r.get("mhz") else "-"
            kc = f"{r['kcycles']:.0f}" if r.get("kcycles") else "-"
            lo, hi = r["spread_ms"]
            out.append(f"| {i + 1} | `{r['desc']}`{tag} | {r['smem'] / 1024:.0f} | "
                       f"{r['ms']:.4f} | {lo:.4f}-{hi:.4f} | "
                       f"{_rate(rep['shape'], r['ms'], skinny_like)} | {mhz} | {kc} | {rel} |")
        out += ["", "<details><summary>all candidates (first timing)</summary>", "",
                "| configuration | ms | parity | max abs err |", "|---|---|---|---|"]
        for r in sorted(rep["results"], key=lambda r: r.get("first_ms", math.inf)):
            ms = f"{r['first_ms']:.4f}" if "first_ms" in r else "-"
            out.append(f"| `{r['desc']}` | {ms} | {'ok' if r['parity'] else 'FAIL'} | "
                       f"{r['max_abs_err']:.3g} |")
        out += ["", "</details>", ""]
    return "\n".join(out) + "\n"


DEFAULT_SWEEP = [("cube8192", "relu", False), ("mlp_up", "relu", False),
                 ("mlp_up", "gelu", True), ("decode", "relu", False),
                 ("decode_n4096", "relu", False), ("decode_m16_n8192_k4096", "relu", False),
                 ("decode_m64_n2048_k8192", "relu", False),
                 ("decode_n1024_k16384", "relu", False),
                 ("decode_n14336_k4096", "relu", False), ("cube1024", "relu", False)]


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--workloads", default=None,
                    help="comma list of name[:act[:bias]] (default: the standard sweep)")
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--rounds", type=int, default=7)
    ap.add_argument("--round-steps", type=int, default=None,
                    help="launches per block in the re-timing rounds (default: --steps)")
    ap.add_argument("--cool", type=float, default=0.0,
                    help="seconds of idle before each re-timing block")
    ap.add_argument("--only", default=None,
                    help="';'-separated configurations kernel,block_n,stages,group_rows,splits "
                         "to time instead of the candidate space (with AUTO added)")
    ap.add_argument("--leaders", type=int, default=6)
    ap.add_argument("--out", default=None, help="write the markdown table here")
    ap.add_argument("--json", default=None, help="write all results as JSON here")
    ap.add_argument("--host", action="store_true",
                    help="sweep the host-buffer entry point's panel plans instead")
    args = ap.parse_args(argv)
    import torch
    if not torch.cuda.is_available():
        raise SystemExit("the sweep needs a CUDA device")
    if args.host:
        names = (args.workloads or "cube8192,mlp_up,decode").split(",")
        reports = [sweep_host(WORKLOADS[n], args.steps, args.rounds, seed=i,
                              log=lambda *x: print(*x, file=sys.stderr, flush=True))
                   for i, n in enumerate(names)]
        command = "python -m tiled_tensor_core_05_b200.tune " + " ".join(argv or sys.argv[1:])
        md = host_markdown(reports, command.strip(), torch.cuda.get_device_name())
        if args.out:
            with open(args.out, "w") as f:
                f.write(md)
        else:
            print(md)
        if args.json:
            with open(args.json, "w") as f:
                json.dump(reports, f, indent=1)
        return
    plan = DEFAULT_SWEEP
    if args.workloads:
        plan = []
        for item in args.workloads.split(","):
            parts = item.split(":")
            plan.append((parts[0], parts[1] if len(parts) > 1 else "relu",
                         len(parts) > 2 and parts[2] == "bias"))
    only = None
    if args.only:
        keys = ("kernel", "block_n", "stages", "group_rows", "splits")
        only = [dict(zip(keys, (int(v) for v in item.split(","))))
                for item in args.only.split(";") if item.strip()]
    from .clocks import ClockSampler, gpu_id_for
    sampler = ClockSampler(gpu_id_for(torch.cuda.current_device()))
    sampler.wait_first()
    reports = []
    try:
        for i, (name, act, use_bias) in enumerate(plan):
            w = WORKLOADS[name]
            reports.append(sweep_workload(w, act, use_bias, args.steps, args.rounds,
                                          args.leaders, sampler=sampler, seed=i,
                                          round_steps=args.round_steps, cool_s=args.cool,
                                          only=only,
                                          log=lambda *x: print(*x, file=sys.stderr, flush=True)))
    finally:
        sampler.stop()
    device = torch.cuda.get_device_name()
    command = "python -m tiled_tensor_core_05_b200.tune " + " ".join(argv or sys.argv[1:])
    md = to_markdown(reports, command.strip(), device)
    if args.out:
        with open(args.out, "w") as f:
            f.write(md)
    else:
        print(md)
    if args.json:
        with open(args.json, "w") as f:
            json.dump(reports, f, indent=1)


if __name__ == "__main__":
    main()
