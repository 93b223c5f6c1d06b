"""The multi-rank logic of bench.py on CPU with a 2-rank gloo process group:
the job time is the max over ranks, the job rate counts every rank's replica,
and the reference arm runs on rank 0 only."""
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [3.0, 7.5][rank]
        got = bench.max_over_ranks(local, dist)
        rate = bench.job_rate(100.0, world, got)
        q.put((rank, got, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, rate in results:
        assert got == 7.5                       # slowest rank
        assert rate == pytest.approx(2 * 100.0 / 7.5e-3)


def test_single_process_helpers():
    assert bench.max_over_ranks(4.0, None) == 4.0
    assert bench.job_rate(10.0, 1, 1.0) == pytest.approx(10_000.0)


def test_reference_arm_other_ranks_do_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "cube256"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--workload", "cube256"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_shard_record_is_strong_scaling():
    from tiled_tensor_core_05_b200 import workloads
    w = workloads.WORKLOADS["decode"]
    one = bench.shard_record(w, 1, 0, 0.0716, False)
    two = bench.shard_record(w, 2, 1, 0.0358, True)
    assert one["columns_per_rank"] == 28672 and two["columns_per_rank"] == 14336
    assert one["scaling"] == two["scaling"] == "strong"
    # the same whole problem in half the time: twice the job rate
    assert two["value"] == pytest.approx(2 * one["value"], rel=1e-3)
    assert one["value"] == pytest.approx(w.bytes_min / 0.0716e-3 / 1e9, rel=1e-3)
