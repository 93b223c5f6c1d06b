"""Column sharding across ranks (no GPU): the partition of the columns, and
the all-gather of the blocks with 2- and 3-rank gloo process groups (the local
product is a plain CPU stand-in here; the GPU test runs the library's
kernel)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from tiled_tensor_core_05_b200 import shard


@pytest.mark.parametrize("N", [1, 255, 256, 1000, 4096, 28672, 28672 + 8])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_column_ranges_cover_disjoint_aligned_balanced(N, world):
    ranges = [shard.column_range(N, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == N
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0  # contiguous, disjoint, in rank order
    for n0, n1 in ranges:
        assert n0 <= n1
        if n1 > n0:  # empty ranges past the last tile sit at N
            assert n0 % shard.TILE == 0
    tiles = [-(-(n1 - n0) // shard.TILE) for n0, n1 in ranges]
    assert max(tiles) - min(tiles) <= 1
    with pytest.raises(ValueError):
        shard.column_range(N, world, world)


def _cpu_gemm(a, b_block, bias_block, act, out_block):
    x = a.float() @ b_block.float()
    if bias_block is not None:
        x += bias_block.float()
    if act == "relu":
        x = torch.relu(x)
    out_block.copy_(x.half())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    try:
        _work(rank, world, port, q)
    except Exception as e:  # report instead of leaving the parent to time out
        q.put((rank, f"error: {e!r}", False, False))
        raise


def _work(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(5)
        M, K, N = 8, 32, 700
        a = torch.randn(M, K, generator=g).half()
        b = torch.randn(K, N, generator=g).half()
        bias = torch.randn(N, generator=g).half()
        want = torch.empty(M, N, dtype=torch.float16)
        _cpu_gemm(a, b, bias, "relu", want)
        # whole B, gather into a fresh tensor
        full = shard.gemm_sharded(a, b, bias=bias, rank=rank, world=world, gather=True,
                                  local_gemm=_cpu_gemm)
        ok_full = torch.equal(full, want)
        # this rank's own block of B, no gather
        n0, n1 = shard.column_range(N, world, rank)
        blk = shard.gemm_sharded(a, b[:, n0:n1].contiguous(), n_total=N, bias=bias,
                                 rank=rank, world=world, local_gemm=_cpu_gemm)
        ok_blk = torch.equal(blk, want[:, n0:n1])
        # gather into a caller's output
        out = torch.full((M, N), 7.0, dtype=torch.float16)
        shard.gemm_sharded(a, b, bias=bias, out=out, rank=rank, world=world, gather=True,
                           local_gemm=_cpu_gemm)
        ok_out = torch.equal(out, want)
        q.put((rank, ok_full, ok_blk, ok_out))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gather_across_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    errors = [r for r in results if isinstance(r[1], str)]
    assert not errors, errors
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(r[0] for r in results) == list(range(world))
    assert all(r[1] and r[2] and r[3] for r in results), results
