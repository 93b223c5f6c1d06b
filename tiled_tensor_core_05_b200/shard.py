"""Column-sharded GEMM across ranks (one process per GPU): each rank owns a
contiguous block of whole 256-column tiles of B and C and computes
C[:, n0:n1] = act(A @ B[:, n0:n1] + bias[n0:n1]) with the library's kernels,
reading only its block of B (a small-M product on G GPUs streams 1/G of the
weights each).  No exchange is needed to compute the blocks: the activation
applies column by column, so nothing is reduced across ranks.  With
``gather=True`` the blocks are all-gathered so that every rank holds the whole
C (a torch.distributed collective: NCCL between GPUs).

The split of the columns is the tensor-parallel reading of the small-batch
split idea of "Writing high-performance kernels in TileLang" (atlascloud.ai
blog), section "La parte buena: las optimizaciones son de una sola línea cada
una", applied to N instead of K so that no partial sums cross GPUs.
"""
from __future__ import annotations

from typing import Callable

import torch

from . import ops

TILE = 256  # columns per shard unit: whole tiles of the kernels' widest column tiling


def column_range(N: int, world: int, rank: int, align: int = TILE) -> tuple[int, int]:
    """[n0, n1): the columns of an N-column output that `rank` of `world` owns:
    contiguous runs of whole `align`-column tiles, as even as the tile count
    allows (ranks past the last tile get an empty range)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    tiles = -(-N // align)
    base, extra = divmod(tiles, world)
    t0 = rank * base + min(rank, extra)
    t1 = t0 + base + (1 if rank < extra else 0)
    return min(N, t0 * align), min(N, t1 * align)


def _default_local(a, b_block, bias_block, act, out_block):
    return ops.gemm_general(a, b_block, bias_block, act, out_block)


def gemm_sharded(a: torch.Tensor, b: torch.Tensor, *, n_total: int | None = None,
                 bias: torch.Tensor | None = None, act: str = "relu",
                 out: torch.Tensor | None = None, rank: int = 0, world: int = 1,
                 gather: bool = False, group=None,
                 local_gemm: Callable | None = None) -> torch.Tensor:
    """This rank's column block of act(a @ b + bias).

    ``b`` is either the whole (K, N) matrix (the rank reads only its columns,
    through a strided view) or this rank's own (K, n1 - n0) block, in which
    case ``n_total`` = N must be given; ``bias`` is the whole length-N bias or
    None.  Returns the (M, n1 - n0) block, written into ``out`` (the whole
    (M, N) output, of which this rank writes its columns) when given.  With
    ``gather=True`` every rank gets the whole (M, N) result (``group``: the
    torch.distributed group, default the world).
    ``local_gemm(a, b_block, bias_block, act, out_block)`` computes one block
    (default: the library's fused kernel)."""
    local = local_gemm or _default_local
    N = int(n_total) if n_total is not None else b.shape[1]
    M = a.shape[0]
    n0, n1 = column_range(N, world, rank)
    b_block = b[:, n0:n1] if b.shape[1] == N else b
    if b_block.shape[1] != n1 - n0:
        raise ValueError(f"rank {rank} owns {n1 - n0} columns; b has {b.shape[1]}")
    if out is not None and tuple(out.shape) != (M, N):
        raise ValueError("out must be the whole (M, N) output")
    bias_block = None if bias is None else bias[n0:n1]
    if out is not None:
        out_block = out[:, n0:n1]
    else:
        out_block = torch.empty((M, n1 - n0), dtype=a.dtype, device=a.device)
    if n1 > n0:
        local(a, b_block, bias_block, act, out_block)
    if not gather:
        return out_block
    if world == 1:  # the block is the whole result
        return out if out is not None else out_block
    import torch.distributed as dist
    # One collective into one contiguous buffer of `world` equal-size blocks:
    # rank 0's block is the widest, narrower ones are padded to it.  The
    # blocks cannot land in C directly: a column block of row-major C is a
    # strided region, and the collective moves contiguous buffers; the copy
    # out of the buffer is M x N x 2 bytes on the device (1.8 MB for a 32-row
    # decode product).
    r00, r01 = column_range(N, world, 0)
    width = r01 - r00
    if n1 - n0 == width:
        send = out_block.contiguous()
    else:
        send = torch.zeros((M, width), dtype=out_block.dtype, device=out_block.device)
        send[:, :n1 - n0] = out_block
    gathered = torch.empty((world, M, width), dtype=send.dtype, device=send.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(gathered, send, group=group)
    else:  # gloo has no single-buffer form: the same buffer as a list of views
        dist.all_gather(list(gathered.unbind(0)), send, group=group)
    full = out if out is not None else torch.empty((M, N), dtype=a.dtype, device=a.device)
    for r in range(world):
        r0, r1 = column_range(N, world, r)
        if r1 <= r0 or (out is not None and r == rank):  # empty, or written in place
            continue
        full[:, r0:r1] = gathered[r, :, :r1 - r0]
    return full
