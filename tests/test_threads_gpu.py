"""Concurrent use from several host threads, each on its own CUDA stream: the
library's host-side state (device table, per-stream small-M workspaces,
kernel attribute and occupancy caches) is shared, and every result must equal
the one a single thread gets (all kernels are deterministic)."""
import threading

import pytest
import torch

from tiled_tensor_core_05_b200 import ops, workloads

pytestmark = pytest.mark.gpu

SHAPES = [  # (M, N, K, path): tile, pair, 512-row pair and split-K small-M kernels
    (300, 520, 264, ops.PATH_TILE),
    (1024, 2048, 512, ops.PATH_TILE_PAIR),
    (1536, 1024, 4096, ops.PATH_TILE_PAIR_TALL),
    (32, 1024, 8192, ops.PATH_SKINNY),
    (48, 4096, 2048, ops.PATH_AUTO),
]


def test_concurrent_threads_on_own_streams():
    torch.cuda.set_device(0)
    inputs = []
    for i, (m, n, k, path) in enumerate(SHAPES):
        a, b = workloads.make_inputs(m, n, k, seed=60 + i, a_scale=1.0 / k ** 0.5)
        inputs.append((a.cuda(), b.cuda(), path))
    # reference results, one thread, default stream
    want = []
    for a, b, path in inputs:
        want.append(ops.gemm_f16_ex(a, b, relu=True, path=path))
    torch.cuda.synchronize()

    errors = []

    def worker(tid):
        try:
            stream = torch.cuda.Stream()
            with torch.cuda.stream(stream):
                outs = []
                for rep in range(6):
                    for j in range(len(inputs)):
                        a, b, path = inputs[(j + tid) % len(inputs)]
                        outs.append(((j + tid) % len(inputs),
                                     ops.gemm_f16_ex(a, b, relu=True, path=path)))
                stream.synchronize()
            for idx, c in outs:
                if not torch.equal(c.view(torch.int16), want[idx].view(torch.int16)):
                    errors.append(f"thread {tid}: shape {SHAPES[idx]} differs")
                    return
        except Exception as e:  # reported below, the test thread asserts
            errors.append(f"thread {tid}: {e!r}")

    threads = [threading.Thread(target=worker, args=(t,)) for t in range(4)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not any(t.is_alive() for t in threads), "a worker did not finish"
    assert not errors, errors
    assert ops.device_status() == 0
