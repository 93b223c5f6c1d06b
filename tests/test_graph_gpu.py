"""The device-pointer entry points inside CUDA graphs: calls on every kernel
family (single-SM tile, 256- and 512-row CTA pairs, the small-M kernel with
k-slices) captured once on a stream, replayed, and compared element by
element with the oracle of the fused GEMM + ReLU ("Writing high-performance
kernels in TileLang", atlascloud.ai blog, section "Escribamos un GEMM").
Replays read the live input buffers (new values copied in between replays
give the new products) and repeated replays give the same bits (the small-M
kernel's arrival counters return to zero after every call).
"""
import pytest
import torch

from gpu_util import check_parity
from tiled_tensor_core_05_b200 import ops, workloads

pytestmark = pytest.mark.gpu

CASES = [((256, 256, 256), ops.PATH_TILE), ((600, 1096, 704), ops.PATH_TILE_PAIR),
         ((1100, 600, 520), ops.PATH_TILE_PAIR_TALL), ((32, 1000, 4096), ops.PATH_SKINNY),
         ((7, 304, 200), ops.PATH_AUTO)]


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    ops.lib()
    yield
    torch.cuda.synchronize()
    assert ops.device_status() == 0, "a kernel reported a device-side timeout"


def test_capture_and_replay(oracle_mod):
    s = torch.cuda.Stream()
    bufs = []
    for i, ((m, n, k), path) in enumerate(CASES):
        a, b = workloads.make_inputs(m, n, k, seed=7000 + i, b_scale=1.0 / k ** 0.5)
        da, db = a.cuda(), b.cuda()
        dc = torch.empty((m, n), dtype=torch.float16, device="cuda")
        bufs.append((da, db, dc, path))
    torch.cuda.synchronize()
    # first calls outside the capture: per-stream workspace, kernel attributes
    with torch.cuda.stream(s):
        for da, db, dc, path in bufs:
            ops.gemm_f16_ex(da, db, dc, relu=True, path=path, stream=s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for da, db, dc, path in bufs:
            ops.gemm_f16_ex(da, db, dc, relu=True, path=path, stream=s)
    for rnd in range(2):
        # new inputs in the captured buffers, outputs poisoned, then replay
        refs = []
        for i, (da, db, dc, path) in enumerate(bufs):
            m, k = da.shape
            n = db.shape[1]
            a, b = workloads.make_inputs(m, n, k, seed=7100 + 10 * rnd + i,
                                         b_scale=1.0 / k ** 0.5)
            da.copy_(a)
            db.copy_(b)
            dc.fill_(float("nan"))
            refs.append(oracle_mod.gemm_relu(a, b))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        first = [dc.clone() for _, _, dc, _ in bufs]
        for (da, db, dc, path), ref in zip(bufs, refs):
            check_parity(dc.cpu().numpy(), ref, True, f"graph replay {tuple(dc.shape)} path {path}")
        g.replay()
        torch.cuda.synchronize()
        for (_, _, dc, path), f in zip(bufs, first):
            assert torch.equal(dc.view(torch.int16), f.view(torch.int16)), f"replay bits, {path}"
    del g
