"""The allocation-free entry point, gemm_relu_f16_noalloc.

Some callers must not allocate device memory while they run: plugins whose
enqueue step may not allocate, processes whose GPU memory belongs to a pool
allocator, and latency-critical loops where cudaMalloc's implicit device
synchronisation would stall other work.  For them gemm_relu_f16_noalloc runs
the small-M kernel with its scratch (fp32 partial tiles and arrival
counters) in a fixed array inside the library, limited to M <= 32.

These tests call it through the C ABI, twice in a row on the same inputs
(the second call finds the first call's leftovers in the shared array), and
compare each result with the allocating entry point gemm_relu_f16 and with
the CPU oracle (the plain fp64 definition, which shares no code with either
entry point), within the tolerance the other GPU tests use and with the same
sign and zero pattern.  They set up everything they need, so they pass on
their own in a fresh process as well as after the rest of the suite; the file
name makes pytest collect them last.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ATOL = RTOL = 1e-2
SCRATCH_LIMIT = -7  # GEMM_ERR_SCRATCH_LIMIT


def _dev(x: torch.Tensor) -> torch.Tensor:
    """fp16 CPU matrix -> device, row stride rounded up to a multiple of 8."""
    r, c = x.shape
    ld = (c + 7) // 8 * 8
    buf = torch.zeros((r, ld), dtype=torch.float16, device="cuda")
    buf[:, :c] = x.cuda()
    return buf[:, :c]


def _ld(t: torch.Tensor) -> int:
    return int(t.stride(0)) if t.size(0) > 1 else (int(t.size(1)) + 7) // 8 * 8


def _call(fn, a, b, c):
    M, K = a.shape
    N = b.shape[1]
    return fn(a.data_ptr(), b.data_ptr(), c.data_ptr(), M, N, K, _ld(a), _ld(b), _ld(c),
              torch.cuda.current_stream().cuda_stream)


def _close(c: torch.Tensor, ref) -> bool:
    """Within the tolerance of a device result (tensor) or an oracle result."""
    c64 = c.double().cpu().numpy()
    r64 = ref.double().cpu().numpy() if isinstance(ref, torch.Tensor) else np.float64(ref)
    return bool(np.all(np.abs(c64 - r64) <= ATOL + RTOL * np.abs(r64)))


def _same_relu_pattern(c: torch.Tensor, ref: np.ndarray) -> bool:
    """c > 0 wherever ref > 1e-2, no negative value, no -0, no NaN."""
    bits = c.cpu().contiguous().view(torch.int16).numpy()
    c64 = c.double().cpu().numpy()
    r64 = np.asarray(ref, dtype=np.float64)
    return bool((c64[r64 > ATOL] > 0).all() and (c64 >= 0).all() and not (bits == -32768).any()
                and not np.isnan(c64).any())


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "needs a CUDA device"
    torch.cuda.set_device(0)
    from tiled_tensor_core_05_b200 import ops
    return ops.lib()


@pytest.mark.parametrize("m,n,k,seed", [(32, 8192, 4096, 41), (5, 1000, 1000, 42),
                                        (32, 129, 257, 43), (1, 3000, 8200, 44)])
def test_noalloc_matches_allocating_entry_point_on_two_calls(lib, m, n, k, seed):
    from tiled_tensor_core_05_b200 import workloads
    a_cpu, b_cpu = workloads.make_inputs(m, n, k, seed=seed)
    a, b = _dev(a_cpu), _dev(b_cpu)
    ref = _dev(torch.zeros((m, n), dtype=torch.float16))
    outs = [_dev(torch.full((m, n), 7.0, dtype=torch.float16)) for _ in range(2)]
    assert _call(lib.gemm_relu_f16, a, b, ref) == 0
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for c in outs:  # two calls in a row share (and reuse) the fixed scratch
        assert _call(lib.gemm_relu_f16_noalloc, a, b, c) == 0
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    import oracle
    want = oracle.gemm_relu(a_cpu, b_cpu).astype(np.float64)
    for i, c in enumerate(outs):
        assert _close(c, ref), f"call {i + 1} differs from gemm_relu_f16"
        assert _close(c, want), f"call {i + 1} differs from the oracle"
        assert _same_relu_pattern(c, want), f"call {i + 1}: sign or zero pattern differs"
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    # nothing was allocated on the device by the two calls
    assert free_before - free_after < (1 << 20), (free_before, free_after)


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    from tiled_tensor_core_05_b200 import ops
    a = torch.zeros((33, 64), dtype=torch.float16, device="cuda")
    b = torch.zeros((64, 64), dtype=torch.float16, device="cuda")
    c = torch.full((33, 64), 3.0, dtype=torch.float16, device="cuda")
    assert _call(lib.gemm_relu_f16_noalloc, a, b, c) == SCRATCH_LIMIT
    assert "M <= 32" in ops.status_string(SCRATCH_LIMIT)
    torch.cuda.synchronize()
    assert (c == 3.0).all()  # nothing was launched
