"""The streaming-read probe (a measurement tool beside the GEMM): it reads
every byte once, which the XOR of all 32-bit words shows, for sizes that are
and are not multiples of the grid's step, and rejects bad arguments."""
import numpy as np
import pytest
import torch

from tiled_tensor_core_05_b200 import ops

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_words", [0, 4, 12, 4 * 592 * 512 * 4, 4 * 592 * 512 * 4 + 36,
                                     3_000_004])
def test_probe_reads_every_word(n_words):
    g = torch.Generator().manual_seed(n_words)
    host = torch.randint(-2**31, 2**31 - 1, (max(n_words, 1),), generator=g,
                         dtype=torch.int64).to(torch.int32)[:n_words]
    buf = host.cuda()
    sink = ops.read_probe(buf)
    torch.cuda.synchronize()
    want = np.bitwise_xor.reduce(host.numpy().view(np.uint32)) if n_words else 0
    assert int(sink.cpu().numpy().view(np.uint32)[0]) == int(want)


def test_probe_argument_errors():
    buf = torch.zeros(64, dtype=torch.int32, device="cuda")
    sink = torch.zeros(4, dtype=torch.int32, device="cuda")
    lib = ops.lib()
    s = torch.cuda.current_stream().cuda_stream
    assert lib.gemm_read_probe(buf.data_ptr(), 100, sink.data_ptr(), s) == -1   # not % 16
    assert lib.gemm_read_probe(buf.data_ptr() + 4, 64, sink.data_ptr(), s) == -2
    assert lib.gemm_read_probe(buf.data_ptr(), 64, None, s) == -1
    # far past the end of the allocation that holds `buf` (torch carves small
    # tensors out of 2 MiB segments, so only a span beyond the segment is
    # detectable)
    assert lib.gemm_read_probe(buf.data_ptr(), 1 << 26, sink.data_ptr(), s) == -1
    host = torch.zeros(64, dtype=torch.int32)
    assert lib.gemm_read_probe(host.data_ptr(), 64, sink.data_ptr(), s) == -1
