"""The read-bandwidth stream (pa_stream_read) on the GPU: every 32-bit word of
the buffer is read exactly once, which the XOR of the CTAs' sinks shows (it
equals the XOR of the buffer, computed here with numpy), for sizes that fill
the unrolled loop, leave a ragged tail, or are smaller than one wave."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_343_b200 as pa
    return pa


@pytest.mark.parametrize("words,ctas", [
    (1 << 24, 148 * 4),          # 64 MiB: many full rounds of four loads
    ((1 << 22) + 4 * 37, 148),   # a ragged tail after the unrolled rounds
    (4 * 5, 3),                  # fewer 16-byte words than threads
    (0, 7),                      # nothing to read: every sink entry is 0
])
def test_stream_read_reads_every_word_once(pa, words, ctas):
    g = torch.Generator().manual_seed(words + ctas)
    host = torch.randint(-(1 << 31), (1 << 31) - 1, (words,), dtype=torch.int64, generator=g)
    host = host.to(torch.int32)
    buf = host.cuda()
    sink = torch.full((ctas,), -1, dtype=torch.int32, device="cuda")
    pa.stream_read(buf, sink)
    torch.cuda.synchronize()
    want = np.bitwise_xor.reduce(host.numpy().view(np.uint32)) if words else np.uint32(0)
    got = np.bitwise_xor.reduce(sink.cpu().numpy().view(np.uint32))
    assert int(got) == int(want)
    if words == 0:
        assert torch.count_nonzero(sink).item() == 0
