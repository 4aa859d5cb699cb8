"""pkv_stream_read, the read-only pass the benchmark uses as a second HBM denominator: it reads a
device buffer without changing it, its sink word stays untouched for ordinary data, and its rate on
a buffer far larger than L2 is a plausible HBM figure (between 1 and 12 TB/s on a B200)."""
import pytest
import torch

from paged_kv_cache_324_b200 import binding as B

pytestmark = pytest.mark.gpu


def test_stream_read_leaves_the_buffer_and_sink_alone():
    dev = torch.device("cuda:0")
    buf = torch.arange(1 << 20, dtype=torch.int32, device=dev)
    before = buf.clone()
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    B.stream_read(buf, sink)
    torch.cuda.synchronize()
    assert torch.equal(buf, before)
    assert int(sink.item()) == 0


def test_stream_read_rate_is_an_hbm_rate():
    dev = torch.device("cuda:0")
    buf = torch.ones(1 << 30, dtype=torch.uint8, device=dev)        # 1 GiB, eight times L2
    B.stream_read(buf)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(5):
        B.stream_read(buf)
    e.record()
    torch.cuda.synchronize()
    gbs = 5 * buf.numel() / (s.elapsed_time(e) * 1e-3) / 1e9
    assert 1000.0 < gbs < 12000.0, gbs
