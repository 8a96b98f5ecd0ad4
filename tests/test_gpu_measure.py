"""hyb_stream_read (the plain-read floor bench.py reports beside each decode
workload): the XOR it folds into the sink equals the XOR of the buffer's
32-bit words computed on the host."""
import numpy as np
import pytest
import torch

import int8_paged_kv_hybrid_b200 as hk

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nbytes", [16, 4096 + 16, 1 << 20, 34227200, (256 << 20) + 48])
def test_stream_read_xor(nbytes):
    g = torch.Generator().manual_seed(nbytes)
    host = torch.randint(-2**31, 2**31 - 1, (nbytes // 4,), dtype=torch.int32, generator=g)
    dev = host.cuda()
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    hk.hyb_stream_read(dev, sink)
    torch.cuda.synchronize()
    want = np.bitwise_xor.reduce(host.numpy().view(np.uint32))
    assert int(sink.cpu().numpy().view(np.uint32)[0]) == int(want)
    # a second read XORs the same word in again: back to zero
    hk.hyb_stream_read(dev, sink)
    torch.cuda.synchronize()
    assert int(sink.item()) == 0


def test_stream_read_rejections():
    buf = torch.zeros(64, dtype=torch.int32, device="cuda")
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(hk.HybError):
        hk.hyb_stream_read(buf[1:5], sink)  # 4-byte offset: not 16-byte aligned
    with pytest.raises(hk.HybError):
        hk.hyb_stream_read(buf[:6], sink)  # 24 bytes
    hk.hyb_stream_read(buf[:0], sink)  # nothing to read
    torch.cuda.synchronize()
    assert int(sink.item()) == 0
