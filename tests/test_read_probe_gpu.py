"""pa_read_probe reads what it says: the 128-bit-load probe folds every 32-bit
word of the buffer into the sink (XOR), the bulk-copy probe the first word of
every 16 KiB chunk, and the scattered-tile probe runs to completion with no
timed-out wait. The numbers it is timed for are the decode path's read
ceilings."""
import numpy as np
import pytest
import torch

from paged_kv_cache_391_b200 import pa

pytestmark = pytest.mark.gpu


def _buf(nbytes, seed):
    rng = np.random.default_rng(seed)
    host = rng.integers(0, 2**32, size=nbytes // 4, dtype=np.uint32)
    return host, torch.from_numpy(host.view(np.int32)).cuda()


@pytest.mark.parametrize("nbytes", [16, 4096, 16384 * 5 + 48, 37 << 20])
def test_vector_probe_folds_every_word(nbytes):
    host, dev = _buf(nbytes, nbytes)
    sink = torch.zeros(1, dtype=torch.int64, device="cuda")
    pa.read_probe(dev, sink, method=0)
    torch.cuda.synchronize()
    assert int(sink.item()) & 0xffffffff == int(np.bitwise_xor.reduce(host))


@pytest.mark.parametrize("nbytes", [16, 16384, 16384 * 5 + 48, 37 << 20])
def test_bulk_probe_reads_every_chunk(nbytes):
    host, dev = _buf(nbytes, nbytes + 1)
    sink = torch.zeros(1, dtype=torch.int64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.read_probe(dev, sink, method=1, dev_error=err)
    torch.cuda.synchronize()
    firsts = host[::4096]                      # the first word of each 16 KiB chunk
    assert int(sink.item()) & 0xffffffff == int(np.bitwise_xor.reduce(firsts))
    assert int(err.item()) == 0


def test_scattered_probe_completes():
    _, dev = _buf(64 << 20, 3)
    sink = torch.zeros(1, dtype=torch.int64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(3):
        pa.read_probe(dev, sink, method=2, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
