"""kvd_read_stream (the read-only bandwidth probe of the roofline) reads every
byte it is given: its XOR checksum must equal the host's over the same words,
in both forms, on a buffer whose size is not a multiple of the bulk chunk."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_decode_scatters_b200 as m
    m.kvd_read_device_error(clear=True)
    return m


@pytest.mark.parametrize("words", [4, 1000, (64 << 20) // 4 + 12, (300 << 20) // 4 + 4])
def test_read_stream_checksum(kvd, words):
    g = torch.Generator().manual_seed(words)
    host = torch.randint(-2 ** 31, 2 ** 31 - 1, (words,), dtype=torch.int64, generator=g).to(torch.int32)
    want = int(np.bitwise_xor.reduce(host.numpy().view(np.uint32)))
    buf = host.cuda()
    for mode in (kvd.KVD_READ_VECTOR, kvd.KVD_READ_BULK):
        sink = kvd.kvd_read_stream(buf, mode)
        torch.cuda.synchronize()
        got = int(sink.cpu().numpy().view(np.uint32)[0])
        assert got == want, f"mode {mode}: {got:#x} != {want:#x}"
    assert kvd.kvd_read_device_error() == 0
