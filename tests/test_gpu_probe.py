"""GPU check of the read-bandwidth probe (pa_read_probe): every 32-bit word
of the buffer is read exactly once, so the XOR it leaves in the sink equals
the XOR of the buffer computed on the host, for sizes from one 16-byte unit
to above L2, with ragged remainders after the unrolled rounds."""

import numpy as np
import pytest
import torch

import paged_kv_cache_364_b200 as pk
from gpu_util import needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.mark.parametrize("n_words", [4, 4 * 7, 4 * 512 * 4 * 3 + 4, 4 * 148 * 2048 * 4 + 4 * 37,
                                     (300 << 20) // 4])
def test_probe_reads_every_word_once(n_words):
    g = torch.Generator().manual_seed(n_words)
    host = torch.randint(-2 ** 31, 2 ** 31 - 1, (n_words,), dtype=torch.int32, generator=g)
    buf = host.cuda()
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk.read_probe(buf, sink)
    want = np.bitwise_xor.reduce(host.numpy().view(np.uint32))
    assert int(sink.cpu().numpy().view(np.uint32)[0]) == int(want)
    # a second pass XORs the same value in again: the sink returns to zero
    pk.read_probe(buf, sink)
    assert int(sink.item()) == 0
    assert pk.device_errors() == 0


def test_probe_rejects_a_ragged_size():
    buf = torch.zeros(10, dtype=torch.int32, device="cuda")        # 40 bytes
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(Exception, match="16-byte"):
        pk.read_probe(buf, sink)
