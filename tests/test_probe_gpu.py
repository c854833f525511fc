"""The streaming-read probe that the benchmark reports beside the roofline:
it reads every byte it is given (a buffer folded to the sentinel constant
sets the sink, any other leaves it alone) and measures a plausible HBM read
bandwidth on a buffer far above the L2."""
import numpy as np
import pytest
import torch

from sparse_long_context_ffd_b200 import ffd

pytestmark = pytest.mark.gpu

SENTINEL = 0x9E3779B9


def _buffer_folding_to(value, n16, where):
    """n16 16-byte words, all zero except word `where`, whose four lanes XOR to value."""
    words = np.zeros((n16, 4), dtype=np.uint32)
    words[where] = [value ^ 0x01020304, 0x01020304, 0, 0]
    return torch.from_numpy(words.view(np.uint8).reshape(-1)).cuda()


@pytest.mark.parametrize("n16,where", [(1, 0), (4096, 4095), (1 << 22, 12345)])
def test_probe_reads_every_word(n16, where):
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    ffd.read_probe(_buffer_folding_to(SENTINEL, n16, where), sink)
    torch.cuda.synchronize()
    # exactly one thread folds the sentinel word; any other fold leaves the sink
    assert int(sink.item()) & 0xFFFFFFFF == SENTINEL
    sink.zero_()
    ffd.read_probe(_buffer_folding_to(SENTINEL ^ 1, n16, where), sink)
    torch.cuda.synchronize()
    assert int(sink.item()) == 0


def test_probe_bandwidth_is_plausible():
    import bench
    gbs = bench.read_probe_gbs(torch.device("cuda"), gib=2, iters=5)
    assert 1000.0 < gbs < 9000.0  # HBM3e: a few TB/s, below the 8 TB/s nominal
