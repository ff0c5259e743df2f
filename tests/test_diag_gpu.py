"""The read-floor diagnostic (sa_diag_read_floor): both modes read every byte of the buffer
once -- the XOR of all its 32-bit words comes back -- on sizes that do and do not divide
evenly among the blocks, so the floor the bench times really reads what the decode reads."""
import numpy as np
import pytest
import torch

from online_softmax_attention_sm_b200 import SAError, sa_check_status, sa_diag_read_floor

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("n_words", [4, 4 * 1237, 1 << 20, 16 * 1000003])
def test_read_floor_reads_every_word(mode, n_words):
    g = torch.Generator().manual_seed(n_words + mode)
    buf = torch.randint(-2 ** 31, 2 ** 31 - 1, (n_words,), generator=g, dtype=torch.int32)
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa_diag_read_floor(buf.cuda(), sink, mode)
    sa_check_status()
    want = np.bitwise_xor.reduce(buf.numpy().view(np.uint32))
    assert int(sink.cpu().numpy().view(np.uint32)[0]) == int(want)


def test_read_floor_rejects_ragged_sizes():
    buf = torch.zeros(3, dtype=torch.int32, device="cuda")       # 12 bytes: not a multiple of 16
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(SAError):
        sa_diag_read_floor(buf, sink, 0)
