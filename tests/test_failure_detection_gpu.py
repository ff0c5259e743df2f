"""Failure detection without a GPU fault: every device wait in the library is bounded; a
wait that runs out records a timeout in a device status word and the kernel returns, so
the host sees SA_ERR_TIMEOUT from sa_check_status and the context stays usable."""
import ctypes
import time

import pytest
import torch

from online_softmax_attention_sm_b200 import lib, sa_attn_fwd, sa_check_status
from online_softmax_attention_sm_b200.sa_attn import SA_ERR_TIMEOUT, SA_OK, SAError
from online_softmax_attention_sm_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_the_context_survives():
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib().sa_check_status(stream) == SA_OK           # clean start
    t0 = time.time()
    assert lib().sa_selftest_bounded_wait(stream) == SA_OK
    rc = lib().sa_check_status(stream)                       # synchronises
    waited = time.time() - t0
    assert rc == SA_ERR_TIMEOUT, lib().sa_last_error().decode()
    assert "expired" in lib().sa_last_error().decode()
    assert 1.0 < waited < 30.0
    assert lib().sa_check_status(stream) == SA_OK           # the word was cleared
    # the context is still usable: a normal call runs and checks out
    q, k, v = (t.cuda() for t in make_qkv(1, 256, 256, 2, 2, 64, "fp16", seed=3))
    o, lse = sa_attn_fwd(q, k, v, causal=True)
    sa_check_status()
    assert torch.isfinite(o.float()).all()


def test_binding_raises_on_timeout():
    lib().sa_selftest_bounded_wait(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    with pytest.raises(SAError) as e:
        sa_check_status()
    assert e.value.code == SA_ERR_TIMEOUT
    sa_check_status()
