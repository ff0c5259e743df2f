"""The decode entry point that allocates nothing (sa_attn_decode_noalloc).

It serves callers that cannot give the library device memory for scratch (runtimes that
reserve all GPU memory up front, hosts whose allocator is out of reach of the calling
code); its scratch is a fixed area inside the library.  Checked here through the C ABI
against the workspace-taking sa_attn_decode, on calls in a row that reuse the area with
different shapes, plus the size limit.  This file is collected last on purpose: a run
that stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from online_softmax_attention_sm_b200 import lib, sa_attn_decode, sa_check_status
from online_softmax_attention_sm_b200.sa_attn import SA_BF16, SA_ERR_UNSUPPORTED, SA_FP16, SA_OK
from online_softmax_attention_sm_b200.inputs import make_qkv
from gpu_helpers import LSE_TOL, O_TOL

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
DT = {"fp16": SA_FP16, "bf16": SA_BF16}


def noalloc(q, k, v, o, lse, scale, dtype, num_splits=0):
    B, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    return lib().sa_attn_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()), B, Sk, Hq, Hkv, D,
        ctypes.c_float(scale), DT[dtype], num_splits,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


# two different shapes back to back, then the first again: each call finds the previous
# call's leftovers in the shared scratch area
CALLS = [(4, 32768, 14, 2, 64, "fp16"), (2, 5000, 16, 2, 128, "bf16"), (4, 32768, 14, 2, 64, "fp16")]


def test_noalloc_decode_matches_workspace_decode():
    for i, (B, Sk, Hq, Hkv, D, dt) in enumerate(CALLS):
        q, k, v = (t.to(DEV) for t in make_qkv(B, 1, Sk, Hq, Hkv, D, dt, seed=100 + i, decode=True))
        scale = 1.0 / np.sqrt(D)
        ref_o, ref_lse = sa_attn_decode(q, k, v, scale=scale)
        o = torch.full_like(q, 7.0)
        lse = torch.full((B, Hq), 7.0, dtype=torch.float32, device=DEV)
        assert noalloc(q, k, v, o, lse, scale, dt) == SA_OK, lib().sa_last_error().decode()
        sa_check_status()
        err = (o.float() - ref_o.float()).abs().max().item()
        lerr = (lse - ref_lse).abs().max().item()
        assert err <= O_TOL[dt], f"call {i}: max |O - O_ref| = {err:.3e}"
        assert lerr <= LSE_TOL, f"call {i}: max |LSE - LSE_ref| = {lerr:.3e}"


def test_noalloc_rejects_problems_beyond_its_scratch():
    B, Sk, Hq, Hkv, D = 64, 32768, 64, 8, 128      # with 96 splits: ~186 MB of split states
    q = torch.zeros((B, Hq, D), dtype=torch.bfloat16, device=DEV)
    k = torch.zeros((B, 128, Hkv, D), dtype=torch.bfloat16, device=DEV)   # never read
    o = torch.full_like(q, 3.0)
    lse = torch.full((B, Hq), 3.0, dtype=torch.float32, device=DEV)
    fake_k = ctypes.c_void_p(k.data_ptr())
    rc = lib().sa_attn_decode_noalloc(ctypes.c_void_p(q.data_ptr()), fake_k, fake_k,
                                      ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
                                      B, Sk, Hq, Hkv, D, ctypes.c_float(0.1), SA_BF16, 96,
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == SA_ERR_UNSUPPORTED
    assert "scratch" in lib().sa_last_error().decode()
    sa_check_status()
    assert torch.all(o == 3.0) and torch.all(lse == 3.0)
