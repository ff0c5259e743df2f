"""The decode entry point that allocates nothing (sa_attn_decode_noalloc).

It serves callers that cannot give the library device memory for scratch (runtimes that
reserve all GPU memory up front, hosts whose allocator is out of reach of the calling
code); its scratch is a fixed area inside the library.  Checked here through the C ABI
against the workspace-taking sa_attn_decode, on calls in a row that reuse the area with
different shapes: the two run the same kernels with the same split plan, so the results
must be bit-identical (a stale or aliased byte in the shared area would show), plus the
size limit.  The library's device code (the area included) is loaded by the first call
into it -- here the reference decode, before any measured call.  This file is collected
last on purpose: a run that stops at the first failure has already run every other test.
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
        assert torch.equal(o, ref_o) and torch.equal(lse, ref_lse), f"call {i}: not bit-identical"


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 2 splits of 64 keys for 64 x 128 rows of D = 128: 8.65 MB of split states, over the 8 MiB
    # area.  K/V really hold Sk rows, so even if the size check failed to stop the call it
    # could only compute, never read outside the buffers.
    B, Sk, Hq, Hkv, D, ns = 64, 128, 128, 8, 128, 2
    assert B * Hq * ns * (D + 4) * 4 > 8 << 20
    q = torch.zeros((B, Hq, D), dtype=torch.bfloat16, device=DEV)
    k = torch.zeros((B, Sk, Hkv, D), dtype=torch.bfloat16, device=DEV)
    v = torch.zeros_like(k)
    o = torch.full_like(q, 3.0)
    lse = torch.full((B, Hq), 3.0, dtype=torch.float32, device=DEV)
    rc = noalloc(q, k, v, o, lse, 0.1, "bf16", num_splits=ns)
    assert rc == SA_ERR_UNSUPPORTED
    assert "scratch" in lib().sa_last_error().decode()
    sa_check_status()
    assert torch.all(o == 3.0) and torch.all(lse == 3.0)
