"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and the
fp64 oracle on the same seeded inputs, and compare element by element."""
import math

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import (sa_attn_fwd, sa_attn_fwd_simple, sa_attn_decode,
                                               sa_check_status)
from online_softmax_attention_sm_b200.inputs import make_qkv

# tolerances of the spec: max-abs on O (fp16 2e-3, bf16 1e-2), on LSE 1e-3
O_TOL = {"fp16": 2e-3, "bf16": 1e-2}
LSE_TOL = 1e-3

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")


def dev():
    return torch.device("cuda:0")


def f64(t):
    return t.detach().double().cpu().numpy()


def assert_close(o_gpu, lse_gpu, O, L, dtype, what=""):
    o = f64(o_gpu)
    assert np.all(np.isfinite(o)), f"{what}: non-finite O"
    err = np.abs(o - O).max() if o.size else 0.0
    assert err <= O_TOL[dtype], f"{what}: max |O - oracle| = {err:.3e} > {O_TOL[dtype]}"
    if lse_gpu is not None:
        l = f64(lse_gpu)
        inf_g, inf_o = np.isneginf(l), np.isneginf(L)
        assert np.array_equal(inf_g, inf_o), f"{what}: -inf LSE pattern differs"
        fin = ~inf_o
        lerr = np.abs(l[fin] - L[fin]).max() if fin.any() else 0.0
        assert lerr <= LSE_TOL, f"{what}: max |LSE - oracle| = {lerr:.3e} > {LSE_TOL}"
    return err


def run_fwd_case(B, Sq, Sk, Hq, Hkv, D, causal, dtype, seed=1, scale=None, simple=False, in_scale=1.0):
    q, k, v = make_qkv(B, Sq, Sk, Hq, Hkv, D, dtype, seed=seed, input_scale=in_scale)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    fn = sa_attn_fwd_simple if simple else sa_attn_fwd
    o, lse = fn(q.to(dev()), k.to(dev()), v.to(dev()), causal=causal, scale=scale)
    sa_check_status()
    O, L = oracle.attention(f64(q), f64(k), f64(v), scale, causal)
    return assert_close(o, lse, O, L, dtype, f"fwd B{B} Sq{Sq} Sk{Sk} H{Hq}/{Hkv} D{D} c{int(causal)} {dtype}")


def run_decode_case(B, Sk, Hq, Hkv, D, dtype, num_splits=0, seed=2, scale=None):
    q, k, v = make_qkv(B, 1, Sk, Hq, Hkv, D, dtype, seed=seed, decode=True)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o, lse = sa_attn_decode(q.to(dev()), k.to(dev()), v.to(dev()), scale=scale, num_splits=num_splits)
    sa_check_status()
    O, L = oracle.decode(f64(q), f64(k), f64(v), scale)
    return assert_close(o, lse, O, L, dtype, f"decode B{B} Sk{Sk} H{Hq}/{Hkv} D{D} splits{num_splits} {dtype}")
