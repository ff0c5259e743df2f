"""Parity at the full workload sizes, in the launch configuration the bench times.

Prefill workloads up to 4096 tokens are checked on every output; the 32768-token GQA
workload (full S x S scores would be 32 GiB in fp64) on a seeded sample of rows per head:
the four sink rows, the rows around the first tile boundaries, the last row and 256
uniform rows.  Its backward (the bench's seeded dO) on dQ of sampled rows of every head
and on dK / dV of keys in the last five key tiles (the rows that see them are few enough
to form whole).  The decode workload is checked in full."""
import math

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import sa_attn_bwd, sa_attn_decode, sa_attn_fwd, sa_check_status
from online_softmax_attention_sm_b200.inputs import make_dout, make_workload_inputs, sample_rows
from online_softmax_attention_sm_b200.workloads import WORKLOADS
from gpu_helpers import LSE_TOL, O_TOL, assert_close, dev, f64

pytestmark = pytest.mark.gpu

FULL = ["mha_s128_d64_fp16", "mha_causal_s2048_d64_fp16", "mha_s4096_d128_bf16",
        "mha_causal_s4096_d128_bf16"]


@pytest.mark.parametrize("name", FULL)
def test_prefill_workload_full(name):
    w = WORKLOADS[name]
    q, k, v = make_workload_inputs(w)
    o, lse = sa_attn_fwd(q.to(dev()), k.to(dev()), v.to(dev()), causal=w.causal, scale=w.scale)
    sa_check_status()
    O, L = oracle.attention(f64(q), f64(k), f64(v), w.scale, w.causal)
    assert_close(o, lse, O, L, w.dtype, name)


def test_long_gqa_causal_sampled_rows():
    w = WORKLOADS["gqa_causal_s32768_d128_bf16_sinks"]
    q, k, v = make_workload_inputs(w)
    o, lse = sa_attn_fwd(q.to(dev()), k.to(dev()), v.to(dev()), causal=True, scale=w.scale)
    sa_check_status()
    o, lse = o.cpu(), lse.cpu()
    qn, kn, vn = q.float().numpy(), k.float().numpy(), v.float().numpy()   # exact widening
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    worst_o = worst_l = 0.0
    for h in range(w.Hq):
        rows = sample_rows(w.Sq, 256, seed=w.seed + h, extra=(32767,))
        O, L = oracle.attention_rows(qn, kn, vn, w.scale, True, 0, h, rows)
        worst_o = max(worst_o, np.abs(f64(o[0, rows, h]) - O).max())
        worst_l = max(worst_l, np.abs(f64(lse[0, h, rows]) - L).max())
    assert worst_o <= O_TOL["bf16"], f"max |O - oracle| on sampled rows = {worst_o:.3e}"
    assert worst_l <= LSE_TOL, f"max |LSE - oracle| on sampled rows = {worst_l:.3e}"


# backward tolerance: 3u * max |g| over the sample (u = 2^-8 for bf16: one rounding of the
# result, one of each multiplied 16-bit operand).  dQ keeps the small-size tests' floor,
# 3u * max(1, max |g|); the last keys' dK and dV are sums over a few rows of weights near
# 1 / Sk (|g| ~ 1e-2 at 32768 keys), where a floor of 1 would accept all-zero gradients
BWD_UNIT = {"fp16": 2.0 ** -11, "bf16": 2.0 ** -8}


def backward_sampled_errors(q, k, v, do, grads, scale, dtype, n_rows, keys, kv_heads, seed):
    """(name, max |err|, tolerance) of dQ on sampled rows of every query head and of dK, dV
    on `keys` of `kv_heads`, against the oracle's sampled backward (batch 0, causal)."""
    qn, kn, vn, don = (t.float().numpy() for t in (q, k, v, do))     # exact widening
    dq, dk, dv = (f64(g) for g in grads)
    u = BWD_UNIT[dtype]
    Sq, Hq = q.shape[1], q.shape[2]
    got, want = [], []
    for h in range(Hq):
        rows = sample_rows(Sq, n_rows, seed=seed + h, extra=(Sq - 1,))
        want.append(oracle.attention_backward_rows(qn, kn, vn, don, scale, True, 0, h, rows))
        got.append(dq[0, rows, h])
    got, want = np.concatenate(got), np.concatenate(want)
    out = [("dq", np.abs(got - want).max(), 3 * u * max(1.0, np.abs(want).max()))]
    gk, gv, wk, wv = [], [], [], []
    for kvh in kv_heads:
        a, b = oracle.attention_backward_keys(qn, kn, vn, don, scale, True, 0, kvh, keys)
        wk.append(a)
        wv.append(b)
        gk.append(dk[0, keys, kvh])
        gv.append(dv[0, keys, kvh])
    for name, g, w in (("dk", gk, wk), ("dv", gv, wv)):
        g, w = np.concatenate(g), np.concatenate(w)
        out.append((name, np.abs(g - w).max(), 3 * u * np.abs(w).max()))
    for name, g in zip(("dq", "dk", "dv"), (dq, dk, dv)):
        out.append((name + " finite", 0.0 if np.all(np.isfinite(g)) else np.inf, 0.0))
    return out


def test_long_gqa_causal_backward_sampled():
    w = WORKLOADS["gqa_causal_s32768_d128_bf16_sinks"]
    q, k, v = make_workload_inputs(w)
    do = make_dout(w.B, w.Sq, w.Hq, w.D, w.dtype, seed=w.seed)
    qd, kd, vd, dod = (t.to(dev()) for t in (q, k, v, do))
    o, lse = sa_attn_fwd(qd, kd, vd, causal=True, scale=w.scale)
    grads = sa_attn_bwd(qd, kd, vd, o, lse, dod, causal=True, scale=w.scale)
    sa_check_status()
    grads = tuple(g.cpu() for g in grads)
    del qd, kd, vd, dod, o, lse
    Sk = w.Sk
    keys = sorted({Sk - 640, Sk - 639, Sk - 513, Sk - 512, Sk - 385, Sk - 384, Sk - 257, Sk - 256,
                   Sk - 129, Sk - 128, Sk - 70, Sk - 2, Sk - 1})
    for name, err, tol in backward_sampled_errors(q, k, v, do, grads, w.scale, w.dtype, n_rows=24, keys=keys,
                                                  kv_heads=(0, w.Hkv - 1), seed=w.seed):
        assert err <= tol, f"{name}: max |err| on the sample = {err:.3e} > {tol:.3e}"


def test_decode_workload_full():
    w = WORKLOADS["gqa_decode_sk32768_d64_fp16"]
    q, k, v = make_workload_inputs(w)
    o, lse = sa_attn_decode(q.to(dev()), k.to(dev()), v.to(dev()), scale=w.scale)
    sa_check_status()
    O, L = oracle.decode(f64(q), f64(k), f64(v), w.scale)
    assert_close(o, lse, O, L, w.dtype, w.name)
