"""Attention backward on the GPU (sa_attn_bwd) against the fp64 oracle's attention_backward:
dQ, dK, dV for a seeded upstream gradient, causal and not, ragged and unequal lengths
(bottom-right alignment, rows without keys), GQA (dK / dV summed over the query heads of a
KV head), both head dims and dtypes; the causal-leak property (dQ of row i bit-identical when
keys after i change); determinism; zero-size problems."""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import sa_attn_bwd, sa_attn_fwd, sa_check_status
from online_softmax_attention_sm_b200.inputs import make_dout, make_qkv
from gpu_helpers import dev, f64

pytestmark = pytest.mark.gpu

# max-abs tolerance on dQ, dK, dV, derived from the arithmetic: each gradient is rounded
# once to the I/O dtype (at most u |g|, u = 2^-11 fp16, 2^-8 bf16) and its fp32 sums
# multiply operands that were each rounded once (P, dS, and O inside Delta), whose errors
# stay within about 2u of the result; so 3u * max(1, max |g|), and never below the
# flash-attn-volta page's 3e-3 budget for its fp16 backward.  (Causal dV grows with the
# sequence: the first keys collect the weights of every row, |dV| ~ 7 at 1024 rows.)
UNIT = {"fp16": 2.0 ** -11, "bf16": 2.0 ** -8}


def tol(dt, ref):
    return max(3e-3 if dt == "fp16" else 0.0, 3 * UNIT[dt] * max(1.0, float(np.abs(ref).max())))


def run(B, Sq, Sk, Hq, Hkv, D, dt, causal, seed, scale=None):
    q, k, v = make_qkv(B, Sq, Sk, Hq, Hkv, D, dt, seed=seed)
    do = make_dout(B, Sq, Hq, D, dt, seed=seed)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    qd, kd, vd, dod = (t.to(dev()) for t in (q, k, v, do))
    o, lse = sa_attn_fwd(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = sa_attn_bwd(qd, kd, vd, o, lse, dod, causal=causal, scale=scale)
    sa_check_status()
    return (q, k, v, do, scale), (dq, dk, dv)


CASES = [
    # B, Sq, Sk, Hq, Hkv, D, dtype, causal
    (1, 256, 256, 2, 2, 64, "fp16", True),
    (2, 300, 300, 4, 4, 128, "bf16", False),
    (1, 640, 640, 8, 2, 128, "bf16", True),
    (1, 200, 450, 4, 1, 64, "fp16", True),       # Sq < Sk: chunk after a cached prefix
    (1, 450, 200, 2, 2, 64, "bf16", True),       # Sq > Sk: the first 250 rows see no key
    (2, 129, 257, 6, 3, 128, "fp16", False),
    (1, 1024, 1024, 4, 1, 64, "bf16", True),
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_backward_matches_oracle(case):
    B, Sq, Sk, Hq, Hkv, D, dt, causal = case
    (q, k, v, do, scale), got = run(B, Sq, Sk, Hq, Hkv, D, dt, causal, seed=zlib.crc32(str(case).encode()) % 1000)
    want = oracle.attention_backward(f64(q), f64(k), f64(v), f64(do), scale, causal)
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        g = f64(g)
        assert np.all(np.isfinite(g)), f"{case} {name}: non-finite"
        err, t = np.abs(g - w).max(), tol(dt, w)
        assert err <= t, f"{case} {name}: max |err| = {err:.3e} > {t:.3e}"


def test_backward_causal_leak_and_determinism():
    # dQ of row i depends on no key after i: change keys and values after row 300 and rows
    # 0-300 of dQ stay bit-identical; a second run gives identical bits
    B, S, Hq, Hkv, D = 1, 512, 4, 2, 128
    q, k, v = (t.to(dev()) for t in make_qkv(B, S, S, Hq, Hkv, D, "bf16", seed=91))
    do = make_dout(B, S, Hq, D, "bf16", seed=91).to(dev())
    o, lse = sa_attn_fwd(q, k, v, causal=True)
    dq, dk, dv = sa_attn_bwd(q, k, v, o, lse, do, causal=True)
    dq2, dk2, dv2 = sa_attn_bwd(q, k, v, o, lse, do, causal=True)
    sa_check_status()
    assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2)
    k3, v3 = k.clone(), v.clone()
    k3[:, 301:] = torch.randn_like(k3[:, 301:].float()).to(k3.dtype)
    v3[:, 301:] = torch.randn_like(v3[:, 301:].float()).to(v3.dtype)
    o3, lse3 = sa_attn_fwd(q, k3, v3, causal=True)
    dq3, _, _ = sa_attn_bwd(q, k3, v3, o3, lse3, do, causal=True)
    sa_check_status()
    assert torch.equal(dq[:, :301], dq3[:, :301])


def test_backward_empty_problems_zero_fill():
    q, k, v = (t.to(dev()) for t in make_qkv(1, 0, 64, 2, 2, 64, "fp16", seed=1))
    o = torch.empty_like(q)
    lse = torch.empty((1, 2, 0), dtype=torch.float32, device=dev())
    dk = torch.full_like(k, 5.0)
    dv = torch.full_like(v, 5.0)
    sa_attn_bwd(q, k, v, o, lse, torch.empty_like(q), dk=dk, dv=dv)
    sa_check_status()
    assert torch.all(dk == 0) and torch.all(dv == 0)
