"""FP8 (e4m3) forward on the GPU (sa_attn_fwd_fp8) against the fp64 oracle's attention_fp8
(attention of the dequantised inputs): causal and not, ragged lengths, Sq != Sk, GQA.

Tolerance, derived from the arithmetic: the products Q K^T of e4m3 values are exact and
summed in fp32, so the error of O comes from rounding each weight p_j = 2^(s_j - m) to e4m3
for P V (relative error u = 2^-4 for normal values; O is normalised by the sum of the
rounded weights, so O_gpu - O = sum_j (p~_j - p_j)(v_j - O) / sum_j p~_j) and from rounding
O to bf16 (2^-8 |O|):
    |O_gpu - O| <= u/(1-u) sum_j P_j |v_j - O| + 2^-8 |O| + a,
with P the exact normalised weights.  Weights below e4m3's normal range (2^-6 of the
reference) have an absolute rounding error of at most 2^-10 instead; `a` = 2e-3 covers
their sum here (their errors are unbiased; at most a few hundredths of the mass sit there).
The LSE uses fp32 sums of unrounded weights: 1e-3 as for the 16-bit forward."""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import sa_attn_fwd_block_sparse_fp8, sa_attn_fwd_fp8, sa_check_status
from online_softmax_attention_sm_b200.inputs import make_qkv_fp8, stem_block_mask

pytestmark = pytest.mark.gpu

U = 2.0 ** -4


def first_order_bound(q, k, v, scale, causal, O, block_mask=None):
    """Per-element bound u/(1-u) sum_j P_ij |v_jd - O_id| + 2^-8 |O_id| + 2e-3 from the
    dequantised inputs and the oracle's O (numpy float64, [B,S,H,D] layouts); with a block
    mask, P is over the keys the mask keeps."""
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    bound = np.zeros_like(O)
    rows, cols = np.arange(Sq)[:, None], np.arange(Sk)[None, :]
    vis = (cols <= rows + Sk - Sq) if causal else np.ones((Sq, Sk), bool)
    for b in range(B):
        for h in range(Hq):
            vbh = vis if block_mask is None else vis & block_mask[b, h][rows // 128, cols // 128]
            s = np.where(vbh, scale * q[b, :, h] @ k[b, :, h // G].T, -np.inf)
            m = s.max(axis=1, keepdims=True)
            m = np.where(np.isfinite(m), m, 0.0)
            p = np.exp(s - m)
            p /= np.maximum(p.sum(axis=1, keepdims=True), 1e-300)
            vv = v[b, :, h // G]                                    # [Sk, D]
            dev_ = np.abs(vv[None, :, :] - O[b, :, h][:, None, :])  # [Sq, Sk, D]
            bound[b, :, h] = U / (1 - U) * np.einsum("ij,ijd->id", p, dev_)
    return bound + 2.0 ** -8 * np.abs(O) + 2e-3


CASES = [
    # B, Sq, Sk, Hq, Hkv, causal
    (1, 300, 300, 2, 2, False),
    (1, 700, 700, 4, 1, True),
    (2, 200, 500, 4, 2, True),
    (1, 129, 1000, 2, 2, False),
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_fp8_forward_within_the_derived_bound(case):
    B, Sq, Sk, Hq, Hkv, causal = case
    q8, k8, v8, qd, kd, vd = make_qkv_fp8(B, Sq, Sk, Hq, Hkv, 128, seed=zlib.crc32(str(case).encode()) % 1000)
    scale = 1.0 / math.sqrt(128)
    dev = torch.device("cuda:0")
    o, lse = sa_attn_fwd_fp8(q8.to(dev), k8.to(dev), v8.to(dev), qd, kd, vd, causal=causal, scale=scale)
    sa_check_status()
    O, L = oracle.attention_fp8(q8.numpy(), k8.numpy(), v8.numpy(), qd, kd, vd, scale, causal)
    q, k, v = (oracle.decode_e4m3(x.numpy()) * d for x, d in ((q8, qd), (k8, kd), (v8, vd)))
    og, lg = o.double().cpu().numpy(), lse.double().cpu().numpy()
    assert np.all(np.isfinite(og))
    err = np.abs(og - O)
    bound = first_order_bound(q, k, v, scale, causal, O)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), f"{case}: err {err[worst]:.3e} > bound {bound[worst]:.3e} at {worst}"
    fin = np.isfinite(L)
    assert np.array_equal(np.isneginf(lg), np.isneginf(L))
    assert np.abs(lg[fin] - L[fin]).max() <= 1e-3


@pytest.mark.parametrize("causal", [True, False])
def test_fp8_block_sparse_within_the_derived_bound(causal):
    # the Stem page's fp8 block-sparse prefill: a Stem-shaped mask over e4m3 inputs
    B, S, Hq, Hkv = 1, 1024, 4, 2
    q8, k8, v8, qd, kd, vd = make_qkv_fp8(B, S, S, Hq, Hkv, 128, seed=71 + int(causal))
    mask = stem_block_mask(B, Hq, S, S, causal, seed=5, initial_blocks=1, window_blocks=2, keep_ratio=0.3)
    scale = 1.0 / math.sqrt(128)
    dev = torch.device("cuda:0")
    o, lse = sa_attn_fwd_block_sparse_fp8(q8.to(dev), k8.to(dev), v8.to(dev), mask.to(dev), qd, kd, vd,
                                          causal=causal, scale=scale)
    sa_check_status()
    q, k, v = (oracle.decode_e4m3(x.numpy()) * d for x, d in ((q8, qd), (k8, kd), (v8, vd)))
    O, L = oracle.attention_block_sparse(q, k, v, mask.numpy(), scale, causal)
    og, lg = o.double().cpu().numpy(), lse.double().cpu().numpy()
    err = np.abs(og - O)
    bound = first_order_bound(q, k, v, scale, causal, O, block_mask=mask.numpy() != 0)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), f"err {err[worst]:.3e} > bound {bound[worst]:.3e} at {worst}"
    fin = np.isfinite(L)
    assert np.array_equal(np.isneginf(lg), np.isneginf(L))
    assert np.abs(lg[fin] - L[fin]).max() <= 1e-3
