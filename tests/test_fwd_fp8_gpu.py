"""FP8 (e4m3) forward on the GPU (sa_attn_fwd_fp8) against the fp64 oracle's attention_fp8
(attention of the dequantised inputs): causal and not, ragged lengths, Sq != Sk, GQA.

Tolerance, derived from the arithmetic: the products Q K^T of e4m3 values are exact and
summed in fp32, so the error of O comes from rounding each weight p_j = 2^(s_j - m) to e4m3
for P V (relative error u = 2^-4 for normal values; O is normalised by the sum of the
rounded weights, so O_gpu - O = sum_j (p~_j - p_j)(v_j - O) / sum_j p~_j) and from rounding
O to bf16 (2^-8 |O|):
    |O_gpu - O| <= u/(1-u) sum_j P_j |v_j - O| + 2^-8 |O| + a,
with P the exact normalised weights.  Weights below e4m3's normal range (under 2^-14 of the
row max, the kernel offsetting its weights by 2^8) have an absolute rounding error of at most
2^-18 of the row max instead; `a` = 2e-3 covers their sum at up to 1024 keys.
The LSE uses fp32 sums of unrounded weights: 1e-3 as for the 16-bit forward.

At the bench's 32768-token size the weights below e4m3's normal range matter: the kernel
writes them as p_j = 2^(s_j - m_ref + 8) with its reference m_ref at most 0.75 (log2 units)
below the row max, so only a weight under 2^-14 of the row max can be subnormal (under 2^-6
after the offset), with an absolute rounding error of at most 2^-10, i.e. 2^-18 of the row
max, and only one under 2^-18 of the max can round to zero.  On long rows that a few sink keys dominate, tens
of thousands of weights sit there.  The check on sampled rows is the first-order bound of
the normal-range weights plus one fixed absolute term,
    |O_gpu - O| <= (u/(1-u) + 1e-4) sum_j P_j |v_j - O| + 2^-8 |O| + 2e-3 + A,   A = 0.05,
the 1e-4 for the exponentials computed on the FMA pipe (relative error 7.6e-5).  A covers the
subnormal and zero weights: their errors are signed (round to nearest), each at most
min(p_j, 2^-18) of the row max, and their sum in O, sum_j (p~_j - p_j)(v_j - O) / sum_j p~_j,
stays under 0.04 on every sampled row in a host emulation of the kernel's rounding.  The
worst case of that sum, sum_j min(p_j, 2^-18) |v_j - O| / ((1-u) sum_j p_j), is checked
as well (a second bound that holds whatever the signs).
The LSE, from unrounded weights, keeps its 1e-3."""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import sa_attn_fwd_block_sparse_fp8, sa_attn_fwd_fp8, sa_check_status
from online_softmax_attention_sm_b200.inputs import make_qkv_fp8, sample_rows, stem_block_mask
from online_softmax_attention_sm_b200.workloads import WORKLOADS

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


A_FIXED = 0.05          # the subnormal and zero weights' share of the O error (module docstring)
SUBNORMAL = 2.0 ** -18  # e4m3's subnormal spacing (2^-9) over 2 and the offset 2^8, relative to the row max


def long_row_bounds(k, v, q_rows, scale, rows, Sq, O):
    """The two bounds of the module docstring for query rows `rows` (causal, bottom-right) of
    one head: k, v [Sk, D] and q_rows [n, D] dequantised float64, O [n, D] the oracle's output
    of those rows.  Returns (fixed, worst): fixed = first-order + A, worst = first-order + the
    subnormal worst case; both [n, D]."""
    Sk = k.shape[0]
    fixed, worst = np.zeros_like(O), np.zeros_like(O)
    for r, i in enumerate(rows):
        n = min(Sk, i + Sk - Sq + 1)
        s = scale * (k[:n] @ q_rows[r])
        p = np.exp(s - s.max())                           # relative to the row max
        Z = p.sum()
        dev_ = np.abs(v[:n] - O[r])
        base = (U / (1 - U) + 1e-4) * (p @ dev_) / Z + 2.0 ** -8 * np.abs(O[r]) + 2e-3
        fixed[r] = base + A_FIXED
        worst[r] = base + (np.minimum(p, SUBNORMAL) @ dev_) / ((1 - U) * Z)
    return fixed, worst


def fp8_sampled_errors(q8, k8, v8, qd, kd, vd, scale, o, lse, heads, n_rows, seed):
    """Largest |O - oracle| / bound (the fixed and the worst-case bound) and |LSE - oracle|
    over sampled rows of `heads` (batch 0, causal): o [B, Sq, Hq, D] and lse [B, Hq, Sq] as
    float64 arrays."""
    Sq, Hq = q8.shape[1], q8.shape[2]
    G = Hq // k8.shape[2]
    worst_fixed = worst_case = worst_l = 0.0
    for h in heads:
        kvh = h // G
        qh = oracle.decode_e4m3(q8[:, :, h:h + 1].numpy()) * qd
        kh = oracle.decode_e4m3(k8[:, :, kvh:kvh + 1].numpy()) * kd
        vh = oracle.decode_e4m3(v8[:, :, kvh:kvh + 1].numpy()) * vd
        rows = sample_rows(Sq, n_rows, seed=seed + h, extra=(Sq - 1,))
        O, L = oracle.attention_rows(qh, kh, vh, scale, True, 0, 0, rows)
        fixed, worst = long_row_bounds(kh[0, :, 0], vh[0, :, 0], qh[0, rows, 0], scale, rows, Sq, O)
        err = np.abs(o[0, rows, h] - O)
        worst_fixed = max(worst_fixed, float((err / fixed).max()))
        worst_case = max(worst_case, float((err / worst).max()))
        worst_l = max(worst_l, float(np.abs(lse[0, h, rows] - L).max()))
    return worst_fixed, worst_case, worst_l


def test_fp8_long_gqa_causal_sampled_rows():
    # the bench's FP8 leg: the 32768-token GQA workload's draws (sinks included) in e4m3
    w = WORKLOADS["gqa_causal_s32768_d128_bf16_sinks"]
    q8, k8, v8, qd, kd, vd = make_qkv_fp8(w.B, w.Sq, w.Sk, w.Hq, w.Hkv, w.D, seed=w.seed,
                                          input_scale=w.input_scale, k_sink_rows=w.k_sink_rows,
                                          k_sink_factor=w.k_sink_factor)
    dev = torch.device("cuda:0")
    o, lse = sa_attn_fwd_fp8(q8.to(dev), k8.to(dev), v8.to(dev), qd, kd, vd, causal=True, scale=w.scale)
    sa_check_status()
    o, lse = o.double().cpu().numpy(), lse.double().cpu().numpy()
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    worst_fixed, worst_case, worst_l = fp8_sampled_errors(q8, k8, v8, qd, kd, vd, w.scale, o, lse,
                                                          heads=range(0, w.Hq, 4), n_rows=24, seed=w.seed)
    assert worst_fixed <= 1.0, f"max |O - oracle| / (first-order + {A_FIXED}) on sampled rows = {worst_fixed:.3f}"
    assert worst_case <= 1.0, f"max |O - oracle| / (first-order + subnormal worst case) = {worst_case:.3f}"
    assert worst_l <= 1e-3, f"max |LSE - oracle| on sampled rows = {worst_l:.3e}"
