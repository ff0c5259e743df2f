"""Parity with the fp64 oracle at sizes the other tests leave out: a long-context decode at
D = 128 (its split cap of 96), a large-batch decode (many head tiles in the grid's y and z),
and a long D = 64 prefill (GQA causal, 8192 tokens, fp16 and bf16) checked on sampled rows
of every head, the last row included.

The prefill's keys carry sinks (the first 4 keys scaled by 8), so many rows are dominated by
one or two V rows and |O| reaches 2-4, where one rounding of O to the output dtype is worth up
to 2^-9 |O| (bf16) or 2^-12 |O| (fp16) on its own; the O bound is the fixed tolerance of the
other tests plus 2^-8 |O| (bf16) or 2^-11 |O| (fp16), twice that rounding."""
import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import sa_attn_decode_num_splits, sa_attn_fwd, sa_check_status
from online_softmax_attention_sm_b200.inputs import make_qkv, sample_rows
from gpu_helpers import LSE_TOL, O_TOL, dev, f64, run_decode_case

pytestmark = pytest.mark.gpu


def test_long_decode_d128():
    # 32768 keys at D = 128 for one KV head: the automatic plan hits the 96-split cap of the
    # D = 128 combine, then rounds each split up to whole 64-token stages (ceil(32768 / 96)
    # -> 384 tokens): 86 splits
    assert sa_attn_decode_num_splits(1, 32768, 8, 1, 128) == 86
    run_decode_case(1, 32768, 8, 1, 128, "bf16", seed=41)


def test_large_batch_decode():
    # 96 sequences x 8 KV heads x 2 head groups (G = 20): 1536 head tiles
    run_decode_case(96, 1000, 160, 8, 64, "fp16", seed=42)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_long_prefill_d64_sampled_rows(dtype):
    B, S, Hq, Hkv, D = 1, 8192, 16, 4, 64
    q, k, v = make_qkv(B, S, S, Hq, Hkv, D, dtype, seed=43, k_sink_rows=4, k_sink_factor=8.0)
    scale = 1.0 / np.sqrt(D)
    o, lse = sa_attn_fwd(q.to(dev()), k.to(dev()), v.to(dev()), causal=True, scale=scale)
    sa_check_status()
    o, lse = o.cpu(), lse.cpu()
    qn, kn, vn = q.float().numpy(), k.float().numpy(), v.float().numpy()   # exact widening
    rel = {"fp16": 2.0 ** -11, "bf16": 2.0 ** -8}[dtype]
    worst_o = worst_l = 0.0
    for h in range(Hq):
        rows = sample_rows(S, 48, seed=43 + h, extra=(0, 127, 128, S - 1))
        O, L = oracle.attention_rows(qn, kn, vn, scale, True, 0, h, rows)
        err = np.abs(f64(o[0, rows, h]) - O)
        worst_o = max(worst_o, (err / (O_TOL[dtype] + rel * np.abs(O))).max())
        worst_l = max(worst_l, np.abs(f64(lse[0, h, rows]) - L).max())
    assert worst_o <= 1.0, f"max |O - oracle| / (tolerance + rel |O|) on sampled rows = {worst_o:.3f}"
    assert worst_l <= LSE_TOL, f"max |LSE - oracle| on sampled rows = {worst_l:.3e}"
