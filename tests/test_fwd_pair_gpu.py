"""The CTA-pair forward (sa_attn_fwd_pair): each unit of 256 query rows on a two-CTA cluster
with 2-SM tensor-core products.  Checked element by element against the fp64 oracle on
ragged, causal / non-causal, Sq != Sk, GQA and both 16-bit dtypes (D = 128), and bit for bit
against the one-CTA kernel, which computes the same arithmetic in the same order."""
import math

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import SAError, sa_attn_fwd, sa_attn_fwd_pair, sa_attn_fwd_varlen, sa_check_status
from online_softmax_attention_sm_b200.inputs import make_qkv
from gpu_helpers import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")

CASES = [
    # B, Sq, Sk, Hq, Hkv, causal, dtype
    (1, 256, 256, 2, 2, False, "bf16"),
    (1, 300, 300, 4, 2, True, "bf16"),
    (1, 300, 300, 4, 2, False, "fp16"),
    (2, 200, 500, 4, 1, True, "bf16"),
    (1, 700, 300, 2, 2, True, "fp16"),       # rows that see no key
    (1, 1000, 1000, 8, 2, True, "bf16"),
    (1, 129, 1025, 2, 2, False, "bf16"),
    (3, 513, 513, 6, 3, True, "fp16"),
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_pair_forward_matches_oracle(case):
    B, Sq, Sk, Hq, Hkv, causal, dt = case
    q, k, v = make_qkv(B, Sq, Sk, Hq, Hkv, 128, dt, seed=sum(case[:5]))
    o, lse = sa_attn_fwd_pair(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal)
    sa_check_status()
    O, L = oracle.attention(f64(q), f64(k), f64(v), 1 / math.sqrt(128), causal)
    assert_close(o, lse, O, L, dt, f"pair {case}")


@pytest.mark.parametrize("case", [(1, 1000, 1000, 8, 2, True, "bf16"), (2, 513, 700, 4, 2, True, "fp16"),
                                  (1, 384, 384, 2, 2, False, "bf16")])
def test_pair_forward_bit_identical_to_the_one_cta_kernel(case):
    # the packed entry point always runs the one-CTA kernel
    B, Sq, Sk, Hq, Hkv, causal, dt = case
    q, k, v = (t.to(DEV) for t in make_qkv(B, Sq, Sk, Hq, Hkv, 128, dt, seed=9))
    op, lp = sa_attn_fwd_pair(q, k, v, causal=causal)
    cq = torch.tensor([Sq * i for i in range(B + 1)], dtype=torch.int32, device=DEV)
    ck = torch.tensor([Sk * i for i in range(B + 1)], dtype=torch.int32, device=DEV)
    ov, lv = sa_attn_fwd_varlen(q.reshape(B * Sq, Hq, 128), k.reshape(B * Sk, Hkv, 128), v.reshape(B * Sk, Hkv, 128),
                                cq, ck, Sq, Sk, causal=causal)
    sa_check_status()
    assert torch.equal(op.reshape(B * Sq, Hq, 128), ov)
    assert torch.equal(lp.permute(1, 0, 2).reshape(Hq, B * Sq), lv)


def test_pair_forward_rejects_d64():
    q, k, v = (t.to(DEV) for t in make_qkv(1, 128, 128, 2, 2, 64, "fp16", seed=1))
    with pytest.raises(SAError):
        sa_attn_fwd_pair(q, k, v)
