"""Single-kernel split-KV decode on the GPU (sa_attn_decode_single: the last split of each
head tile merges, no combine launch) against the fp64 oracle's decode, bit identity with
the two-kernel decode (same partial states, same merge arithmetic), repeated calls (the
arrival counters reset themselves), and the 32768-key workload."""
import math

import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import sa_attn_decode, sa_attn_decode_single, sa_check_status
from online_softmax_attention_sm_b200.inputs import make_qkv
from gpu_helpers import assert_close, dev, f64

pytestmark = pytest.mark.gpu

CASES = [
    # B, Sk, Hq, Hkv, D, dtype, num_splits
    (1, 32768, 14, 2, 64, "fp16", 0),
    (2, 5000, 8, 8, 128, "bf16", 0),
    (3, 777, 32, 4, 64, "bf16", 5),
    (1, 64, 16, 1, 128, "fp16", 1),
    (4, 2048, 6, 3, 64, "fp16", 40),
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_single_kernel_decode_matches_oracle_and_two_kernel(case):
    B, Sk, Hq, Hkv, D, dt, ns = case
    q, k, v = make_qkv(B, 1, Sk, Hq, Hkv, D, dt, seed=Sk + B, decode=True)
    scale = 1.0 / math.sqrt(D)
    qd, kd, vd = q.to(dev()), k.to(dev()), v.to(dev())
    o1, l1 = sa_attn_decode_single(qd, kd, vd, scale=scale, num_splits=ns)
    o2, l2 = sa_attn_decode(qd, kd, vd, scale=scale, num_splits=ns)
    sa_check_status()
    O, L = oracle.decode(f64(q), f64(k), f64(v), scale)
    assert_close(o1, l1, O, L, dt, f"single {case}")
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_single_kernel_decode_repeated_calls():
    # each tile's last split zeroes its counter: back-to-back calls stay correct
    q, k, v = (t.to(dev()) for t in make_qkv(4, 1, 32768, 14, 2, 64, "fp16", seed=20261202 + 4, decode=True))
    ref, lref = sa_attn_decode(q, k, v)
    for _ in range(20):
        o, l = sa_attn_decode_single(q, k, v)
    sa_check_status()
    assert torch.equal(o, ref) and torch.equal(l, lref)
