"""GPU parity of the split-KV decode (sa_attn_decode: split kernel + PDL combine) against the
fp64 oracle, and its invariants."""
import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import (sa_attn_decode, sa_attn_decode_num_splits,
                                               sa_attn_decode_workspace_size, sa_check_status)
from online_softmax_attention_sm_b200.inputs import make_qkv
from gpu_helpers import assert_close, dev, f64, run_decode_case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Sk", [1, 63, 64, 65, 1000, 4097])
@pytest.mark.parametrize("splits", [1, 2, 0, 10000])
def test_decode_parity(Sk, splits, D, dtype):
    run_decode_case(2, Sk, 14, 2, D, dtype, num_splits=splits, seed=Sk + splits)


@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (8, 8), (8, 1), (16, 1), (20, 1), (32, 2), (7, 7)])
def test_decode_head_packing(Hq, Hkv):
    # G = 1 .. 20: one or two 16-row head groups per KV head
    run_decode_case(3, 777, Hq, Hkv, 64, "fp16", seed=Hq * 10 + Hkv)
    run_decode_case(1, 300, Hq, Hkv, 128, "bf16", num_splits=3, seed=Hq + Hkv)


def test_decode_split_count_invariance():
    q, k, v = make_qkv(2, 1, 5000, 14, 2, 64, "fp16", seed=21, decode=True)
    q, k, v = q.to(dev()), k.to(dev()), v.to(dev())
    ref_o, ref_l = sa_attn_decode(q, k, v, num_splits=1)
    for ns in (2, 5, 17, 0, 79):
        o, l = sa_attn_decode(q, k, v, num_splits=ns)
        assert (o.float() - ref_o.float()).abs().max().item() <= 2e-3
        assert (l - ref_l).abs().max().item() <= 1e-4
    sa_check_status()


def test_decode_deterministic():
    q, k, v = make_qkv(4, 1, 32768, 14, 2, 64, "fp16", seed=22, decode=True)
    q, k, v = q.to(dev()), k.to(dev()), v.to(dev())
    o, l = sa_attn_decode(q, k, v)
    for _ in range(3):
        o2, l2 = sa_attn_decode(q, k, v)
        assert torch.equal(o, o2) and torch.equal(l, l2)
    sa_check_status()


def test_decode_matches_last_prefill_row():
    # a single query sees every key: the decode equals the last causal prefill row
    from online_softmax_attention_sm_b200 import sa_attn_fwd
    q, k, v = make_qkv(1, 700, 700, 8, 2, 64, "fp16", seed=23)
    q, k, v = q.to(dev()), k.to(dev()), v.to(dev())
    o, l = sa_attn_fwd(q, k, v, causal=True)
    od, ld = sa_attn_decode(q[:, -1].contiguous(), k, v)
    sa_check_status()
    assert (od.float() - o[:, -1].float()).abs().max().item() <= 2e-3
    assert (ld - l[:, :, -1]).abs().max().item() <= 1e-3


def test_decode_empty_keys():
    q, k, v = make_qkv(2, 1, 0, 4, 2, 64, "fp16", seed=24, decode=True)
    o, l = sa_attn_decode(q.to(dev()), k.to(dev()), v.to(dev()))
    sa_check_status()
    assert torch.all(o == 0) and torch.all(torch.isneginf(l))


def test_decode_workspace_contract():
    B, Sk, Hq, Hkv, D = 4, 32768, 14, 2, 64
    ns = sa_attn_decode_num_splits(B, Sk, Hq, Hkv, D)
    assert 1 <= ns <= Sk // 64
    need = sa_attn_decode_workspace_size(B, Sk, Hq, Hkv, D)
    assert need == B * Hq * ns * (D + 4) * 4
    q, k, v = make_qkv(B, 1, Sk, Hq, Hkv, D, "fp16", seed=25, decode=True)
    # garbage scratch, canary past the declared size
    ws = torch.full((need + 4096,), 0x5A, dtype=torch.uint8, device=dev())
    o, l = sa_attn_decode(q.to(dev()), k.to(dev()), v.to(dev()), workspace=ws)
    sa_check_status()
    assert torch.all(ws[-4096:] == 0x5A), "wrote past the declared workspace size"
    O, L = oracle.decode(f64(q), f64(k), f64(v), 1 / 8.0)
    assert_close(o, l, O, L, "fp16", "workspace contract")


def test_decode_one_workspace_serves_many_shapes():
    # a serving loop: the KV length grows and the batch changes between calls that reuse
    # one workspace sized for the largest call
    shapes = [(2, 100, 14, 2, 64, "fp16"), (8, 9000, 16, 2, 128, "bf16"), (1, 5000, 8, 8, 64, "fp16"),
              (3, 8191, 16, 1, 128, "bf16"), (2, 101, 14, 2, 64, "fp16")]
    ws = torch.full((max(sa_attn_decode_workspace_size(*sh[:5]) for sh in shapes),), 0x77,
                    dtype=torch.uint8, device=dev())
    for i, (B, Sk, Hq, Hkv, D, dt) in enumerate(shapes):
        q, k, v = make_qkv(B, 1, Sk, Hq, Hkv, D, dt, seed=30 + i, decode=True)
        o, l = sa_attn_decode(q.to(dev()), k.to(dev()), v.to(dev()), workspace=ws)
        sa_check_status()
        O, L = oracle.decode(f64(q), f64(k), f64(v), 1 / np.sqrt(D))
        assert_close(o, l, O, L, dt, f"reuse #{i}")
