"""Packed variable-length prefill on the GPU (sa_attn_fwd_varlen) against the fp64 oracle's
attention_varlen: ragged mixes that span several 128-row tiles and end mid-tile, empty
sequences and sequences without keys, query chunks shorter than their keys (bottom-right
causal alignment), GQA, both head dims and dtypes; rows outside every sequence untouched;
bit identity with the dense forward for equal lengths; invalid offsets reported through
the device status word; the 32768-token length mix at full size on sampled rows."""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import SAError, sa_attn_fwd, sa_attn_fwd_varlen, sa_check_status
from online_softmax_attention_sm_b200.inputs import make_qkv, varlen_lengths
from gpu_helpers import assert_close, dev, f64

pytestmark = pytest.mark.gpu


def packed_inputs(lens_q, lens_k, Hq, Hkv, D, dtype, seed, lead=0, tail=0):
    """Seeded packed q [lead + sum(lens_q) + tail, Hq, D], k/v [sum(lens_k) + tail, Hkv, D] and
    int32 offsets (sequence 0 starting at query row `lead`)."""
    cq = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32) + lead
    ck = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    tq, tk = int(cq[-1]) + tail, int(ck[-1]) + tail
    q, k, v = make_qkv(1, tq, tk, Hq, Hkv, D, dtype, seed=seed)
    return q[0], k[0], v[0], torch.from_numpy(cq), torch.from_numpy(ck)


def run_varlen(q, k, v, cq, ck, causal, scale, out=None, lse=None):
    lq = (cq[1:] - cq[:-1]).tolist()
    lk = (ck[1:] - ck[:-1]).tolist()
    return sa_attn_fwd_varlen(q.to(dev()), k.to(dev()), v.to(dev()), cq.to(dev()), ck.to(dev()),
                              max(lq + [0]), max(lk + [0]), causal=causal, scale=scale, out=out, lse=lse)


CASES = [
    # lengths q, lengths k (None: same), Hq, Hkv, D, dtype, causal
    ([1, 127, 128, 129, 300, 0, 513], None, 4, 2, 64, "fp16", True),
    ([1000, 3, 256, 257], None, 8, 2, 128, "bf16", False),
    ([200, 64, 1], [1000, 64, 300], 6, 3, 64, "bf16", True),       # chunks after cached prefixes
    ([5, 40, 130], [0, 70, 130], 4, 4, 128, "fp16", False),        # a sequence without keys
    ([2048, 700, 1, 255], None, 16, 4, 128, "bf16", True),
    ([333, 1200], [100, 1500], 7, 7, 64, "fp16", True),            # queries beyond their keys too
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_varlen_matches_oracle(case):
    lq, lk, Hq, Hkv, D, dt, causal = case
    lk = lq if lk is None else lk
    q, k, v, cq, ck = packed_inputs(lq, lk, Hq, Hkv, D, dt, seed=zlib.crc32(str(case).encode()) % 1000)
    scale = 1.0 / math.sqrt(D)
    o, lse = run_varlen(q, k, v, cq, ck, causal, scale)
    sa_check_status()
    O, L = oracle.attention_varlen(f64(q), f64(k), f64(v), cq.numpy(), ck.numpy(), scale, causal)
    assert_close(o, lse, O, L, dt, f"varlen {case}")


def test_varlen_leaves_rows_outside_the_sequences_alone():
    lq = [70, 0, 260]
    q, k, v, cq, ck = packed_inputs(lq, lq, 4, 2, 64, "bf16", seed=5, lead=9, tail=21)
    out = torch.full(q.shape, 7.0, dtype=q.dtype, device=dev())
    lse = torch.full((4, q.shape[0]), 5.0, dtype=torch.float32, device=dev())
    run_varlen(q, k, v, cq, ck, True, 0.125, out=out, lse=lse)
    sa_check_status()
    O, L = oracle.attention_varlen(f64(q), f64(k), f64(v), cq.numpy(), ck.numpy(), 0.125, True)
    a, b = int(cq[0]), int(cq[-1])
    assert_close(out[a:b], lse[:, a:b], O[a:b], L[:, a:b], "bf16", "covered rows")
    assert torch.all(out[:a] == 7.0) and torch.all(out[b:] == 7.0)
    assert torch.all(lse[:, :a] == 5.0) and torch.all(lse[:, b:] == 5.0)


@pytest.mark.parametrize("D,dt,causal", [(64, "fp16", True), (128, "bf16", True), (128, "fp16", False)])
def test_varlen_equal_lengths_equal_dense_bit_for_bit(D, dt, causal):
    B, S, Hq, Hkv = 3, 777, 8, 2
    q, k, v = make_qkv(B, S, S, Hq, Hkv, D, dt, seed=41)
    od, ld = sa_attn_fwd(q.to(dev()), k.to(dev()), v.to(dev()), causal=causal, scale=0.1)
    cu = torch.arange(0, (B + 1) * S, S, dtype=torch.int32)
    ov, lv = run_varlen(q.reshape(B * S, Hq, D), k.reshape(B * S, Hkv, D), v.reshape(B * S, Hkv, D), cu, cu,
                        causal, 0.1)
    sa_check_status()
    assert torch.equal(od.reshape(B * S, Hq, D), ov)
    assert torch.equal(ld.permute(1, 0, 2).reshape(Hq, B * S), lv)


def test_varlen_reports_a_sequence_longer_than_max_seqlen():
    lq = [100, 600]
    q, k, v, cq, ck = packed_inputs(lq, lq, 2, 1, 64, "fp16", seed=3)
    sa_attn_fwd_varlen(q.to(dev()), k.to(dev()), v.to(dev()), cq.to(dev()), ck.to(dev()), 256, 600,
                       causal=True)
    with pytest.raises(SAError, match="max_seqlen_q"):
        sa_check_status()
    # offsets running backwards are reported the same way, and nothing is written outside
    bad = torch.tensor([0, 300, 200], dtype=torch.int32)
    out = torch.zeros(q.shape, dtype=q.dtype, device=dev())
    sa_attn_fwd_varlen(q.to(dev()), k.to(dev()), v.to(dev()), bad.to(dev()), ck.to(dev()), 600, 600,
                       causal=True, out=out)
    with pytest.raises(SAError):
        sa_check_status()
    # the status word is cleared: the next valid call reports nothing
    o, lse = run_varlen(q, k, v, cq, ck, True, 0.125)
    sa_check_status()
    O, L = oracle.attention_varlen(f64(q), f64(k), f64(v), cq.numpy(), ck.numpy(), 0.125, True)
    assert_close(o, lse, O, L, "fp16", "after a reported error")


def test_varlen_32k_mix_sampled_rows():
    # the 32768-token length mix of the varlen prefill workload (Hq 32, Hkv 8, D 128, bf16,
    # causal) at full size; the oracle on sampled rows of every sequence
    lens = varlen_lengths(32768, 16, seed=20261202 + 6)
    Hq, Hkv, D = 32, 8, 128
    q, k, v, cq, ck = packed_inputs(lens, lens, Hq, Hkv, D, "bf16", seed=20261202 + 6)
    scale = 1.0 / math.sqrt(D)
    o, lse = run_varlen(q, k, v, cq, ck, True, scale)
    sa_check_status()
    o, lse = o.cpu(), lse.cpu()
    rng = np.random.default_rng(6)
    for b, n in enumerate(lens):
        a = int(cq[b])
        rows = sorted({0, 127, 128, n - 1} | set(rng.integers(0, n, 6).tolist()))
        rows = [r for r in rows if 0 <= r < n]
        qs, ks, vs = q[None, a:a + n], k[None, a:a + n], v[None, a:a + n]
        for h in rng.choice(Hq, 3, replace=False):
            O, L = oracle.attention_rows(f64(qs), f64(ks), f64(vs), scale, True, 0, int(h), rows)
            idx = [a + r for r in rows]
            assert_close(o[idx, h], lse[h, idx], O, L, "bf16", f"seq {b} (len {n}) head {h}")
