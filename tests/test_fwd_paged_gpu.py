"""Packed queries against a paged K/V cache on the GPU (sa_attn_fwd_paged, chunked prefill)
against the fp64 oracle's attention_paged_prefill: shuffled pages of 128 and 256 keys,
query chunks shorter than their keys (bottom-right causal alignment), full prefills,
sequences without keys, lengths past the table (clamped), GQA, both head dims and dtypes;
bit identity with the packed (varlen) forward when the same keys sit in pages."""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import sa_attn_fwd_paged, sa_attn_fwd_varlen, sa_check_status
from online_softmax_attention_sm_b200.inputs import make_qkv
from gpu_helpers import assert_close, dev, f64

pytestmark = pytest.mark.gpu


def paged_case(lens_q, lens_k, Hq, Hkv, D, dt, page, seed, spare=2):
    """Packed q, and the keys of each sequence in shuffled pages of a cache (plus spare
    pages of junk), with the block table and the key lengths."""
    max_blocks = max(1, max(-(-n // page) for n in lens_k))
    tq, tk = sum(lens_q), sum(lens_k)
    q, k, v = (t[0] for t in make_qkv(1, tq, max(tk, 1), Hq, Hkv, D, dt, seed=seed))
    n_pages = len(lens_k) * max_blocks + spare
    g = torch.Generator().manual_seed(seed + 1)
    perm = torch.randperm(n_pages, generator=g)
    kc = torch.randn((n_pages, page, Hkv, D), generator=g).to(q.dtype)
    vc = torch.randn((n_pages, page, Hkv, D), generator=g).to(q.dtype)
    table = torch.zeros((len(lens_k), max_blocks), dtype=torch.int32)
    k0 = 0
    for b, n in enumerate(lens_k):
        for i in range(max_blocks):
            slot = int(perm[b * max_blocks + i])
            table[b, i] = slot
            rows = max(0, min(page, n - i * page))
            if rows:
                kc[slot, :rows] = k[k0 + i * page:k0 + i * page + rows]
                vc[slot, :rows] = v[k0 + i * page:k0 + i * page + rows]
        k0 += n
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lens_q)]), dtype=torch.int32)
    return q, k, v, kc, vc, table, torch.tensor(lens_k, dtype=torch.int32), cq


CASES = [
    # lengths q, lengths k, Hq, Hkv, D, dtype, page, causal
    ([100, 1, 300], [612, 1, 300], 4, 2, 128, "bf16", 128, True),     # chunks after cached prefixes
    ([257, 50], [257, 700], 8, 2, 64, "fp16", 256, True),
    ([64, 200], [0, 900], 4, 4, 128, "fp16", 128, False),              # a sequence without keys
    ([129, 129], [129, 1000], 6, 3, 64, "bf16", 128, False),
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_paged_prefill_matches_oracle(case):
    lq, lk, Hq, Hkv, D, dt, page, causal = case
    q, _, _, kc, vc, table, sk, cq = paged_case(lq, lk, Hq, Hkv, D, dt, page, seed=zlib.crc32(str(case).encode()) % 1000)
    scale = 1.0 / math.sqrt(D)
    o, lse = sa_attn_fwd_paged(q.to(dev()), kc.to(dev()), vc.to(dev()), cq.to(dev()), table.to(dev()), sk.to(dev()),
                               max(lq), causal=causal, scale=scale)
    sa_check_status()
    O, L = oracle.attention_paged_prefill(f64(q), f64(kc), f64(vc), cq.numpy(), table.numpy(), sk.numpy(), scale,
                                          causal)
    assert_close(o, lse, O, L, dt, f"paged prefill {case}")


def test_paged_prefill_clamps_lengths_past_the_table():
    lq, lk = [50, 50], [300, 256]
    q, _, _, kc, vc, table, sk, cq = paged_case(lq, lk, 2, 1, 64, "fp16", 128, seed=4)
    long = torch.tensor([10 ** 6, 256], dtype=torch.int32)       # -> the table's 384 keys
    o, lse = sa_attn_fwd_paged(q.to(dev()), kc.to(dev()), vc.to(dev()), cq.to(dev()), table.to(dev()),
                               long.to(dev()), 50, causal=True, scale=0.125)
    sa_check_status()
    O, L = oracle.attention_paged_prefill(f64(q), f64(kc), f64(vc), cq.numpy(), table.numpy(), long.numpy(), 0.125,
                                          True)
    assert_close(o, lse, O, L, "fp16", "clamped")


@pytest.mark.parametrize("causal", [True, False])
def test_paged_prefill_equals_varlen_bit_for_bit(causal):
    lens = [700, 129, 1000]
    q, k, v, kc, vc, table, sk, cq = paged_case(lens, lens, 8, 2, 128, "bf16", 128, seed=12)
    ov, lv = sa_attn_fwd_varlen(q.to(dev()), k.to(dev()), v.to(dev()), cq.to(dev()), cq.to(dev()), 1000, 1000,
                                causal=causal, scale=0.1)
    op, lp = sa_attn_fwd_paged(q.to(dev()), kc.to(dev()), vc.to(dev()), cq.to(dev()), table.to(dev()), sk.to(dev()),
                               1000, causal=causal, scale=0.1)
    sa_check_status()
    assert torch.equal(ov, op) and torch.equal(lv, lp)
