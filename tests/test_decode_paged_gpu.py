"""Paged-KV decode on the GPU (sa_attn_decode_paged) against the fp64 oracle's
decode_paged: caches of shuffled pages, sequences of their own lengths (empty, one token,
ragged last pages, multi-page), page sizes 64/128/256, both head dims and dtypes; bit
identity with the dense decode when the same keys sit in pages; the 32K decode workload in
paged form at full size."""
import zlib

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import sa_attn_decode, sa_attn_decode_paged, sa_check_status
from online_softmax_attention_sm_b200.inputs import make_qkv
from gpu_helpers import assert_close, dev, f64

pytestmark = pytest.mark.gpu

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}


def paged_inputs(B, Hq, Hkv, D, dtype, page_size, lens, seed, spare_pages=3):
    """Random q and a page pool holding each sequence's keys in shuffled pages (plus unused
    pages), with the block table that finds them.  Lengths may be 0 or ragged."""
    max_blocks = max(1, max(-(-n // page_size) for n in lens))
    Sk = max_blocks * page_size
    q, k, v = make_qkv(B, 1, Sk, Hq, Hkv, D, dtype, seed=seed, decode=True)
    n_pages = B * max_blocks + spare_pages
    g = torch.Generator().manual_seed(seed + 7)
    perm = torch.randperm(n_pages, generator=g)[:B * max_blocks]
    table = perm.view(B, max_blocks).to(torch.int32)
    kc = torch.randn((n_pages, page_size, Hkv, D), generator=g).to(q.dtype)   # junk in unused rows
    vc = torch.randn((n_pages, page_size, Hkv, D), generator=g).to(q.dtype)
    for b in range(B):
        for i in range(max_blocks):
            kc[table[b, i]] = k[b, i * page_size:(i + 1) * page_size]
            vc[table[b, i]] = v[b, i * page_size:(i + 1) * page_size]
    seqlens = torch.tensor(lens, dtype=torch.int32)
    return q, kc, vc, table, seqlens


CASES = [
    # B, Hq, Hkv, D, dtype, page_size, lengths
    (3, 14, 2, 64, "fp16", 64, [1000, 64, 1]),
    (4, 8, 8, 128, "bf16", 128, [0, 129, 300, 4096]),
    (2, 16, 1, 64, "bf16", 256, [777, 513]),
    (5, 7, 7, 128, "fp16", 64, [65, 63, 0, 2000, 1]),
    (1, 32, 8, 128, "bf16", 64, [5000]),
]


@pytest.mark.parametrize("case", CASES)
def test_paged_decode_matches_oracle(case):
    B, Hq, Hkv, D, dt, ps, lens = case
    q, kc, vc, table, seqlens = paged_inputs(B, Hq, Hkv, D, dt, ps, lens, seed=zlib.crc32(str(case).encode()) % 1000)
    scale = 1.0 / np.sqrt(D)
    O, L = oracle.decode_paged(f64(q), f64(kc), f64(vc), table.numpy(), seqlens.numpy(), scale)
    o, lse = sa_attn_decode_paged(q.to(dev()), kc.to(dev()), vc.to(dev()), table.to(dev()), seqlens.to(dev()),
                                  scale=scale)
    sa_check_status()
    assert_close(o, lse, O, L, dt, f"paged {case}")


@pytest.mark.parametrize("num_splits", [1, 3, 40])
def test_paged_decode_any_split_count(num_splits):
    B, Hq, Hkv, D, dt, ps, lens = 2, 6, 2, 64, "fp16", 64, [3000, 700]
    q, kc, vc, table, seqlens = paged_inputs(B, Hq, Hkv, D, dt, ps, lens, seed=31)
    O, L = oracle.decode_paged(f64(q), f64(kc), f64(vc), table.numpy(), seqlens.numpy(), 0.125)
    o, lse = sa_attn_decode_paged(q.to(dev()), kc.to(dev()), vc.to(dev()), table.to(dev()), seqlens.to(dev()),
                                  scale=0.125, num_splits=num_splits)
    sa_check_status()
    assert_close(o, lse, O, L, dt, f"num_splits={num_splits}")


@pytest.mark.parametrize("D,dt,ps", [(64, "fp16", 64), (128, "bf16", 128)])
def test_paged_equals_dense_bit_for_bit(D, dt, ps):
    # the same keys in shuffled pages: same plan, same arithmetic, only the addresses differ
    B, Hq, Hkv, Sk = 3, 8, 2, 4096
    q, kc, vc, table, seqlens = paged_inputs(B, Hq, Hkv, D, dt, ps, [Sk] * B, seed=77)
    k = torch.stack([torch.cat([kc[table[b, i]] for i in range(Sk // ps)]) for b in range(B)])
    v = torch.stack([torch.cat([vc[table[b, i]] for i in range(Sk // ps)]) for b in range(B)])
    od, ld = sa_attn_decode(q.to(dev()), k.to(dev()), v.to(dev()), scale=0.1)
    op, lp = sa_attn_decode_paged(q.to(dev()), kc.to(dev()), vc.to(dev()), table.to(dev()), seqlens.to(dev()),
                                  scale=0.1)
    sa_check_status()
    assert torch.equal(od, op) and torch.equal(ld, lp)


def test_paged_decode_32k_workload_matches_dense():
    # gqa_decode_sk32768_d64_fp16 with its K/V cut into 64-token pages and shuffled
    B, Hq, Hkv, D, Sk, ps = 4, 14, 2, 64, 32768, 64
    q, k, v = (t.to(dev()) for t in make_qkv(B, 1, Sk, Hq, Hkv, D, "fp16", seed=20261202 + 4, decode=True))
    nb = Sk // ps
    perm = torch.randperm(B * nb, generator=torch.Generator().manual_seed(5)).to(dev())
    kc = torch.empty((B * nb, ps, Hkv, D), dtype=k.dtype, device=dev())
    vc = torch.empty_like(kc)
    kc[perm] = k.reshape(B * nb, ps, Hkv, D)
    vc[perm] = v.reshape(B * nb, ps, Hkv, D)
    table = perm.view(B, nb).to(torch.int32)
    seqlens = torch.full((B,), Sk, dtype=torch.int32, device=dev())
    od, ld = sa_attn_decode(q, k, v)
    op, lp = sa_attn_decode_paged(q, kc, vc, table, seqlens)
    sa_check_status()
    assert torch.equal(od, op) and torch.equal(ld, lp)


def test_paged_decode_lengths_beyond_the_table_are_clamped():
    B, Hq, Hkv, D, dt, ps, lens = 2, 4, 1, 64, "fp16", 64, [200, 90]
    q, kc, vc, table, seqlens = paged_inputs(B, Hq, Hkv, D, dt, ps, lens, seed=3)
    long = torch.tensor([10 ** 6, -5], dtype=torch.int32)          # -> the whole table, and 0
    O, L = oracle.decode_paged(f64(q), f64(kc), f64(vc), table.numpy(), long.numpy(), 0.125)
    o, lse = sa_attn_decode_paged(q.to(dev()), kc.to(dev()), vc.to(dev()), table.to(dev()), long.to(dev()),
                                  scale=0.125)
    sa_check_status()
    assert_close(o, lse, O, L, dt, "clamped lengths")
    assert torch.all(o[1] == 0) and torch.all(torch.isneginf(lse[1]))
