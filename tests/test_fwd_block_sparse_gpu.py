"""Block-sparse prefill on the GPU (sa_attn_fwd_block_sparse) against the fp64 oracle's
attention_block_sparse: random and Stem-shaped block masks, causal and not, ragged Sq / Sk
(last blocks partial), Sq != Sk, GQA, both head dims and dtypes; a Q tile whose first kept
key block is not its unit's first; empty masks and masks that keep only blocks past the
diagonal; bit identity with the dense forward when every block is kept; the 32768-token
Stem-mask workload at full size on sampled rows."""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import sa_attn_fwd, sa_attn_fwd_block_sparse, sa_check_status
from online_softmax_attention_sm_b200.inputs import make_qkv, make_workload_inputs, sample_rows, stem_block_mask
from online_softmax_attention_sm_b200.workloads import WORKLOADS
from gpu_helpers import assert_close, dev, f64

pytestmark = pytest.mark.gpu


def nblk(n):
    return -(-n // 128)


def run_case(B, Sq, Sk, Hq, Hkv, D, dt, causal, mask, seed):
    q, k, v = make_qkv(B, Sq, Sk, Hq, Hkv, D, dt, seed=seed)
    scale = 1.0 / math.sqrt(D)
    o, lse = sa_attn_fwd_block_sparse(q.to(dev()), k.to(dev()), v.to(dev()), mask.to(dev()), causal=causal,
                                      scale=scale)
    sa_check_status()
    O, L = oracle.attention_block_sparse(f64(q), f64(k), f64(v), mask.numpy(), scale, causal)
    assert_close(o, lse, O, L, dt, f"block-sparse B{B} Sq{Sq} Sk{Sk} H{Hq}/{Hkv} D{D} {dt} c{int(causal)}")


CASES = [
    # B, Sq, Sk, Hq, Hkv, D, dtype, causal, density
    (1, 1024, 1024, 4, 2, 64, "fp16", True, 0.5),
    (2, 700, 900, 4, 4, 128, "bf16", False, 0.4),
    (1, 1000, 1300, 8, 2, 128, "bf16", True, 0.6),     # Sq != Sk, bottom-right
    (2, 513, 513, 3, 1, 64, "bf16", False, 0.25),
    (1, 1536, 1536, 2, 2, 128, "fp16", True, 0.15),
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_block_sparse_random_masks(case):
    B, Sq, Sk, Hq, Hkv, D, dt, causal, dens = case
    seed = zlib.crc32(str(case).encode()) % 1000
    g = torch.Generator().manual_seed(seed)
    mask = (torch.rand((B, Hq, nblk(Sq), nblk(Sk)), generator=g) < dens).to(torch.uint8)
    run_case(B, Sq, Sk, Hq, Hkv, D, dt, causal, mask, seed)


@pytest.mark.parametrize("D,dt", [(64, "fp16"), (128, "bf16")])
def test_block_sparse_stem_mask(D, dt):
    B, S, Hq, Hkv = 1, 4096, 8, 2
    mask = stem_block_mask(B, Hq, S, S, True, seed=17, initial_blocks=2, window_blocks=2, keep_ratio=0.2)
    run_case(B, S, S, Hq, Hkv, D, dt, True, mask, seed=18)


def test_block_sparse_tile_starting_late():
    # query block 0 keeps only key block 5, query block 1 keeps blocks 0-3: the unit's list
    # is 0 1 2 3 5 and Q tile 0 joins at the last step; rows of block 2 keep nothing
    B, S, Hq, Hkv, D = 1, 768, 2, 1, 64
    mask = torch.zeros((B, Hq, 6, 6), dtype=torch.uint8)
    mask[:, :, 0, 5] = 1
    mask[:, :, 1, :4] = 1
    mask[:, :, 3, 1] = 1
    mask[:, :, 4:, 4:] = 1
    run_case(B, S, S, Hq, Hkv, D, "fp16", False, mask, seed=5)


@pytest.mark.parametrize("causal", [False, True])
def test_block_sparse_all_kept_equals_dense_bit_for_bit(causal):
    B, Sq, Sk, Hq, Hkv, D = 2, 900, 900, 4, 2, 128
    q, k, v = (t.to(dev()) for t in make_qkv(B, Sq, Sk, Hq, Hkv, D, "bf16", seed=61))
    mask = torch.ones((B, Hq, nblk(Sq), nblk(Sk)), dtype=torch.uint8, device=dev())
    od, ld = sa_attn_fwd(q, k, v, causal=causal, scale=0.09)
    ob, lb = sa_attn_fwd_block_sparse(q, k, v, mask, causal=causal, scale=0.09)
    sa_check_status()
    assert torch.equal(od, ob) and torch.equal(ld, lb)


def test_block_sparse_nothing_visible():
    # an empty mask, and (causal) a mask that keeps only blocks past the diagonal
    B, S, Hq, Hkv, D = 1, 640, 2, 2, 64
    q, k, v = (t.to(dev()) for t in make_qkv(B, S, S, Hq, Hkv, D, "fp16", seed=7))
    for causal, mask in ((False, torch.zeros((B, Hq, 5, 5), dtype=torch.uint8)),
                         (True, torch.triu(torch.ones((5, 5), dtype=torch.uint8), 1).expand(B, Hq, 5, 5).contiguous())):
        o, lse = sa_attn_fwd_block_sparse(q, k, v, mask.to(dev()), causal=causal)
        sa_check_status()
        rows = slice(0, 512) if causal else slice(0, S)     # causal: the last block keeps nothing past it
        assert torch.all(o[:, rows] == 0) and torch.all(torch.isneginf(lse[:, :, rows]))


def test_block_sparse_32k_stem_workload_sampled_rows():
    w = WORKLOADS["gqa_causal_s32768_d128_bf16_sinks"]
    q, k, v = make_workload_inputs(w)
    mask = stem_block_mask(w.B, w.Hq, w.Sq, w.Sk, True, seed=w.seed + 4)
    o, lse = sa_attn_fwd_block_sparse(q.to(dev()), k.to(dev()), v.to(dev()), mask.to(dev()), causal=True,
                                      scale=w.scale)
    sa_check_status()
    o, lse = o.cpu(), lse.cpu()
    rows = sample_rows(w.Sq, 48, seed=w.seed + 4, extra=(511, 512, 16383, 16384))
    rng = np.random.default_rng(8)
    for h in sorted(set([0, 31] + rng.choice(w.Hq, 3, replace=False).tolist())):
        O, L = oracle.attention_block_sparse_rows(f64(q), f64(k), f64(v), mask.numpy(), w.scale, True, 0, h, rows)
        assert_close(o[0, rows, h], lse[0, h, rows], O, L, "bf16", f"stem 32K head {h}")
