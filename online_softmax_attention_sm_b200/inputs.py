"""Seeded synthetic inputs shared by the CUDA path's tests, the bench and the oracle.

This module only draws random numbers and rounds them to the storage dtype; it
contains none of the attention arithmetic.  Recipe (fixed, so every consumer sees
identical bits):

* one CPU ``torch.Generator`` seeded with ``seed``; Q, then K, then V are drawn in
  that order as float32 N(0,1) (``torch.randn``);
* each is multiplied by ``input_scale`` (exact for powers of two);
* K rows ``0 .. k_sink_rows-1`` (every batch and KV head) are multiplied by
  ``k_sink_factor`` (x8 is exact), V is left alone;
* the float32 values are rounded to fp16 / bf16 (round-to-nearest-even).

Layouts: prefill Q [B, Sq, Hq, D], K/V [B, Sk, Hkv, D]; decode Q [B, Hq, D].
All tensors are contiguous CPU tensors of the storage dtype.

Packed variable-length batches draw their sequence lengths with :func:`varlen_lengths`
and their tokens with ``make_qkv(1, total, total, ...)`` (sequence after sequence).
"""
from __future__ import annotations

import torch

DTYPES = {"fp16": torch.float16, "bf16": torch.bfloat16, "fp32": torch.float32}


def make_qkv(B, Sq, Sk, Hq, Hkv, D, dtype="fp16", seed=0, input_scale=1.0,
             k_sink_rows=0, k_sink_factor=1.0, decode=False):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    qshape = (B, Hq, D) if decode else (B, Sq, Hq, D)
    q = torch.randn(qshape, generator=g, dtype=torch.float32)
    k = torch.randn((B, Sk, Hkv, D), generator=g, dtype=torch.float32)
    v = torch.randn((B, Sk, Hkv, D), generator=g, dtype=torch.float32)
    if input_scale != 1.0:
        q.mul_(input_scale)
        k.mul_(input_scale)
        v.mul_(input_scale)
    if k_sink_rows:
        k[:, :k_sink_rows].mul_(k_sink_factor)
    t = DTYPES[dtype]
    return q.to(t).contiguous(), k.to(t).contiguous(), v.to(t).contiguous()


def make_workload_inputs(w, seed=None):
    """Inputs of a :class:`workloads.Workload` (decode workloads give Q as [B, Hq, D])."""
    return make_qkv(w.B, w.Sq, w.Sk, w.Hq, w.Hkv, w.D, w.dtype,
                    w.seed if seed is None else seed, w.input_scale,
                    w.k_sink_rows, w.k_sink_factor, decode=(w.kind == "decode"))


def sample_rows(Sq, n_random, seed, extra=()):
    """Seeded set of query rows for checking a long sequence row by row: the
    first four rows, the rows around the first 128-row tile boundaries, the last
    row, any ``extra`` rows, plus ``n_random`` uniform rows.  Sorted, unique, < Sq."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 7919)
    fixed = [0, 1, 2, 3, 127, 128, 129, 255, 256, 257, Sq - 1] + list(extra)
    rnd = torch.randint(0, Sq, (n_random,), generator=g).tolist() if n_random else []
    return sorted({r for r in fixed + rnd if 0 <= r < Sq})


def varlen_lengths(total, n, seed):
    """A seeded mix of n sequence lengths (each >= 1) summing to `total`: weights
    2^(4u), u ~ U(0, 1) (a 16x spread between the shortest and the longest), scaled to
    the total and floored, the remainder given one token at a time to the first
    sequences."""
    if n <= 0 or total < n:
        raise ValueError("need 1 <= n <= total")
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 104729)
    w = torch.pow(2.0, 4.0 * torch.rand(n, generator=g, dtype=torch.float64))
    lens = [max(1, int(x)) for x in (w / w.sum() * total).floor().tolist()]
    i = 0
    while sum(lens) < total:
        lens[i % n] += 1
        i += 1
    while sum(lens) > total:                  # only if flooring to >= 1 overshot
        j = max(range(n), key=lambda t: lens[t])
        lens[j] -= 1
    return lens


def stem_block_mask(B, Hq, Sq, Sk, causal, seed, initial_blocks=4, window_blocks=4, keep_ratio=0.1,
                    block=128):
    """A seeded block mask [B, Hq, ceil(Sq/block), ceil(Sk/block)] (uint8, 1 = keep) shaped like
    the selection of the Stem page's block-sparse prefill: for every query block, the first
    `initial_blocks` key blocks (sinks) and the last `window_blocks` key blocks it can see
    (sliding window) are kept, and of the key blocks in between a fraction `keep_ratio`
    (rounded) is drawn uniformly at random -- a stand-in for the page's top-k by block score.
    "Can see": with causal, up to the block holding key (last row of the query block) +
    Sk - Sq; otherwise every key block."""
    nq, nk = -(-Sq // block), -(-Sk // block)
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 611953)
    mask = torch.zeros((B, Hq, nq, nk), dtype=torch.uint8)
    for qi in range(nq):
        last_row = min(Sq, (qi + 1) * block) - 1
        kmax = min(nk - 1, (last_row + Sk - Sq) // block) if causal else nk - 1
        if kmax < 0:
            continue
        lo, hi = min(initial_blocks, kmax + 1), max(0, kmax + 1 - window_blocks)
        mask[:, :, qi, :lo] = 1
        mask[:, :, qi, hi:kmax + 1] = 1
        mid = hi - lo
        take = int(round(keep_ratio * mid)) if mid > 0 else 0
        if take:
            r = torch.rand((B, Hq, mid), generator=g)
            idx = r.topk(take, dim=-1).indices + lo
            mask[:, :, qi].scatter_(-1, idx, 1)
    return mask


def make_dout(B, Sq, Hq, D, dtype="fp16", seed=0):
    """Upstream gradient dO [B, Sq, Hq, D] for the backward: float32 N(0,1) from a generator
    seeded with seed + 7777, rounded to the storage dtype."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 7777)
    return torch.randn((B, Sq, Hq, D), generator=g, dtype=torch.float32).to(DTYPES[dtype]).contiguous()


def quantize_e4m3(x):
    """Per-tensor FP8 quantisation of a float tensor: descale = max |x| / 448 (448 is the
    largest e4m3 value), codes = x / descale rounded to e4m3 (torch's float8_e4m3fn
    conversion, round to nearest even), returned as a uint8 tensor of codes and the float
    descale factor (x ~ value(codes) * descale)."""
    amax = float(x.abs().max())
    d = amax / 448.0 if amax > 0 else 1.0
    return (x / d).to(torch.float8_e4m3fn).view(torch.uint8).contiguous(), d


def make_qkv_fp8(B, Sq, Sk, Hq, Hkv, D, seed=0, input_scale=1.0, k_sink_rows=0, k_sink_factor=1.0):
    """make_qkv's float32 draws (same recipe and seed), each tensor quantised to e4m3 with
    its own descale: returns (q8, k8, v8, q_descale, k_descale, v_descale)."""
    q, k, v = make_qkv(B, Sq, Sk, Hq, Hkv, D, "fp32", seed, input_scale, k_sink_rows, k_sink_factor)
    (q8, qd), (k8, kd), (v8, vd) = quantize_e4m3(q), quantize_e4m3(k), quantize_e4m3(v)
    return q8, k8, v8, qd, kd, vd
