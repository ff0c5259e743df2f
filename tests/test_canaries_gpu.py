"""Out-of-bounds writes, checked without a memory checker: every output and workspace of the
backward, block-sparse, paged (prefill and decode), FP8 and CTA-pair paths is a window into a
larger buffer whose pads hold a sentinel, and the pads must come back untouched (and the
windows correct against the oracle).  Ragged sizes, so the last tiles are partial."""
import math

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import (sa_attn_bwd, sa_attn_bwd_workspace_size, sa_attn_decode_paged,
                                               sa_attn_decode_paged_workspace_size, sa_attn_fwd,
                                               sa_attn_fwd_block_sparse, sa_attn_fwd_block_sparse_workspace_size,
                                               sa_attn_fwd_fp8, sa_attn_fwd_paged, sa_attn_fwd_pair, sa_check_status)
from online_softmax_attention_sm_b200.inputs import make_dout, make_qkv, make_qkv_fp8, stem_block_mask
from gpu_helpers import assert_close, f64
from test_decode_paged_gpu import paged_inputs
from test_fwd_paged_gpu import paged_case

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
PAD = 4096


class Guarded:
    """A tensor of `shape` inside a buffer with PAD sentinel elements on both sides."""

    def __init__(self, shape, dtype, sentinel):
        n = int(np.prod(shape))
        self.buf = torch.full((PAD + n + PAD,), sentinel, dtype=dtype, device=DEV)
        self.t = self.buf[PAD:PAD + n].view(*shape)
        self.sentinel = sentinel

    def intact(self):
        return bool(torch.all(self.buf[:PAD] == self.sentinel)) and bool(torch.all(self.buf[-PAD:] == self.sentinel))


def test_backward_writes_only_its_gradients_and_workspace():
    B, Sq, Sk, Hq, Hkv, D, dt = 1, 300, 423, 4, 2, 64, "bf16"
    q, k, v = (t.to(DEV) for t in make_qkv(B, Sq, Sk, Hq, Hkv, D, dt, seed=61))
    do = make_dout(B, Sq, Hq, D, dt, seed=61).to(DEV)
    o, lse = sa_attn_fwd(q, k, v, causal=True)
    gq = Guarded(q.shape, q.dtype, 5.0)
    gk, gv = Guarded(k.shape, k.dtype, 5.0), Guarded(v.shape, v.dtype, 5.0)
    need = sa_attn_bwd_workspace_size(B, Sq, Hq)
    ws = Guarded((need,), torch.uint8, 0x5A)
    sa_attn_bwd(q, k, v, o, lse, do, causal=True, workspace=ws.t, dq=gq.t, dk=gk.t, dv=gv.t)
    sa_check_status()
    assert gq.intact() and gk.intact() and gv.intact() and ws.intact()
    want = oracle.attention_backward(f64(q), f64(k), f64(v), f64(do), 1 / math.sqrt(D), True)
    for got, ref in zip((gq.t, gk.t, gv.t), want):
        assert np.abs(f64(got) - ref).max() <= 3 * 2.0 ** -8 * max(1.0, float(np.abs(ref).max()))


def test_block_sparse_writes_only_its_outputs_and_list_workspace():
    B, Sq, Sk, Hq, Hkv, D, dt = 1, 700, 555, 4, 2, 128, "fp16"
    q, k, v = make_qkv(B, Sq, Sk, Hq, Hkv, D, dt, seed=62)
    mask = stem_block_mask(B, Hq, Sq, Sk, True, seed=3, initial_blocks=1, window_blocks=1, keep_ratio=0.5)
    need = sa_attn_fwd_block_sparse_workspace_size(B, Sq, Sk, Hq)
    ws = Guarded((need,), torch.uint8, 0x5A)
    go, gl = Guarded((B, Sq, Hq, D), torch.float16, 7.0), Guarded((B, Hq, Sq), torch.float32, 9.0)
    sa_attn_fwd_block_sparse(q.to(DEV), k.to(DEV), v.to(DEV), mask.to(DEV), causal=True, workspace=ws.t, out=go.t,
                             lse=gl.t)
    sa_check_status()
    assert go.intact() and gl.intact() and ws.intact()
    O, L = oracle.attention_block_sparse(f64(q), f64(k), f64(v), mask.numpy(), 1 / math.sqrt(D), True)
    assert_close(go.t, gl.t, O, L, dt, "block-sparse canaries")


def test_paged_prefill_writes_only_its_outputs():
    lq, lk, Hq, Hkv, D, dt, page = [100, 1, 300], [612, 1, 300], 4, 2, 128, "bf16", 128
    q, _, _, kc, vc, table, sk, cq = paged_case(lq, lk, Hq, Hkv, D, dt, page, seed=63)
    tq = sum(lq)
    go, gl = Guarded((tq, Hq, D), q.dtype, 7.0), Guarded((Hq, tq), torch.float32, 9.0)
    sa_attn_fwd_paged(q.to(DEV), kc.to(DEV), vc.to(DEV), cq.to(DEV), table.to(DEV), sk.to(DEV), max(lq), causal=True,
                      out=go.t, lse=gl.t)
    sa_check_status()
    assert go.intact() and gl.intact()
    O, L = oracle.attention_paged_prefill(f64(q), f64(kc), f64(vc), cq.numpy(), table.numpy(), sk.numpy(),
                                          1 / math.sqrt(D), True)
    assert_close(go.t, gl.t, O, L, dt, "paged prefill canaries")


def test_paged_decode_writes_only_its_outputs_and_workspace():
    B, Hq, Hkv, D, dt, ps, lens = 5, 7, 7, 128, "fp16", 64, [65, 63, 0, 2000, 1]
    q, kc, vc, table, seqlens = paged_inputs(B, Hq, Hkv, D, dt, ps, lens, seed=64)
    need = sa_attn_decode_paged_workspace_size(B, Hq, Hkv, D, ps, table.shape[1])
    ws = Guarded((need,), torch.uint8, 0x5A)
    go, gl = Guarded((B, Hq, D), q.dtype, 7.0), Guarded((B, Hq), torch.float32, 9.0)
    sa_attn_decode_paged(q.to(DEV), kc.to(DEV), vc.to(DEV), table.to(DEV), seqlens.to(DEV), workspace=ws.t, out=go.t,
                         lse=gl.t)
    sa_check_status()
    assert go.intact() and gl.intact() and ws.intact()
    O, L = oracle.decode_paged(f64(q), f64(kc), f64(vc), table.numpy(), seqlens.numpy(), 1 / math.sqrt(D))
    assert_close(go.t, gl.t, O, L, dt, "paged decode canaries")


def test_fp8_and_pair_forwards_write_only_their_outputs():
    B, S, Hq, Hkv = 1, 333, 4, 2
    q8, k8, v8, qd, kd, vd = make_qkv_fp8(B, S, S, Hq, Hkv, 128, seed=65)
    go, gl = Guarded((B, S, Hq, 128), torch.bfloat16, 7.0), Guarded((B, Hq, S), torch.float32, 9.0)
    sa_attn_fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), qd, kd, vd, causal=True, out=go.t, lse=gl.t)
    sa_check_status()
    assert go.intact() and gl.intact()
    q, k, v = (t.to(DEV) for t in make_qkv(B, S, S, Hq, Hkv, 128, "bf16", seed=66))
    go, gl = Guarded((B, S, Hq, 128), torch.bfloat16, 7.0), Guarded((B, Hq, S), torch.float32, 9.0)
    sa_attn_fwd_pair(q, k, v, causal=True, out=go.t, lse=gl.t)
    sa_check_status()
    assert go.intact() and gl.intact()
    O, L = oracle.attention(f64(q), f64(k), f64(v), 1 / math.sqrt(128), True)
    assert_close(go.t, gl.t, O, L, "bf16", "pair canaries")
