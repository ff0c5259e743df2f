"""GPU parity of the tcgen05 prefill kernel (sa_attn_fwd) against the fp64 oracle, plus
the invariants that need no oracle: causal leak, GQA vs repeated KV, determinism,
buffer canaries, empty and fully masked inputs."""
import math

import numpy as np
import pytest
import torch

import oracle
from online_softmax_attention_sm_b200 import sa_attn_fwd, sa_check_status
from online_softmax_attention_sm_b200.inputs import make_qkv
from gpu_helpers import assert_close, dev, f64, run_fwd_case

pytestmark = pytest.mark.gpu

# shapes spanning several 128-row tiles and 256-row units, ragged tails on both sides,
# Sq != Sk both ways, G in {1, 2, 4, 7, 8}
SHAPES = [
    # B, Sq,  Sk,  Hq, Hkv, D
    (1, 1, 1, 1, 1, 64),
    (1, 7, 7, 2, 2, 64),
    (1, 127, 127, 2, 1, 64),
    (1, 128, 128, 2, 2, 64),
    (1, 129, 129, 4, 2, 128),
    (2, 255, 255, 2, 2, 128),
    (1, 256, 256, 4, 1, 64),
    (1, 300, 300, 7, 1, 128),
    (2, 1000, 1000, 8, 1, 64),
    (1, 513, 1000, 4, 4, 128),
    (1, 1000, 513, 4, 2, 64),
    (1, 1, 777, 4, 2, 128),
    (1, 200, 64, 2, 2, 128),
]


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_fwd_parity(shape, causal, dtype):
    B, Sq, Sk, Hq, Hkv, D = shape
    run_fwd_case(B, Sq, Sk, Hq, Hkv, D, causal, dtype, seed=hash(shape) % 1000)


@pytest.mark.parametrize("scale", [0.0, -0.2, 0.5])
def test_fwd_scale_values(scale):
    # scale 0: every visible key has the same weight; negative scales flip the ordering
    run_fwd_case(1, 300, 300, 2, 1, 64, True, "fp16", seed=3, scale=scale)
    run_fwd_case(1, 300, 300, 2, 1, 128, False, "bf16", seed=4, scale=scale)


def test_fwd_zero_query_is_mean_of_values():
    q, k, v = make_qkv(1, 256, 256, 2, 2, 64, "fp16", seed=5)
    q.zero_()
    o, lse = sa_attn_fwd(q.to(dev()), k.to(dev()), v.to(dev()), causal=True)
    sa_check_status()
    vv = f64(v)[0, :, :, :]
    ref = np.cumsum(vv, axis=0) / np.arange(1, 257)[:, None, None]
    np.testing.assert_allclose(f64(o)[0], ref, atol=2e-3)
    np.testing.assert_allclose(f64(lse)[0], np.log(np.arange(1, 257))[None, :].repeat(2, 0), atol=1e-3)


def test_fwd_large_magnitudes_stay_finite():
    # scores of several hundred: no overflow thanks to the running max.  Inputs are 6x the
    # workloads' N(0,1), so |O| reaches ~20 and rounding O to bf16 alone costs up to half
    # an ulp there (0.0625): the absolute tolerance scales with the values, here by 8.
    q, k, v = make_qkv(1, 600, 600, 2, 2, 128, "bf16", seed=6, input_scale=6.0)
    o, lse = sa_attn_fwd(q.to(dev()), k.to(dev()), v.to(dev()), causal=True)
    sa_check_status()
    O, L = oracle.attention(f64(q), f64(k), f64(v), 1 / math.sqrt(128), True)
    assert np.all(np.isfinite(f64(o))) and np.all(np.isfinite(f64(lse)))
    assert np.abs(f64(o) - O).max() <= 8e-2
    assert np.abs(f64(lse) - L).max() <= 1e-3


def test_fwd_causal_leak_bit_identical():
    # flash-attn-volta page, "Backward correctness": perturbing keys/values after row i
    # must leave row i bit-identical; here for the forward
    q, k, v = make_qkv(1, 640, 640, 4, 2, 128, "bf16", seed=7)
    q, k, v = q.to(dev()), k.to(dev()), v.to(dev())
    o, lse = sa_attn_fwd(q, k, v, causal=True)
    for i in (0, 127, 128, 255, 256, 383, 500):
        k2, v2 = k.clone(), v.clone()
        k2[:, i + 1:] = torch.randn_like(k2[:, i + 1:].float()).to(k2.dtype) * 4
        v2[:, i + 1:] = -v2[:, i + 1:]
        o2, lse2 = sa_attn_fwd(q, k2, v2, causal=True)
        assert torch.equal(o2[:, :i + 1], o[:, :i + 1]), f"row <= {i} changed"
        assert torch.equal(lse2[:, :, :i + 1], lse[:, :, :i + 1])
    sa_check_status()


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_gqa_equals_repeated_kv(causal):
    q, k, v = make_qkv(2, 300, 300, 8, 2, 64, "fp16", seed=8)
    q, k, v = q.to(dev()), k.to(dev()), v.to(dev())
    o, lse = sa_attn_fwd(q, k, v, causal=causal)
    o2, lse2 = sa_attn_fwd(q, k.repeat_interleave(4, dim=2).contiguous(),
                           v.repeat_interleave(4, dim=2).contiguous(), causal=causal)
    sa_check_status()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_fwd_deterministic():
    q, k, v = make_qkv(1, 1000, 1000, 4, 2, 128, "bf16", seed=9)
    q, k, v = q.to(dev()), k.to(dev()), v.to(dev())
    o, lse = sa_attn_fwd(q, k, v, causal=True)
    for _ in range(3):
        o2, lse2 = sa_attn_fwd(q, k, v, causal=True)
        assert torch.equal(o, o2) and torch.equal(lse, lse2)
    sa_check_status()


def test_fwd_writes_only_its_outputs():
    # canaries around O and LSE stand in for a memory checker
    B, S, H, D = 1, 300, 2, 64
    q, k, v = make_qkv(B, S, S, H, H, D, "fp16", seed=10)
    pad = 4096
    obuf = torch.full((pad + B * S * H * D + pad,), 7.0, dtype=torch.float16, device=dev())
    lbuf = torch.full((pad + B * H * S + pad,), 9.0, dtype=torch.float32, device=dev())
    o = obuf[pad:pad + B * S * H * D].view(B, S, H, D)
    lse = lbuf[pad:pad + B * H * S].view(B, H, S)
    sa_attn_fwd(q.to(dev()), k.to(dev()), v.to(dev()), causal=True, out=o, lse=lse)
    sa_check_status()
    assert torch.all(obuf[:pad] == 7.0) and torch.all(obuf[-pad:] == 7.0)
    assert torch.all(lbuf[:pad] == 9.0) and torch.all(lbuf[-pad:] == 9.0)
    O, L = oracle.attention(f64(q), f64(k), f64(v), 1 / 8.0, True)
    assert_close(o, lse, O, L, "fp16", "canary case")


def test_fwd_without_lse():
    q, k, v = make_qkv(1, 200, 200, 2, 2, 64, "fp16", seed=11)
    o, lse = sa_attn_fwd(q.to(dev()), k.to(dev()), v.to(dev()), causal=False, return_lse=False)
    sa_check_status()
    assert lse is None
    O, _ = oracle.attention(f64(q), f64(k), f64(v), 1 / 8.0, False)
    assert_close(o, None, O, None, "fp16", "no lse")


def test_fwd_empty_keys_and_fully_masked_rows():
    q, k, v = make_qkv(1, 40, 0, 2, 2, 64, "fp16", seed=12)
    o, lse = sa_attn_fwd(q.to(dev()), k.to(dev()), v.to(dev()))
    sa_check_status()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
    # causal with Sq > Sk: the first Sq - Sk rows see no key
    run_fwd_case(1, 400, 100, 2, 1, 128, True, "bf16", seed=13)
    run_fwd_case(2, 300, 30, 2, 2, 64, True, "fp16", seed=14)


def test_fwd_non_default_stream():
    q, k, v = make_qkv(1, 300, 300, 2, 2, 64, "fp16", seed=15)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o, lse = sa_attn_fwd(q.to(dev()), k.to(dev()), v.to(dev()), causal=True, stream=s)
    sa_check_status(s)
    O, L = oracle.attention(f64(q), f64(k), f64(v), 1 / 8.0, True)
    assert_close(o, lse, O, L, "fp16", "side stream")


@pytest.mark.parametrize("causal", [False, True])
def test_simple_kernel_parity(causal):
    run_fwd_case(1, 200, 300, 4, 2, 64, causal, "fp16", seed=16, simple=True)
    run_fwd_case(1, 130, 130, 2, 2, 128, causal, "bf16", seed=17, simple=True)
