"""C-ABI checks that need no GPU: the library loads, exports every symbol the header
declares, and rejects invalid arguments on the host before any device work."""
import ctypes
import math
import os
import re

import pytest

from online_softmax_attention_sm_b200 import build as build_mod
from online_softmax_attention_sm_b200 import sa_attn as sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sa_attn.h")


@pytest.fixture(scope="module")
def L():
    build_mod.build()
    return sa.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = header_functions()
    for n in ("sa_attn_fwd", "sa_attn_decode", "sa_attn_decode_workspace_size", "sa_last_error",
              "sa_check_status"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in header_functions():
        assert hasattr(L, n), f"{n} declared in sa_attn.h but not exported"
        assert n in sa.SIGNATURES, f"{n} has no binding signature"


def test_binding_names_match_header():
    assert set(sa.SIGNATURES) == set(header_functions())


NULL = None
FAKE = ctypes.c_void_p(1 << 20)          # 16-byte aligned, never dereferenced: checks fail first


def fwd(L, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=NULL, B=1, Sq=8, Sk=8, Hq=2, Hkv=2, D=64, causal=0,
        scale=0.125, dtype=0):
    return L.sa_attn_fwd(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, D, causal, scale, dtype, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=NULL), sa.SA_ERR_INVALID),
    (dict(o=NULL), sa.SA_ERR_INVALID),
    (dict(k=NULL), sa.SA_ERR_INVALID),
    (dict(B=-1), sa.SA_ERR_INVALID),
    (dict(Sk=-3), sa.SA_ERR_INVALID),
    (dict(Hq=3, Hkv=2), sa.SA_ERR_INVALID),
    (dict(Hq=2, Hkv=0), sa.SA_ERR_INVALID),
    (dict(D=96), sa.SA_ERR_UNSUPPORTED),
    (dict(D=256), sa.SA_ERR_UNSUPPORTED),
    (dict(dtype=7), sa.SA_ERR_UNSUPPORTED),
    (dict(scale=math.nan), sa.SA_ERR_INVALID),
    (dict(scale=math.inf), sa.SA_ERR_INVALID),
    (dict(causal=2), sa.SA_ERR_INVALID),
    (dict(q=ctypes.c_void_p((1 << 20) + 8)), sa.SA_ERR_INVALID),
    (dict(lse=ctypes.c_void_p((1 << 20) + 4)), sa.SA_ERR_INVALID),
])
def test_fwd_rejects_invalid_arguments(L, kw, code):
    assert fwd(L, **kw) == code
    assert L.sa_last_error().decode() != ""
    assert L.sa_attn_fwd_simple(*[kw.get(n, d) for n, d in
                                  (("q", FAKE), ("k", FAKE), ("v", FAKE), ("o", FAKE), ("lse", NULL))],
                                kw.get("B", 1), kw.get("Sq", 8), kw.get("Sk", 8), kw.get("Hq", 2),
                                kw.get("Hkv", 2), kw.get("D", 64), kw.get("causal", 0),
                                kw.get("scale", 0.125), kw.get("dtype", 0), None) == code


@pytest.mark.parametrize("kw", [dict(B=0), dict(Sq=0), dict(Hq=0, Hkv=0), dict(Hq=0, Hkv=2)])
def test_fwd_empty_problem_is_a_no_op(L, kw):
    # nothing is launched, so null pointers are fine
    assert fwd(L, q=NULL, k=NULL, v=NULL, o=NULL, **kw) == sa.SA_OK


def dec(L, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=NULL, B=1, Sk=64, Hq=2, Hkv=1, D=64, scale=0.125,
        dtype=0, ns=0, ws=FAKE, wsb=1 << 30):
    return L.sa_attn_decode(q, k, v, o, lse, B, Sk, Hq, Hkv, D, scale, dtype, ns, ws, wsb, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=NULL), sa.SA_ERR_INVALID),
    (dict(Hq=3, Hkv=2), sa.SA_ERR_INVALID),
    (dict(D=32), sa.SA_ERR_UNSUPPORTED),
    (dict(dtype=2), sa.SA_ERR_UNSUPPORTED),
    (dict(ns=-1), sa.SA_ERR_INVALID),
    (dict(scale=math.nan), sa.SA_ERR_INVALID),
    (dict(ws=NULL), sa.SA_ERR_WORKSPACE),
    (dict(wsb=16), sa.SA_ERR_WORKSPACE),
    (dict(ws=ctypes.c_void_p((1 << 20) + 4)), sa.SA_ERR_INVALID),
])
def test_decode_rejects_invalid_arguments(L, kw, code):
    assert dec(L, **kw) == code


def test_decode_empty_is_a_no_op(L):
    assert dec(L, q=NULL, k=NULL, v=NULL, o=NULL, B=0) == sa.SA_OK


def test_workspace_size(L):
    # (D + 4) floats per (b, h, split)
    assert L.sa_attn_decode_workspace_size(4, 32768, 14, 2, 64, 1) == 4 * 14 * 1 * 68 * 4
    assert L.sa_attn_decode_workspace_size(4, 32768, 14, 2, 64, 8) == 4 * 14 * 8 * 68 * 4
    # clamped to ceil(Sk / 64) splits, and to 192 (D = 64) / 96 (D = 128)
    assert L.sa_attn_decode_workspace_size(1, 100, 2, 1, 128, 50) == 1 * 2 * 2 * 132 * 4
    def splits(Sk, cap):                      # chunk = ceil(Sk / cap) rounded up to 64 tokens
        chunk = -(-(-(-Sk // cap)) // 64) * 64
        return -(-Sk // chunk)
    assert L.sa_attn_decode_workspace_size(1, 1 << 20, 2, 1, 64, 5000) == 1 * 2 * splits(1 << 20, 192) * 68 * 4
    assert L.sa_attn_decode_workspace_size(1, 1 << 20, 2, 1, 128, 5000) == 1 * 2 * splits(1 << 20, 96) * 132 * 4
    assert splits(1 << 20, 192) <= 192 and splits(1 << 20, 96) <= 96
    assert L.sa_attn_decode_workspace_size(1, 100, 3, 2, 64, 1) == 0      # invalid GQA
    assert L.sa_attn_decode_workspace_size(0, 100, 2, 2, 64, 1) == 0      # empty
    assert L.sa_attn_decode_num_splits(1, 100, 3, 2, 64) == 0
    assert L.sa_attn_decode_num_splits(4, 32768, 14, 2, 64) >= 1


def dec_paged(L, q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, sl=FAKE, o=FAKE, lse=NULL, B=1, Hq=2, Hkv=1, D=64,
              page=64, mb=4, npg=8, scale=0.125, dtype=0, ns=0, ws=FAKE, wsb=1 << 30):
    return L.sa_attn_decode_paged(q, kc, vc, bt, sl, o, lse, B, Hq, Hkv, D, page, mb, npg, scale, dtype, ns,
                                  ws, wsb, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=NULL), sa.SA_ERR_INVALID),
    (dict(bt=NULL), sa.SA_ERR_INVALID),
    (dict(sl=NULL), sa.SA_ERR_INVALID),
    (dict(Hq=3, Hkv=2), sa.SA_ERR_INVALID),
    (dict(D=96), sa.SA_ERR_UNSUPPORTED),
    (dict(page=32), sa.SA_ERR_UNSUPPORTED),
    (dict(page=100), sa.SA_ERR_UNSUPPORTED),
    (dict(mb=0), sa.SA_ERR_INVALID),
    (dict(npg=0), sa.SA_ERR_INVALID),
    (dict(ns=-2), sa.SA_ERR_INVALID),
    (dict(ws=NULL), sa.SA_ERR_WORKSPACE),
    (dict(wsb=16), sa.SA_ERR_WORKSPACE),
    # 192 splits of at most 16384 tokens hold 3145728 tokens (D = 64)
    (dict(page=64, mb=3145728 // 64 + 1), sa.SA_ERR_UNSUPPORTED),
])
def test_paged_decode_rejects_invalid_arguments(L, kw, code):
    assert dec_paged(L, **kw) == code


def test_paged_decode_empty_is_a_no_op(L):
    assert dec_paged(L, q=NULL, kc=NULL, vc=NULL, bt=NULL, sl=NULL, o=NULL, B=0) == sa.SA_OK


def test_paged_workspace_size(L):
    # planned for page_size * max_blocks tokens, like the dense decode of that length ...
    assert (L.sa_attn_decode_paged_workspace_size(4, 14, 2, 64, 64, 512, 0)
            == L.sa_attn_decode_workspace_size(4, 32768, 14, 2, 64, 0))
    assert L.sa_attn_decode_paged_workspace_size(2, 8, 8, 128, 128, 10, 3) == 2 * 8 * 3 * 132 * 4
    # ... but a split takes at most 16384 tokens: one requested split becomes two
    assert L.sa_attn_decode_paged_workspace_size(1, 2, 1, 64, 64, 512, 1) == 1 * 2 * 2 * 68 * 4
    assert L.sa_attn_decode_paged_workspace_size(1, 2, 1, 64, 32, 512, 1) == 0      # bad page size
    assert L.sa_attn_decode_paged_workspace_size(0, 2, 1, 64, 64, 512, 1) == 0      # empty


def fwd_varlen(L, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=NULL, cq=FAKE, ck=FAKE, B=2, mq=64, mk=64, tq=100,
               tk=100, Hq=2, Hkv=1, D=64, causal=1, scale=0.125, dtype=1):
    return L.sa_attn_fwd_varlen(q, k, v, o, lse, cq, ck, B, mq, mk, tq, tk, Hq, Hkv, D, causal, scale, dtype,
                                None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=NULL), sa.SA_ERR_INVALID),
    (dict(o=NULL), sa.SA_ERR_INVALID),
    (dict(cq=NULL), sa.SA_ERR_INVALID),
    (dict(ck=NULL), sa.SA_ERR_INVALID),
    (dict(cq=ctypes.c_void_p((1 << 20) + 2)), sa.SA_ERR_INVALID),
    (dict(B=-1), sa.SA_ERR_INVALID),
    (dict(tq=-5), sa.SA_ERR_INVALID),
    (dict(mq=-1), sa.SA_ERR_INVALID),
    (dict(mk=-1), sa.SA_ERR_INVALID),
    (dict(Hq=3, Hkv=2), sa.SA_ERR_INVALID),
    (dict(D=96), sa.SA_ERR_UNSUPPORTED),
    (dict(dtype=5), sa.SA_ERR_UNSUPPORTED),
    (dict(causal=3), sa.SA_ERR_INVALID),
    (dict(scale=math.nan), sa.SA_ERR_INVALID),
    (dict(k=ctypes.c_void_p((1 << 20) + 8)), sa.SA_ERR_INVALID),
])
def test_fwd_varlen_rejects_invalid_arguments(L, kw, code):
    assert fwd_varlen(L, **kw) == code


@pytest.mark.parametrize("kw", [dict(B=0), dict(tq=0), dict(Hq=0, Hkv=0), dict(mq=0)])
def test_fwd_varlen_empty_problem_is_a_no_op(L, kw):
    args = dict(q=NULL, k=NULL, v=NULL, o=NULL, cq=NULL, ck=NULL)
    args.update(kw)
    assert fwd_varlen(L, **args) == sa.SA_OK


def fwd_sparse(L, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=NULL, m=FAKE, B=1, Sq=256, Sk=256, Hq=2, Hkv=1, D=64,
               causal=1, scale=0.125, dtype=0, ws=FAKE, wsb=1 << 20):
    return L.sa_attn_fwd_block_sparse(q, k, v, o, lse, m, B, Sq, Sk, Hq, Hkv, D, causal, scale, dtype, ws, wsb,
                                      None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=NULL), sa.SA_ERR_INVALID),
    (dict(m=NULL), sa.SA_ERR_INVALID),
    (dict(Hq=3, Hkv=2), sa.SA_ERR_INVALID),
    (dict(D=80), sa.SA_ERR_UNSUPPORTED),
    (dict(causal=2), sa.SA_ERR_INVALID),
    (dict(scale=math.inf), sa.SA_ERR_INVALID),
    (dict(ws=NULL), sa.SA_ERR_WORKSPACE),
    (dict(wsb=32), sa.SA_ERR_WORKSPACE),
    (dict(ws=ctypes.c_void_p((1 << 20) + 8)), sa.SA_ERR_INVALID),
    (dict(Sk=131072 + 1), sa.SA_ERR_UNSUPPORTED),
])
def test_fwd_block_sparse_rejects_invalid_arguments(L, kw, code):
    assert fwd_sparse(L, **kw) == code


def test_fwd_block_sparse_empty_is_a_no_op(L):
    assert fwd_sparse(L, q=NULL, k=NULL, v=NULL, o=NULL, m=NULL, ws=NULL, B=0) == sa.SA_OK


def test_block_sparse_workspace_size(L):
    # one record per (batch, head, 256-row query block): 8 header slots + the longest list,
    # rounded up to 16 bytes, in uint16
    assert L.sa_attn_fwd_block_sparse_workspace_size(1, 256, 256, 2) == 2 * (8 + 8) * 2
    assert L.sa_attn_fwd_block_sparse_workspace_size(2, 32768, 32768, 32) == 2 * 32 * 128 * (8 + 256) * 2
    assert L.sa_attn_fwd_block_sparse_workspace_size(1, 300, 1300, 3) == 3 * 2 * (8 + 16) * 2
    assert L.sa_attn_fwd_block_sparse_workspace_size(1, 256, 131072 + 1, 2) == 0
    assert L.sa_attn_fwd_block_sparse_workspace_size(0, 256, 256, 2) == 0


def bwd(L, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, do=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, B=1, Sq=128, Sk=128, Hq=2,
        Hkv=1, D=64, causal=1, scale=0.125, dtype=1, ws=FAKE, wsb=1 << 20):
    return L.sa_attn_bwd(q, k, v, o, lse, do, dq, dk, dv, B, Sq, Sk, Hq, Hkv, D, causal, scale, dtype, ws, wsb,
                         None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=NULL), sa.SA_ERR_INVALID),
    (dict(lse=NULL), sa.SA_ERR_INVALID),
    (dict(do=NULL), sa.SA_ERR_INVALID),
    (dict(dk=NULL), sa.SA_ERR_INVALID),
    (dict(Hq=3, Hkv=2), sa.SA_ERR_INVALID),
    (dict(D=96), sa.SA_ERR_UNSUPPORTED),
    (dict(causal=4), sa.SA_ERR_INVALID),
    (dict(scale=math.nan), sa.SA_ERR_INVALID),
    (dict(dv=ctypes.c_void_p((1 << 20) + 4)), sa.SA_ERR_INVALID),
    (dict(ws=NULL), sa.SA_ERR_WORKSPACE),
    (dict(wsb=64), sa.SA_ERR_WORKSPACE),
])
def test_bwd_rejects_invalid_arguments(L, kw, code):
    assert bwd(L, **kw) == code


def test_bwd_empty_is_a_no_op(L):
    assert bwd(L, q=NULL, k=NULL, v=NULL, o=NULL, lse=NULL, do=NULL, dq=NULL, dk=NULL, dv=NULL, ws=NULL, B=0) == sa.SA_OK


def test_bwd_workspace_size(L):
    # two fp32 rows (lse2, Delta) per (batch, query head), padded to 128 queries
    assert L.sa_attn_bwd_workspace_size(1, 300, 4) == 2 * 4 * 384 * 4
    assert L.sa_attn_bwd_workspace_size(2, 32768, 32) == 2 * 2 * 32 * 32768 * 4
    assert L.sa_attn_bwd_workspace_size(0, 300, 4) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(q=NULL), sa.SA_ERR_INVALID),
    (dict(Hq=3, Hkv=2), sa.SA_ERR_INVALID),
    (dict(D=96), sa.SA_ERR_UNSUPPORTED),
    (dict(ns=-1), sa.SA_ERR_INVALID),
    (dict(ws=NULL), sa.SA_ERR_WORKSPACE),
])
def test_decode_single_rejects_invalid_arguments(L, kw, code):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=NULL, B=1, Sk=64, Hq=2, Hkv=1, D=64, scale=0.125, dtype=0, ns=0,
                ws=FAKE, wsb=1 << 20)
    args.update(kw)
    a = args
    assert L.sa_attn_decode_single(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Sk"], a["Hq"], a["Hkv"],
                                   a["D"], a["scale"], a["dtype"], a["ns"], a["ws"], a["wsb"], None) == code


@pytest.mark.parametrize("kw,code", [
    (dict(q=NULL), sa.SA_ERR_INVALID),
    (dict(bt=NULL), sa.SA_ERR_INVALID),
    (dict(page=64), sa.SA_ERR_UNSUPPORTED),
    (dict(page=200), sa.SA_ERR_UNSUPPORTED),
    (dict(mb=0), sa.SA_ERR_INVALID),
    (dict(npg=0), sa.SA_ERR_INVALID),
    (dict(Hq=3, Hkv=2), sa.SA_ERR_INVALID),
    (dict(causal=7), sa.SA_ERR_INVALID),
])
def test_fwd_paged_rejects_invalid_arguments(L, kw, code):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, o=FAKE, lse=NULL, cq=FAKE, bt=FAKE, sk=FAKE, B=2, mq=64, tq=100, Hq=2, Hkv=1,
             D=64, page=128, mb=4, npg=8, causal=1, scale=0.125, dtype=0)
    a.update(kw)
    assert L.sa_attn_fwd_paged(a["q"], a["kc"], a["vc"], a["o"], a["lse"], a["cq"], a["bt"], a["sk"], a["B"], a["mq"],
                               a["tq"], a["Hq"], a["Hkv"], a["D"], a["page"], a["mb"], a["npg"], a["causal"],
                               a["scale"], a["dtype"], None) == code


def test_version(L):
    assert re.fullmatch(r"\d+\.\d+\.\d+", sa.sa_version())


def test_library_has_no_cpu_path():
    # the package exposes no host-side compute: every entry point goes through the C ABI
    import online_softmax_attention_sm_b200 as pkg
    src = open(os.path.join(os.path.dirname(pkg.__file__), "sa_attn.py")).read()
    assert "oracle" not in src and "scaled_dot_product" not in src and "softmax(" not in src


def test_binding_rejects_wrong_output_and_workspace_buffers(L):
    # a caller's out / lse of the wrong shape, or a workspace on another device, raises in the
    # binding before anything is launched (host tensors: nothing here reaches a kernel)
    import torch
    f16, u8 = torch.float16, torch.uint8
    q, k = torch.zeros(1, 8, 2, 64, dtype=f16), torch.zeros(1, 8, 1, 64, dtype=f16)
    with pytest.raises(ValueError, match="out must have shape"):
        sa.sa_attn_fwd(q, k, k, out=torch.empty(1, 7, 2, 64, dtype=f16))
    with pytest.raises(ValueError, match="lse must have shape"):
        sa.sa_attn_fwd(q, k, k, lse=torch.empty(1, 2, 7))
    mask = torch.ones(1, 2, 1, 1, dtype=u8)
    with pytest.raises(ValueError, match="lse must have shape"):
        sa.sa_attn_fwd_block_sparse(q, k, k, mask, lse=torch.empty(2, 8))
    with pytest.raises(ValueError, match="workspace: on meta"):
        sa.sa_attn_fwd_block_sparse(q, k, k, mask, workspace=torch.empty(4096, dtype=u8, device="meta"))
    qp, kp = torch.zeros(10, 2, 64, dtype=f16), torch.zeros(10, 1, 64, dtype=f16)
    cu = torch.tensor([0, 10], dtype=torch.int32)
    with pytest.raises(ValueError, match="lse must have shape"):
        sa.sa_attn_fwd_varlen(qp, kp, kp, cu, cu, 10, 10, lse=torch.empty(1, 2, 10))
    kc = torch.zeros(2, 128, 1, 64, dtype=f16)
    table, seqk = torch.zeros(1, 2, dtype=torch.int32), torch.tensor([10], dtype=torch.int32)
    with pytest.raises(ValueError, match="out must have shape"):
        sa.sa_attn_fwd_paged(qp, kc, kc, cu, table, seqk, 10, out=torch.empty(9, 2, 64, dtype=f16))
    q8, k8 = torch.zeros(1, 8, 2, 128, dtype=u8), torch.zeros(1, 8, 1, 128, dtype=u8)
    with pytest.raises(ValueError, match="out must have shape"):
        sa.sa_attn_fwd_fp8(q8, k8, k8, 1.0, 1.0, 1.0, out=torch.empty(1, 8, 2, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="lse must have shape"):
        sa.sa_attn_fwd_block_sparse_fp8(q8, k8, k8, mask, 1.0, 1.0, 1.0, lse=torch.empty(1, 2, 9))
    o, lse = torch.zeros_like(q), torch.zeros(1, 2, 8)
    with pytest.raises(ValueError, match="workspace: on meta"):
        sa.sa_attn_bwd(q, k, k, o, lse, o, workspace=torch.empty(4096, dtype=u8, device="meta"))
    qd, kd = torch.zeros(2, 2, 64, dtype=f16), torch.zeros(2, 64, 1, 64, dtype=f16)
    with pytest.raises(ValueError, match="out must have shape"):
        sa.sa_attn_decode(qd, kd, kd, out=torch.empty(2, 2, 32, dtype=f16))
    with pytest.raises(ValueError, match="lse must have shape"):
        sa.sa_attn_decode(qd, kd, kd, lse=torch.empty(2, 3))
    with pytest.raises(ValueError, match="workspace: on meta"):
        sa.sa_attn_decode(qd, kd, kd, workspace=torch.empty(1 << 16, dtype=u8, device="meta"))
    table2, seq2 = torch.zeros(2, 1, dtype=torch.int32), torch.tensor([10, 10], dtype=torch.int32)
    with pytest.raises(ValueError, match="lse must have shape"):
        sa.sa_attn_decode_paged(qd, kc, kc, table2, seq2, lse=torch.empty(2))
