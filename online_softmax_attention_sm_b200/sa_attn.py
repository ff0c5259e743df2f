"""Python binding of the ``sa_attn`` C ABI (``include/sa_attn.h``).

Argument marshalling only: every step of the computation runs in the CUDA kernels of
``libsa_attn.so``.  torch is used for device memory and the current stream.  The
library must have been built (``online_softmax_attention_sm_b200.build``); if it is
missing, loading raises -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsa_attn.so")

SA_OK, SA_ERR_INVALID, SA_ERR_UNSUPPORTED, SA_ERR_CUDA, SA_ERR_TIMEOUT, SA_ERR_WORKSPACE = 0, -1, -2, -3, -4, -5
SA_FP16, SA_BF16 = 0, 1
_DT = {torch.float16: SA_FP16, torch.bfloat16: SA_BF16}

# exported symbol -> (restype, argtypes)
_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "sa_attn_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "sa_attn_fwd_simple": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "sa_attn_fwd_pair": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "sa_attn_fwd_varlen": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "sa_attn_fwd_block_sparse_workspace_size": (_Z, [_I, _I, _I, _I]),
    "sa_attn_bwd_workspace_size": (_Z, [_I, _I, _I]),
    "sa_attn_fwd_fp8": (_I, [_P] * 5 + [_I] * 7 + [_F, _F, _F, _F, _P]),
    "sa_attn_decode_single": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _P, _Z, _P]),
    "sa_attn_fwd_block_sparse_fp8": (_I, [_P] * 6 + [_I] * 7 + [_F, _F, _F, _F, _P, _Z, _P]),
    "sa_attn_fwd_paged": (_I, [_P] * 8 + [_I] * 10 + [_F, _I, _P]),
    "sa_attn_bwd": (_I, [_P] * 9 + [_I] * 7 + [_F, _I, _P, _Z, _P]),
    "sa_attn_fwd_block_sparse": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _Z, _P]),
    "sa_attn_decode_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "sa_attn_decode_num_splits": (_I, [_I, _I, _I, _I, _I]),
    "sa_attn_decode": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _P, _Z, _P]),
    "sa_attn_decode_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "sa_attn_decode_paged": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P, _Z, _P]),
    "sa_attn_decode_paged_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I, _I]),
    "sa_last_error": (ctypes.c_char_p, []),
    "sa_check_status": (_I, [_P]),
    "sa_version": (ctypes.c_char_p, []),
    "sa_selftest_bounded_wait": (_I, [_P]),
    "sa_diag_read_floor": (_I, [_P, _Z, _P, _I, _P]),
    "sa_diag_exp2_poly": (_I, [_P, _P, _I, _P]),
}

_lib = None


class SAError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"sa_attn error {code}: {msg}")
        self.code = code


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: build it with "
                              "`python -m online_softmax_attention_sm_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(rc):
    if rc != SA_OK:
        raise SAError(rc, lib().sa_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_tensor(name, t, dtype, device):
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_out(name, t, shape, dtype, device):
    """A caller-supplied output buffer: dtype, device, contiguity and exactly `shape` (the
    kernels write every element of that shape, so a smaller buffer would be overrun)."""
    _check_tensor(name, t, dtype, device)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _check_workspace(t, device):
    """Device scratch: on the inputs' device and contiguous (its size is checked by the
    library, which returns SA_ERR_WORKSPACE when it is short)."""
    if t.device != device:
        raise ValueError(f"workspace: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError("workspace must be contiguous")


def sa_attn_fwd(q, k, v, causal=False, scale=None, out=None, lse=None, return_lse=True,
                stream=None, simple=False, pair=False):
    """Attention forward.  q [B,Sq,Hq,D], k/v [B,Sk,Hkv,D] (fp16/bf16, CUDA, contiguous).
    Returns (o [B,Sq,Hq,D], lse [B,Hq,Sq] fp32 or None)."""
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if k.shape != (B, Sk, Hkv, D) or v.shape != k.shape:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    if q.dtype not in _DT:
        raise TypeError(f"unsupported dtype {q.dtype}")
    for n, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(n, t, q.dtype, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    _check_out("out", out, q.shape, q.dtype, q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _check_out("lse", lse, (B, Hq, Sq), torch.float32, q.device)
    fn = lib().sa_attn_fwd_simple if simple else lib().sa_attn_fwd_pair if pair else lib().sa_attn_fwd
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Sq, Sk, Hq, Hkv, D,
              int(bool(causal)), float(scale), _DT[q.dtype], _stream(stream)))
    return out, lse


def sa_attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal=False,
                       scale=None, out=None, lse=None, return_lse=True, stream=None):
    """Attention forward over sequences packed back to back.  q [total_q,Hq,D], k/v
    [total_k,Hkv,D] (fp16/bf16, CUDA, contiguous); cu_seqlens_q/k int32 [B+1] on the same
    device; max_seqlen_q/k host ints bounding every sequence's length.
    Returns (o [total_q,Hq,D], lse [Hq,total_q] fp32 or None)."""
    total_q, Hq, D = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    if k.shape != (total_k, Hkv, D) or v.shape != k.shape:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    if q.dtype not in _DT:
        raise TypeError(f"unsupported dtype {q.dtype}")
    for n, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(n, t, q.dtype, q.device)
    for n, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        _check_tensor(n, t, torch.int32, q.device)
    if cu_seqlens_q.dim() != 1 or cu_seqlens_q.shape != cu_seqlens_k.shape or cu_seqlens_q.numel() < 1:
        raise ValueError(f"cu_seqlens must both be [B+1], got {tuple(cu_seqlens_q.shape)} "
                         f"and {tuple(cu_seqlens_k.shape)}")
    B = cu_seqlens_q.numel() - 1
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    _check_out("out", out, q.shape, q.dtype, q.device)
    if return_lse and lse is None:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    if lse is not None:
        _check_out("lse", lse, (Hq, total_q), torch.float32, q.device)
    _check(lib().sa_attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens_q),
                                    _ptr(cu_seqlens_k), B, int(max_seqlen_q), int(max_seqlen_k), total_q,
                                    total_k, Hq, Hkv, D, int(bool(causal)), float(scale), _DT[q.dtype],
                                    _stream(stream)))
    return out, lse


def sa_attn_fwd_block_sparse_workspace_size(B, Sq, Sk, Hq):
    return int(lib().sa_attn_fwd_block_sparse_workspace_size(B, Sq, Sk, Hq))


def sa_attn_fwd_block_sparse(q, k, v, block_mask, causal=False, scale=None, workspace=None, out=None,
                             lse=None, return_lse=True, stream=None):
    """Block-sparse attention forward.  q [B,Sq,Hq,D], k/v [B,Sk,Hkv,D] (fp16/bf16, CUDA,
    contiguous); block_mask uint8 [B,Hq,ceil(Sq/128),ceil(Sk/128)] on the same device
    (nonzero = keep).  Returns (o [B,Sq,Hq,D], lse [B,Hq,Sq] fp32 or None)."""
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if k.shape != (B, Sk, Hkv, D) or v.shape != k.shape:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    if q.dtype not in _DT:
        raise TypeError(f"unsupported dtype {q.dtype}")
    for n, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(n, t, q.dtype, q.device)
    _check_tensor("block_mask", block_mask, torch.uint8, q.device)
    want = (B, Hq, -(-Sq // 128), -(-Sk // 128))
    if tuple(block_mask.shape) != want:
        raise ValueError(f"block_mask must be {want}, got {tuple(block_mask.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    _check_out("out", out, q.shape, q.dtype, q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _check_out("lse", lse, (B, Hq, Sq), torch.float32, q.device)
    need = sa_attn_fwd_block_sparse_workspace_size(B, Sq, Sk, Hq)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check_workspace(workspace, q.device)
    _check(lib().sa_attn_fwd_block_sparse(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(block_mask),
                                          B, Sq, Sk, Hq, Hkv, D, int(bool(causal)), float(scale), _DT[q.dtype],
                                          _ptr(workspace), workspace.numel() * workspace.element_size(),
                                          _stream(stream)))
    return out, lse


def sa_attn_fwd_fp8(q8, k8, v8, q_descale, k_descale, v_descale, causal=False, scale=None, out=None, lse=None,
                    return_lse=True, stream=None):
    """FP8 attention forward.  q8 [B,Sq,Hq,D], k8/v8 [B,Sk,Hkv,D]: uint8 tensors of e4m3 codes
    (CUDA, contiguous), per-tensor float descales.  Returns (o [B,Sq,Hq,D] bf16, lse [B,Hq,Sq])."""
    B, Sq, Hq, D = q8.shape
    Sk, Hkv = k8.shape[1], k8.shape[2]
    if k8.shape != (B, Sk, Hkv, D) or v8.shape != k8.shape:
        raise ValueError(f"shape mismatch q{tuple(q8.shape)} k{tuple(k8.shape)} v{tuple(v8.shape)}")
    for n, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        _check_tensor(n, t, torch.uint8, q8.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty((B, Sq, Hq, D), dtype=torch.bfloat16, device=q8.device)
    _check_out("out", out, (B, Sq, Hq, D), torch.bfloat16, q8.device)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q8.device)
    if lse is not None:
        _check_out("lse", lse, (B, Hq, Sq), torch.float32, q8.device)
    _check(lib().sa_attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(out), _ptr(lse), B, Sq, Sk, Hq, Hkv, D,
                                 int(bool(causal)), float(scale), float(q_descale), float(k_descale),
                                 float(v_descale), _stream(stream)))
    return out, lse


def sa_attn_fwd_block_sparse_fp8(q8, k8, v8, block_mask, q_descale, k_descale, v_descale, causal=False, scale=None,
                                 workspace=None, out=None, lse=None, return_lse=True, stream=None):
    """FP8 block-sparse forward: q8/k8/v8 uint8 e4m3 codes as in :func:`sa_attn_fwd_fp8`,
    block_mask as in :func:`sa_attn_fwd_block_sparse`.  Returns (o bf16, lse)."""
    B, Sq, Hq, D = q8.shape
    Sk, Hkv = k8.shape[1], k8.shape[2]
    if k8.shape != (B, Sk, Hkv, D) or v8.shape != k8.shape:
        raise ValueError(f"shape mismatch q{tuple(q8.shape)} k{tuple(k8.shape)} v{tuple(v8.shape)}")
    for n, t in (("q8", q8), ("k8", k8), ("v8", v8), ("block_mask", block_mask)):
        _check_tensor(n, t, torch.uint8, q8.device)
    want = (B, Hq, -(-Sq // 128), -(-Sk // 128))
    if tuple(block_mask.shape) != want:
        raise ValueError(f"block_mask must be {want}, got {tuple(block_mask.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty((B, Sq, Hq, D), dtype=torch.bfloat16, device=q8.device)
    _check_out("out", out, (B, Sq, Hq, D), torch.bfloat16, q8.device)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q8.device)
    if lse is not None:
        _check_out("lse", lse, (B, Hq, Sq), torch.float32, q8.device)
    need = sa_attn_fwd_block_sparse_workspace_size(B, Sq, Sk, Hq)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q8.device)
    _check_workspace(workspace, q8.device)
    _check(lib().sa_attn_fwd_block_sparse_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(out), _ptr(lse), _ptr(block_mask),
                                              B, Sq, Sk, Hq, Hkv, D, int(bool(causal)), float(scale),
                                              float(q_descale), float(k_descale), float(v_descale), _ptr(workspace),
                                              workspace.numel() * workspace.element_size(), _stream(stream)))
    return out, lse


def sa_attn_bwd_workspace_size(B, Sq, Hq):
    return int(lib().sa_attn_bwd_workspace_size(B, Sq, Hq))


def sa_attn_bwd(q, k, v, o, lse, dout, causal=False, scale=None, workspace=None, dq=None, dk=None, dv=None,
                stream=None):
    """Attention backward.  q/o/dout [B,Sq,Hq,D], k/v [B,Sk,Hkv,D] (fp16/bf16, CUDA, contiguous),
    lse [B,Hq,Sq] fp32 from the forward.  Returns (dq, dk, dv) shaped like q, k, v."""
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if k.shape != (B, Sk, Hkv, D) or v.shape != k.shape or o.shape != q.shape or dout.shape != q.shape:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)} "
                         f"o{tuple(o.shape)} dout{tuple(dout.shape)}")
    if q.dtype not in _DT:
        raise TypeError(f"unsupported dtype {q.dtype}")
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_tensor(n, t, q.dtype, q.device)
    _check_tensor("lse", lse, torch.float32, q.device)
    if lse.shape != (B, Hq, Sq):
        raise ValueError(f"lse must be [B, Hq, Sq], got {tuple(lse.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for n, t, like in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        _check_tensor(n, t, q.dtype, q.device)
        if t.shape != like.shape:
            raise ValueError(f"{n} must have shape {tuple(like.shape)}")
    need = sa_attn_bwd_workspace_size(B, Sq, Hq)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check_workspace(workspace, q.device)
    _check(lib().sa_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                             _ptr(dv), B, Sq, Sk, Hq, Hkv, D, int(bool(causal)), float(scale), _DT[q.dtype],
                             _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return dq, dk, dv


def sa_attn_fwd_paged(q, k_cache, v_cache, cu_seqlens_q, block_table, seqlens_k, max_seqlen_q, causal=False,
                      scale=None, out=None, lse=None, return_lse=True, stream=None):
    """Packed queries against a paged K/V cache.  q [total_q,Hq,D]; k_cache/v_cache
    [num_pages, page_size, Hkv, D]; cu_seqlens_q int32 [B+1]; block_table int32 [B, max_blocks];
    seqlens_k int32 [B] (all CUDA).  Returns (o [total_q,Hq,D], lse [Hq,total_q])."""
    total_q, Hq, D = q.shape
    num_pages, page_size, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (num_pages, page_size, Hkv, D) or v_cache.shape != k_cache.shape:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k_cache.shape)} v{tuple(v_cache.shape)}")
    if q.dtype not in _DT:
        raise TypeError(f"unsupported dtype {q.dtype}")
    for n, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _check_tensor(n, t, q.dtype, q.device)
    for n, t in (("cu_seqlens_q", cu_seqlens_q), ("block_table", block_table), ("seqlens_k", seqlens_k)):
        _check_tensor(n, t, torch.int32, q.device)
    B = cu_seqlens_q.numel() - 1
    if block_table.dim() != 2 or block_table.shape[0] != B or seqlens_k.shape != (B,):
        raise ValueError("block_table must be [B, max_blocks] and seqlens_k [B]")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    _check_out("out", out, q.shape, q.dtype, q.device)
    if lse is not None:
        _check_out("lse", lse, (Hq, total_q), torch.float32, q.device)
    _check(lib().sa_attn_fwd_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse), _ptr(cu_seqlens_q),
                                   _ptr(block_table), _ptr(seqlens_k), B, int(max_seqlen_q), total_q, Hq, Hkv, D,
                                   page_size, block_table.shape[1], num_pages, int(bool(causal)), float(scale),
                                   _DT[q.dtype], _stream(stream)))
    return out, lse


def sa_attn_fwd_pair(q, k, v, causal=False, scale=None, **kw):
    """The forward on the CTA-pair kernel whatever the shape (D = 128); as sa_attn_fwd."""
    return sa_attn_fwd(q, k, v, causal, scale, pair=True, **kw)


def sa_attn_fwd_simple(q, k, v, causal=False, scale=None, **kw):
    """The diagnostic CUDA-core forward (same contract as :func:`sa_attn_fwd`)."""
    return sa_attn_fwd(q, k, v, causal, scale, simple=True, **kw)


def sa_attn_decode_workspace_size(B, Sk, Hq, Hkv, D, num_splits=0):
    return int(lib().sa_attn_decode_workspace_size(B, Sk, Hq, Hkv, D, num_splits))


def sa_attn_decode_num_splits(B, Sk, Hq, Hkv, D):
    return int(lib().sa_attn_decode_num_splits(B, Sk, Hq, Hkv, D))


def sa_attn_decode(q, k, v, scale=None, num_splits=0, workspace=None, out=None, lse=None,
                   return_lse=True, stream=None, single=False):
    """Split-KV decode.  q [B,Hq,D], k/v [B,Sk,Hkv,D].  Returns (o [B,Hq,D], lse [B,Hq]).
    single=True runs the single-kernel variant (sa_attn_decode_single: the last split of
    each head tile merges, no combine launch)."""
    B, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    if k.shape != (B, Sk, Hkv, D) or v.shape != k.shape:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    if q.dtype not in _DT:
        raise TypeError(f"unsupported dtype {q.dtype}")
    for n, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(n, t, q.dtype, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _check_out("out", out, q.shape, q.dtype, q.device)
    if lse is not None:
        _check_out("lse", lse, (B, Hq), torch.float32, q.device)
    need = sa_attn_decode_workspace_size(B, Sk, Hq, Hkv, D, num_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check_workspace(workspace, q.device)
    fn = lib().sa_attn_decode_single if single else lib().sa_attn_decode
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Sk, Hq, Hkv, D, float(scale), _DT[q.dtype],
              int(num_splits), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return out, lse


def sa_attn_decode_single(q, k, v, **kw):
    """The single-kernel split-KV decode (same contract as :func:`sa_attn_decode`)."""
    return sa_attn_decode(q, k, v, single=True, **kw)


def sa_attn_decode_paged_workspace_size(B, Hq, Hkv, D, page_size, max_blocks, num_splits=0):
    return int(lib().sa_attn_decode_paged_workspace_size(B, Hq, Hkv, D, page_size, max_blocks, num_splits))


def sa_attn_decode_paged(q, k_cache, v_cache, block_table, seqlens, scale=None, num_splits=0,
                         workspace=None, out=None, lse=None, return_lse=True, stream=None):
    """Decode over a paged K/V cache.  q [B,Hq,D]; k_cache/v_cache [num_pages, page_size, Hkv, D];
    block_table [B, max_blocks] int32; seqlens [B] int32 (all CUDA, contiguous).
    Returns (o [B,Hq,D], lse [B,Hq])."""
    B, Hq, D = q.shape
    num_pages, page_size, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (num_pages, page_size, Hkv, D) or v_cache.shape != k_cache.shape:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k_cache.shape)} v{tuple(v_cache.shape)}")
    if q.dtype not in _DT:
        raise TypeError(f"unsupported dtype {q.dtype}")
    for n, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _check_tensor(n, t, q.dtype, q.device)
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError(f"block_table must be [B, max_blocks], got {tuple(block_table.shape)}")
    _check_tensor("block_table", block_table, torch.int32, q.device)
    _check_tensor("seqlens", seqlens, torch.int32, q.device)
    if seqlens.shape != (B,):
        raise ValueError(f"seqlens must be [B], got {tuple(seqlens.shape)}")
    max_blocks = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _check_out("out", out, q.shape, q.dtype, q.device)
    if lse is not None:
        _check_out("lse", lse, (B, Hq), torch.float32, q.device)
    need = sa_attn_decode_paged_workspace_size(B, Hq, Hkv, D, page_size, max_blocks, num_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check_workspace(workspace, q.device)
    _check(lib().sa_attn_decode_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seqlens),
                                      _ptr(out), _ptr(lse), B, Hq, Hkv, D, page_size, max_blocks, num_pages,
                                      float(scale), _DT[q.dtype], int(num_splits), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream)))
    return out, lse


def sa_diag_read_floor(buf, sink, mode=0, stream=None):
    """Diagnostic: read every byte of the contiguous CUDA tensor `buf` once (no attention
    arithmetic), folding it into the int32 CUDA tensor `sink` (one element).  mode 0:
    128-bit loads; mode 1: bulk copies into a shared-memory ring (the decode's way)."""
    if not buf.is_contiguous():
        raise ValueError("buf must be contiguous")
    if sink.dtype != torch.int32 or sink.device != buf.device or sink.numel() < 1:
        raise ValueError("sink must be an int32 tensor on buf's device")
    _check(lib().sa_diag_read_floor(_ptr(buf), buf.numel() * buf.element_size(), _ptr(sink), int(mode),
                                    _stream(stream)))


def sa_diag_exp2_poly(x, out=None, stream=None):
    """Diagnostic: 2^x by the forward kernel's FMA-pipe exponential (x: float32 CUDA tensor)."""
    _check_tensor("x", x, torch.float32, x.device)
    if out is None:
        out = torch.empty_like(x)
    _check_out("out", out, x.shape, torch.float32, x.device)
    _check(lib().sa_diag_exp2_poly(_ptr(x), _ptr(out), x.numel(), _stream(stream)))
    return out


def sa_check_status(stream=None):
    """Synchronise the stream and raise if a bounded device wait expired."""
    _check(lib().sa_check_status(_stream(stream)))


def sa_version():
    return lib().sa_version().decode()
