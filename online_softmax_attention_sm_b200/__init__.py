"""B200 (sm_100a) fused online-softmax attention: prefill forward (dense, packed, paged,
block-sparse, FP8), backward, and split-KV decode (dense, paged, single-launch).

The computation runs in hand-written CUDA kernels behind the C ABI of
``include/sa_attn.h`` (``libsa_attn.so``); :mod:`.sa_attn` is its Python binding.
"""
from .sa_attn import (sa_attn_fwd, sa_attn_fwd_simple, sa_attn_fwd_pair, sa_attn_fwd_varlen, sa_attn_fwd_paged, sa_attn_fwd_block_sparse,
                      sa_attn_fwd_block_sparse_workspace_size, sa_attn_fwd_fp8, sa_attn_fwd_block_sparse_fp8, sa_attn_bwd,
                      sa_attn_bwd_workspace_size,
                      sa_attn_decode, sa_attn_decode_single,
                      sa_attn_decode_workspace_size, sa_attn_decode_num_splits,
                      sa_attn_decode_paged, sa_attn_decode_paged_workspace_size,
                      sa_diag_read_floor, sa_diag_exp2_poly,
                      sa_check_status, sa_version, SAError, lib)

__all__ = ["sa_attn_fwd", "sa_attn_fwd_simple", "sa_attn_fwd_pair", "sa_attn_fwd_varlen", "sa_attn_fwd_paged", "sa_attn_fwd_block_sparse",
           "sa_attn_fwd_block_sparse_workspace_size", "sa_attn_fwd_fp8", "sa_attn_fwd_block_sparse_fp8", "sa_attn_bwd", "sa_attn_bwd_workspace_size",
           "sa_attn_decode", "sa_attn_decode_single", "sa_attn_decode_workspace_size",
           "sa_attn_decode_num_splits", "sa_attn_decode_paged", "sa_attn_decode_paged_workspace_size",
           "sa_diag_read_floor", "sa_diag_exp2_poly", "sa_check_status", "sa_version", "SAError", "lib"]
