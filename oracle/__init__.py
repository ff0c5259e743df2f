"""fp64 CPU oracle for the fused online-softmax attention forward.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (CPU baseline and ``--impl reference``), never by the library.
It shares no code with the CUDA path.  Every function here is pinned by
``tests/test_oracle.py`` to closed forms, invariants and brute force; none is
"parity unpinned".  ``tests/test_oracle_mutants.py`` checks those pins in turn: copies of
this code with one planted mistake each must fail at least one of them.
"""
from .attention import (attention, attention_rows, attention_blockwise, attention_varlen, attention_paged_prefill,
                        attention_block_sparse, attention_block_sparse_rows, block_sparse_pairs,
                        attention_backward, attention_backward_rows, attention_backward_keys, decode_e4m3,
                        attention_fp8, decode, decode_paged, combine_lse)

__all__ = ["attention", "attention_rows", "attention_blockwise", "attention_varlen", "attention_paged_prefill",
           "attention_block_sparse", "attention_block_sparse_rows", "block_sparse_pairs",
           "attention_backward", "attention_backward_rows", "attention_backward_keys", "decode_e4m3",
           "attention_fp8", "decode", "decode_paged", "combine_lse"]
