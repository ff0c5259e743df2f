"""The attention workloads this library is measured and checked on.

Each workload is a plain description of shapes, dtype, masking and the input
recipe; it holds no attention arithmetic.  The shapes follow the forward
benchmarks of the flash-attn-volta page (section "Forward benchmark": (B,N,H,D)
tensors, fp16, causal and non-causal) and the GQA decode layout of the TurboQuant
"Attention API" page (compute_hybrid_attention: query (tokens, Hq, D), KV
(len, Hkv, D)), scaled up to the long-context sizes the StreamAttention page
targets (section "Distributed and Long-Context Variants").
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" or "decode"
    dtype: str           # "fp16" or "bf16"
    B: int
    Sq: int
    Sk: int
    Hq: int
    Hkv: int
    D: int
    causal: bool
    input_scale: float = 1.0      # Q, K, V ~ N(0,1) * input_scale
    k_sink_rows: int = 0          # K[:, :k_sink_rows] *= k_sink_factor
    k_sink_factor: float = 1.0
    seed: int = 20261202
    notes: str = ""

    @property
    def scale(self) -> float:
        # softmax scale 1/sqrt(D), the default of compute_hybrid_attention
        return 1.0 / math.sqrt(self.D)

    @property
    def lengths(self):
        """Packed variable-length workloads ("prefill_varlen": B sequences, Sq = Sk = the
        total tokens): the seeded sequence lengths; None otherwise."""
        if self.kind != "prefill_varlen":
            return None
        from .inputs import varlen_lengths
        return varlen_lengths(self.Sq, self.B, self.seed)

    @property
    def flops(self) -> float:
        """Forward FLOPs under the flash-attn-volta convention 4*B*H*Sq*Sk*D,
        halved for causal (summed over the sequences of a packed workload)."""
        if self.kind == "prefill_varlen":
            f = sum(4.0 * self.Hq * n * n * self.D for n in self.lengths)
        else:
            f = 4.0 * self.B * self.Hq * self.Sq * self.Sk * self.D
        return f / 2 if self.causal else f

    @property
    def kv_bytes(self) -> int:
        """Bytes of K plus V read once (the decode roofline's algorithmic bytes)."""
        return 2 * self.B * self.Sk * self.Hkv * self.D * 2


def block_sparse_flops(mask, Sq, Sk, D, causal, block=128):
    """Forward FLOPs of a block-sparse launch: 4*D per visible (row, key) pair, pairs
    counted per kept block of `mask` [..., ceil(Sq/block), ceil(Sk/block)] under the dense
    visibility rule (causal: key j <= row + Sk - Sq).  Unlike the dense causal convention
    (S*S/2), the diagonal blocks count exactly."""
    import numpy as np
    m = np.asarray(mask) != 0
    nq, nk = m.shape[-2], m.shape[-1]
    rows = np.arange(Sq)
    limit = np.clip(rows + Sk - Sq + 1, 0, Sk) if causal else np.full(Sq, Sk)
    per_block = np.zeros((nq, nk), dtype=np.int64)
    for ki in range(nk):
        c0 = ki * block
        width = min(block, Sk - c0)
        seen = np.clip(limit - c0, 0, width)                   # keys of this block each row sees
        per_block[:, ki] = np.add.reduceat(seen, np.arange(0, Sq, block))
    return 4.0 * D * float((m.reshape(-1, nq, nk).sum(axis=0) * per_block).sum())


WORKLOADS = {
    w.name: w
    for w in [
        Workload("mha_s128_d64_fp16", "prefill", "fp16", 1, 128, 128, 2, 2, 64, False,
                 seed=20261202 + 0, notes="smoke/parity size"),
        Workload("mha_causal_s2048_d64_fp16", "prefill", "fp16", 1, 2048, 2048, 16, 16, 64, True,
                 seed=20261202 + 1),
        Workload("mha_s4096_d128_bf16", "prefill", "bf16", 2, 4096, 4096, 8, 8, 128, False,
                 input_scale=0.5, seed=20261202 + 2),
        Workload("mha_causal_s4096_d128_bf16", "prefill", "bf16", 2, 4096, 4096, 8, 8, 128, True,
                 input_scale=0.5, seed=20261202 + 2),
        Workload("gqa_causal_s32768_d128_bf16_sinks", "prefill", "bf16", 1, 32768, 32768, 32, 8, 128,
                 True, k_sink_rows=4, k_sink_factor=8.0, seed=20261202 + 3),
        Workload("gqa_decode_sk32768_d64_fp16", "decode", "fp16", 4, 1, 32768, 14, 2, 64, False,
                 seed=20261202 + 4),
        # the long prefill's heads over 16 packed sequences of 32768 tokens in all
        Workload("gqa_causal_varlen16_t32768_d128_bf16", "prefill_varlen", "bf16", 16, 32768, 32768,
                 32, 8, 128, True, seed=20261202 + 6,
                 notes="packed sequences, lengths from inputs.varlen_lengths"),
    ]
}
