"""Forward launches that take their work units from the library's shared counter pairs (the
dynamic instance: every packed-sequence forward), many in flight at once on several streams:
each must give exactly the result of a launch run alone.  More launches than a 64-pair pool
would hold, fewer than the library's 1024 pairs, so a launch that picked up a pair still in
use -- units skipped or run twice -- would show as a wrong output."""
import numpy as np
import pytest
import torch

from online_softmax_attention_sm_b200 import sa_attn_fwd_varlen, sa_check_status
from online_softmax_attention_sm_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu


def test_many_dynamic_forwards_on_many_streams_match_a_lone_launch():
    dev = torch.device("cuda:0")
    lens = [700, 129, 1500, 257, 1024]
    total = sum(lens)
    q, k, v = (t[0].to(dev) for t in make_qkv(1, total, total, 8, 2, 64, "bf16", seed=31))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
    ref_o, ref_l = sa_attn_fwd_varlen(q, k, v, cu, cu, max(lens), max(lens), causal=True)
    sa_check_status()
    n_launch, n_stream = 200, 8
    streams = [torch.cuda.Stream(dev) for _ in range(n_stream)]
    outs = [(torch.full_like(q, 9.0), torch.full_like(ref_l, 9.0)) for _ in range(n_launch)]
    torch.cuda.synchronize(dev)
    for i, (o, l) in enumerate(outs):
        s = streams[i % n_stream]
        with torch.cuda.stream(s):
            sa_attn_fwd_varlen(q, k, v, cu, cu, max(lens), max(lens), causal=True, out=o, lse=l, stream=s)
    torch.cuda.synchronize(dev)
    sa_check_status()
    bad = [i for i, (o, l) in enumerate(outs) if not (torch.equal(o, ref_o) and torch.equal(l, ref_l))]
    assert not bad, f"{len(bad)} of {n_launch} launches differ from the lone launch (first: {bad[:5]})"
