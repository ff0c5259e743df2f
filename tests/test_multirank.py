"""Multi-rank host logic on CPU with two gloo ranks: max-over-ranks timing, per-rank
seeds and the weak-scaling aggregate (the GPU path exchanges no data between ranks)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from online_softmax_attention_sm_b200.dist import aggregate_throughput, max_over_ranks, rank_seed
from online_softmax_attention_sm_b200.inputs import make_qkv


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        t = max_over_ranks(1.5 + rank)                       # rank 1 is the slowest
        seed = rank_seed(123, rank)
        qq, _, _ = make_qkv(1, 4, 4, 2, 1, 64, "fp16", seed=seed)
        allq = [torch.empty_like(qq) for _ in range(world)]
        dist.all_gather(allq, qq)                            # test-only check of independence
        q.put((rank, t, seed, all(not torch.equal(allq[0], x) for x in allq[1:])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.5, 2.5]                 # both see the max
    assert res[0][2] == 123 and res[1][2] == 1123            # rank 0 keeps the base seed
    assert all(r[3] for r in res)                            # replicas draw different inputs


def test_single_process_is_identity():
    assert max_over_ranks(3.25) == 3.25
    assert aggregate_throughput(10.0, 4, 2.0) == 20.0
