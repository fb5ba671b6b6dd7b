"""Token-DP exchange on CPU: two gloo ranks, each routing half of a batch with the
oracle, sum their count histograms through the package's exchange step, and
apply Eq. (2); the result equals the single-process update on the whole batch."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_30_b200 import dist as MD
from oracle import moe_oracle as orc

T, d, N, Z, K = 96, 16, 6, 3, 3
E = N + Z


def _batch():
    rng = np.random.default_rng(0)
    return rng.normal(size=(T, d)), rng.normal(size=(E, d)), rng.uniform(-0.05, 0.05, E)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, wr, b = _batch()
        shard = x[rank * T // world:(rank + 1) * T // world]
        idx, _ = orc.biased_topk(orc.softmax_rows(orc.router_logits(shard, wr)), b, K)
        local = torch.from_numpy(orc.expert_counts(idx, E).astype(np.int32))
        glob = MD.global_counts(local, torch.empty_like(local))
        T_all = MD.global_tokens(shard.shape[0])
        b1 = orc.bias_update(b, glob.numpy(), N, K, K * N / E, 0.1, T_all)
        q.put((rank, glob.numpy().tolist(), T_all, b1.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_rank_count_allreduce_matches_single_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, wr, b = _batch()
    idx, _ = orc.biased_topk(orc.softmax_rows(orc.router_logits(x, wr)), b, K)
    counts = orc.expert_counts(idx, E)
    want = orc.bias_update(b, counts, N, K, K * N / E, 0.1, T)
    for rank, glob, T_all, b1 in res:
        assert glob == counts.tolist() and T_all == T
        assert np.array_equal(np.array(b1), want)


def test_single_process_is_identity():
    c = torch.arange(E, dtype=torch.int32)
    assert torch.equal(MD.global_counts(c, torch.empty_like(c)), c)
    assert MD.global_tokens(17) == 17
