"""The multi-rank plumbing of bench.py on CPU (gloo), without a GPU.

Two ranks run the exchange path the benchmark uses -- per-rank activations
(rank_x_seed), T_all = T * world (global_tokens), the count all-reduce
(global_counts) and the maximum of the step times (max_over_ranks) -- with the
routing done by the oracle.  Both ranks must end with the same counts and the
same Eq. (2) bias as one process that routes the two batches together.  The
rank launcher behind `bench.py --gpus N` is checked with a tiny child command.
"""
import os
import subprocess
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_30_b200 import configs as C
from mixture_experts_layer_30_b200 import dist as MD
from mixture_experts_layer_30_b200 import inputs as IN
from oracle import moe_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CFG = C.TINY_F32


def _rank_x(rank):
    L = IN.make_layer_inputs(CFG, device="cpu")
    seed = MD.rank_x_seed(rank)
    if seed is not None:
        L["x"] = IN.make_x(CFG, "cpu", seed=seed)
    return L


def _route_counts(L):
    probs = orc.softmax_rows(orc.router_logits(L["x"].numpy(), L["w_router"].numpy()))
    idx, _ = orc.biased_topk(probs, L["bias"].numpy(), CFG.K)
    return orc.expert_counts(idx, CFG.E).astype(np.int32)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L = _rank_x(rank)
        local = torch.from_numpy(_route_counts(L))
        glob = MD.global_counts(local, torch.empty_like(local))
        T_all = MD.global_tokens(CFG.T)
        b1 = orc.bias_update(L["bias"].numpy(), glob.numpy(), CFG.N, CFG.K, CFG.K_e, CFG.mu,
                             T_all)
        ms = MD.max_over_ranks(1.5 + rank, "cpu")
        q.put((rank, float(L["x"].sum()), glob.tolist(), T_all, b1.tolist(), ms))
    finally:
        dist.destroy_process_group()


def test_bench_exchange_path_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = MD.free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, xs0, g0, T0, b0, m0), (_, xs1, g1, T1, b1, m1) = res
    assert xs0 != xs1                      # each rank routes its own batch
    assert T0 == T1 == 2 * CFG.T           # T_all of Eq. (2) is the global batch
    want = _route_counts(_rank_x(0)) + _route_counts(_rank_x(1))
    assert g0 == g1 == want.tolist()       # counts summed over ranks
    L0 = _rank_x(0)
    b_want = orc.bias_update(L0["bias"].numpy(), want, CFG.N, CFG.K, CFG.K_e, CFG.mu,
                             2 * CFG.T)
    assert b0 == b1 == b_want.tolist()     # the same bias on every rank
    assert m0 == m1 == 2.5                 # step time: the slowest rank


def test_launch_ranks_sets_the_torchrun_environment(tmp_path):
    code = ("import os, sys; p = sys.argv[1]; r = os.environ['RANK']; "
            "open(os.path.join(p, r), 'w').write(' '.join(os.environ[k] for k in "
            "('RANK', 'LOCAL_RANK', 'WORLD_SIZE', 'MASTER_ADDR', 'MASTER_PORT')))")
    rc = MD.launch_ranks([sys.executable, "-c", code, str(tmp_path)], 3, timeout_s=120)
    assert rc == 0
    rows = [open(tmp_path / str(r)).read().split() for r in range(3)]
    assert [r[:3] for r in rows] == [[str(r), str(r), "3"] for r in range(3)]
    assert len({r[4] for r in rows}) == 1 and rows[0][3] == "127.0.0.1"


def test_launch_ranks_stops_the_others_when_one_fails():
    code = ("import os, sys, time; r = int(os.environ['RANK']); "
            "sys.exit(3) if r == 1 else time.sleep(300)")
    rc = MD.launch_ranks([sys.executable, "-c", code], 2, timeout_s=120)
    assert rc != 0


def test_bench_refuses_a_gpu_count_other_than_the_world_size():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 2 and "disagrees with WORLD_SIZE" in r.stderr


def test_both_arms_print_the_same_config():
    import argparse
    sys.path.insert(0, ROOT)
    import bench
    args = bench_args = argparse.Namespace(fp8_experts=False, flush_l2=False)
    cfg = C.LONGCAT_PREFILL
    a = bench.workload_config(cfg, 1, args)
    b = bench.workload_config(cfg, 1, bench_args)
    assert a == b and a["workload"] == cfg.name and a["T"] == cfg.T
    assert set(a) >= {"workload", "T", "d", "N", "Z", "K", "I", "parallelism", "l2"}
    # every function the arms call exists
    for name in ("run_gpu", "run_reference", "cpu_baseline", "decode_block", "time_training",
                 "ClockSampler", "OracleWorkload", "main"):
        assert callable(getattr(bench, name)), name
