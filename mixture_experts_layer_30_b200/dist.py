"""Token data parallelism: the one exchange step of the layer.

Each rank routes its own batch with a full replica of the weights.  T_i and
T_all of Eq. (2) (LongCat-Flash Technical Report, §2.1.1) are global-batch
quantities, so the per-rank count histograms are summed over ranks before the
bias update; every rank then applies the same update to its bias copy.

Also the launch plumbing of a multi-rank run on one node: the per-rank input
seed, the maximum of a time over ranks, and a launcher that starts one
process per GPU with the torchrun environment.
"""
import os
import socket
import subprocess
import sys
import time

import torch
import torch.distributed as dist

# x of rank r > 0 is drawn with its own seed; rank 0 keeps the workload's x
RANK_X_SEED_BASE = 7_000_000


def _multi(group=None) -> bool:
    return dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1


def global_counts(counts_local: torch.Tensor, out: torch.Tensor, group=None) -> torch.Tensor:
    """out = sum over ranks of counts_local ([N+Z] int32), on every rank."""
    out.copy_(counts_local)
    if _multi(group):
        dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out


def global_tokens(T_local: int, group=None) -> int:
    """T_all: tokens of the global batch when every rank holds T_local tokens."""
    if dist.is_available() and dist.is_initialized():
        return T_local * dist.get_world_size(group)
    return T_local


def rank_x_seed(rank: int):
    """Seed of rank ``rank``'s activations (None: the workload's own x)."""
    return None if rank == 0 else RANK_X_SEED_BASE + rank


def max_over_ranks(value: float, device, group=None) -> float:
    """The largest of every rank's ``value`` (e.g. a step time), on every rank."""
    if not _multi(group):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_ranks(cmd, n: int, timeout_s: float = 3600.0, quiet_others: bool = True) -> int:
    """Runs ``cmd`` as n local ranks (RANK, LOCAL_RANK, WORLD_SIZE, MASTER_ADDR,
    MASTER_PORT set as torchrun sets them; rank r on GPU r).  Rank 0 writes to
    this process's stdout; the others' stdout is discarded when quiet_others.
    If a rank fails or the time runs out, the others are terminated.  Returns
    the largest exit code."""
    port = free_port()
    procs = []
    for r in range(n):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(n),
                   LOCAL_WORLD_SIZE=str(n), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        out = subprocess.DEVNULL if (r and quiet_others) else None
        procs.append(subprocess.Popen(cmd, env=env, stdout=out))
    deadline = time.monotonic() + timeout_s
    codes = [None] * n
    while any(c is None for c in codes):
        for i, p in enumerate(procs):
            if codes[i] is None:
                codes[i] = p.poll()
        failed = any(c not in (None, 0) for c in codes)
        if failed or time.monotonic() > deadline:
            for i, p in enumerate(procs):
                if codes[i] is None:
                    p.terminate()
            for i, p in enumerate(procs):
                if codes[i] is None:
                    try:
                        codes[i] = p.wait(timeout=60)
                    except subprocess.TimeoutExpired:
                        p.kill()
                        codes[i] = p.wait()
            if not failed:
                sys.stderr.write(f"launch_ranks: ranks still running after {timeout_s} s\n")
                return 124
            break
        time.sleep(0.05)
    return max(abs(c) for c in codes)
