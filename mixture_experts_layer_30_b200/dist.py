"""Token data parallelism: the one exchange step of the layer.

Each rank routes its own batch with a full replica of the weights.  T_i and
T_all of Eq. (2) (LongCat-Flash Technical Report, §2.1.1) are global-batch
quantities, so the per-rank count histograms are summed over ranks before the
bias update; every rank then applies the same update to its bias copy.
"""
import torch
import torch.distributed as dist


def global_counts(counts_local: torch.Tensor, out: torch.Tensor, group=None) -> torch.Tensor:
    """out = sum over ranks of counts_local ([N+Z] int32), on every rank."""
    out.copy_(counts_local)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out


def global_tokens(T_local: int, group=None) -> int:
    """T_all: tokens of the global batch when every rank holds T_local tokens."""
    if dist.is_available() and dist.is_initialized():
        return T_local * dist.get_world_size(group)
    return T_local
