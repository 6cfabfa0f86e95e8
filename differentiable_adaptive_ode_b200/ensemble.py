"""Host-side plumbing for running one ensemble over several GPUs (one process per GPU).

Trajectories are independent ("gradsolve: fast exact gradients for ODE ensembles on GPUs" §4.4),
so an ensemble is split into contiguous ranges, one per rank, and each rank runs the whole path on
its range with no communication.  The only exchange the path has is the ensemble sum of the
parameter cotangent when theta is shared by all trajectories (the loss is a plain sum over
trajectories, §2.2): after each rank's gs_replay_grad, one all-reduce of m values.
"""
from typing import Tuple


def shard_range(N: int, rank: int, world: int) -> Tuple[int, int]:
    """[begin, end) of rank's contiguous share of N trajectories (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world %d/%d" % (rank, world))
    base, extra = divmod(N, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def allreduce_theta_bar(theta_bar, group=None):
    """Sum a shared-theta cotangent over ranks in place (NCCL on GPU tensors, gloo on CPU)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(theta_bar, op=dist.ReduceOp.SUM, group=group)
    return theta_bar


def max_over_ranks(value: float, device=None) -> float:
    """The largest of a per-rank scalar (used for device times: a job is as slow as its slowest
    rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
