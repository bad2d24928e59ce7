"""Host-side bookkeeping for runs with one process per GPU.

The WKV operator shards over batch rows, channels and heads with no exchange
step, so a multi-GPU run is N independent problems (weak scaling): nothing here
touches the data path.  What the ranks share is the clock: the step time of a
run is the slowest rank's device time, and its throughput is all ranks' work
over that time.
"""

from __future__ import annotations

SEED_STRIDE = 1000  # rank r draws its problem from seed base + SEED_STRIDE * r


def rank_seed(base: int, rank: int) -> int:
    """Seed of rank `rank`'s independent problem."""
    if rank < 0:
        raise ValueError("rank must be >= 0")
    return base + SEED_STRIDE * rank


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks of the default process group (the
    value itself without one).  `device` is where the reduction tensor lives:
    a CUDA device for NCCL, None (CPU) for gloo."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_throughput(units_per_rank: float, world: int, ms_per_step_max: float) -> float:
    """Units per second of the whole job: every rank's units over the slowest
    rank's step time."""
    if world < 1 or ms_per_step_max <= 0:
        raise ValueError("world must be >= 1 and the step time positive")
    return world * units_per_rank / (ms_per_step_max * 1e-3)
