"""One process per GPU: rank discovery, per-rank inputs and the max-over-ranks timing.

Every (sequence, head) of the mixer is independent, so N GPUs run N replicas of the
workload, each on its own seeded batch, with no collective on the data path (weak
scaling).  The only collectives are the barrier around the timed region and one
all-reduce(MAX) of the measured time.  Works with the NCCL backend on GPUs and with gloo on
CPU (the tests use gloo).
"""
from __future__ import annotations

import os

RANK_SEED_STRIDE = 1000  # rank r draws its inputs from seed + 1000 r


def env_rank():
    """(rank, world_size, local_rank) from the launcher's environment (1 process: 0, 1, 0)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s replica of a workload whose single-process seed is `seed`."""
    return seed + RANK_SEED_STRIDE * rank


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """The largest of every rank's x (each rank passes its own; all get the maximum)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, cuda: bool = True):
    """Barrier over all ranks, then (on GPUs) wait for this rank's device work."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if cuda:
        import torch
        torch.cuda.synchronize()


def aggregate(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job throughput of weak scaling: every rank processed `units_per_rank` units in
    at most `seconds` (the max over ranks)."""
    return units_per_rank * world / seconds
