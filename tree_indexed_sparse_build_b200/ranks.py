"""Host-side plumbing for running one replica of the decode path per GPU.

The path shards over (batch, KV head) units with no exchange between them, so N GPUs
run N independent replicas: each rank draws its own seeded cache and queries (its seed
offset by the rank), times its steps on its own device, and the job's time per step is the
slowest rank's.  The only collectives are a barrier around the timed region and one
max-reduction of the per-rank times.  Nothing here touches the method's arithmetic.
"""
from __future__ import annotations

import os
from dataclasses import dataclass

RANK_SEED_STRIDE = 7919  # seed offset between ranks (a prime, so streams never coincide)


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local: int


def rank_info(env=None) -> RankInfo:
    """RANK / WORLD_SIZE / LOCAL_RANK from the launcher's environment (1 rank without one)."""
    env = os.environ if env is None else env
    return RankInfo(int(env.get("RANK", "0")), int(env.get("WORLD_SIZE", "1")),
                    int(env.get("LOCAL_RANK", "0")))


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's replica: every rank routes its own synthetic cache."""
    return seed + RANK_SEED_STRIDE * rank


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_step_per_rank: int, world: int, slowest_ms_per_step: float) -> float:
    """Whole-job throughput: every rank's units per step over the slowest rank's step time."""
    return units_per_step_per_rank * world / (slowest_ms_per_step * 1e-3)
