"""Host-side plumbing for running the decode path on several GPUs.

The path shards over (batch, KV head) units with no exchange between them.  Two ways to use
N GPUs: N independent replicas (each rank draws its own seeded cache and queries, its seed
offset by the rank), or one workload whose units are split over the ranks (unit_range,
below) with the outputs all-gathered.  Each rank times its steps on its own device and the
job's time per step is the slowest rank's: the collectives are a barrier around the timed
region, one max-reduction of the per-rank times, and (split workload) the gather of the
outputs.  Nothing here touches the method's arithmetic.
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


# ---------------------------------------------------------------- one workload over N ranks
#
# The units of one workload -- its (batch, KV head) pairs, flattened as b * kv_heads + h --
# are independent, so N ranks can split them: rank r owns the contiguous range
# unit_range(units, N, r).  Its share is itself a tree set of batch 1 and (u1 - u0) KV heads:
# its K/V rows and its queries are contiguous slices of the flattened tensors (unit_slice,
# query_slice), so nothing is copied.  The outputs come back in unit order with one
# all-gather (gather_units), the only exchange of the path.


def unit_range(units: int, world: int, rank: int) -> tuple[int, int]:
    """[u0, u1) of the units rank `rank` of `world` owns: contiguous, sizes differ by at most
    one (the first units % world ranks take one more)."""
    if world < 1 or not 0 <= rank < world or units < 0:
        raise ValueError(f"bad split of {units} units: rank {rank} of {world}")
    base, extra = divmod(units, world)
    u0 = rank * base + min(rank, extra)
    return u0, u0 + base + (1 if rank < extra else 0)


def unit_slice(cache, u0: int, u1: int):
    """The rows of units [u0, u1) of a [batch, kv_heads, capacity, d] cache, as a contiguous
    [1, u1 - u0, capacity, d] view."""
    B, H, cap, d = cache.shape
    return cache.reshape(1, B * H, cap, d)[:, u0:u1]


def query_slice(Q, group: int, u0: int, u1: int):
    """The queries of units [u0, u1) of [batch, q_heads, nq, d] queries (query head hq reads
    KV head hq // group), as a contiguous [1, (u1 - u0) * group, nq, d] view."""
    B, Hq, nq, d = Q.shape
    return Q.reshape(1, B * Hq, nq, d)[:, u0 * group:u1 * group]


def gather_units(local, units: int, world: int, rank: int, rows_per_unit: int):
    """All-gather a unit-sharded tensor back into unit order on every rank.

    local: this rank's rows, [(u1 - u0) * rows_per_unit, ...] (e.g. its outputs with rows =
    its query heads x nq).  Every rank sends an equal-size buffer (its rows padded to the
    largest share) and keeps the valid rows of each.  Returns [units * rows_per_unit, ...]."""
    if world == 1:
        return local
    import torch
    import torch.distributed as dist
    most = -(-units // world) * rows_per_unit
    buf = torch.zeros((most,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    buf[:local.shape[0]] = local
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf)
    out = []
    for r in range(world):
        u0, u1 = unit_range(units, world, r)
        out.append(parts[r][:(u1 - u0) * rows_per_unit])
    return torch.cat(out)
