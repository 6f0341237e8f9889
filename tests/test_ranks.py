"""Multi-rank host plumbing of the benchmark on CPU (gloo, world size 2, 127.0.0.1).

The path runs one independent replica per GPU: these tests check the rank environment,
that ranks draw different seeded inputs, the barrier and max-over-ranks reduction the
timing uses, the whole-job rate, and that a rank which never joins the reduction makes the
others fail within the process group's timeout instead of hanging.
"""
from __future__ import annotations

import datetime
import os
import socket

import numpy as np
import pytest

from tree_indexed_sparse_build_b200 import ranks, synth
from tree_indexed_sparse_build_b200.workloads import get

torch = pytest.importorskip("torch")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_rank_info_from_environment():
    assert ranks.rank_info({}) == ranks.RankInfo(0, 1, 0)
    assert ranks.rank_info({"RANK": "3", "WORLD_SIZE": "8", "LOCAL_RANK": "3"}) == ranks.RankInfo(3, 8, 3)


def test_rank_replicas_draw_different_inputs():
    w = get("tiny_fp32").with_(needles=0)
    k0 = synth.keys(w.with_(seed=ranks.rank_seed(w.seed, 0)))
    k0b = synth.keys(w.with_(seed=ranks.rank_seed(w.seed, 0)))
    k1 = synth.keys(w.with_(seed=ranks.rank_seed(w.seed, 1)))
    assert np.array_equal(k0, k0b)
    assert not np.array_equal(k0, k1)


def test_weak_scaling_rate():
    # 128 queries per rank per step, 4 ranks, slowest rank 40 us per step
    assert ranks.weak_scaling_rate(128, 4, 0.040) == pytest.approx(128 * 4 / 40e-6)
    assert ranks.max_over_ranks(2.5, 1) == 2.5


def _worker(rank: int, world: int, port: int, out_dir: str, drop_rank: int):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    ri = ranks.rank_info()
    dist.init_process_group("gloo", rank=ri.rank, world_size=ri.world,
                            timeout=datetime.timedelta(seconds=5))
    ranks.barrier(ri.world)
    slowest = ranks.max_over_ranks(1.0 + 0.5 * ri.rank, ri.world)  # per-rank ms per step
    rate = ranks.weak_scaling_rate(128, ri.world, slowest)
    with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
        f.write(f"{slowest} {rate}\n")
    if rank == drop_rank:
        return  # leaves between steps: never joins the next reduction
    try:
        ranks.max_over_ranks(float(rank), ri.world)
        status = "completed"
    except Exception:
        status = "error"
    with open(os.path.join(out_dir, f"r{rank}_next.txt"), "w") as f:
        f.write(status)
    if drop_rank < 0:
        dist.destroy_process_group()


@pytest.mark.parametrize("drop_rank", [-1, 1], ids=["all_ranks", "rank1_leaves"])
def test_gloo_two_ranks(tmp_path, drop_rank):
    import torch.multiprocessing as mp
    mp.start_processes(_worker, args=(2, _free_port(), str(tmp_path), drop_rank), nprocs=2,
                       join=True, start_method="spawn")
    for r in range(2):
        slowest, rate = map(float, (tmp_path / f"r{r}.txt").read_text().split())
        assert slowest == 1.5  # the slower rank's time, on every rank
        assert rate == pytest.approx(128 * 2 / 1.5e-3)
    if drop_rank < 0:
        assert (tmp_path / "r0_next.txt").read_text() == "completed"
        assert (tmp_path / "r1_next.txt").read_text() == "completed"
    else:
        # the remaining rank's collective ends with an error after the 5 s group timeout
        assert (tmp_path / "r0_next.txt").read_text() == "error"
