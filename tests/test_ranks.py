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


# ---------------------------------------------------------------- one workload split over ranks

@pytest.mark.parametrize("units", [1, 3, 5, 32, 33, 64])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_unit_ranges_cover_every_unit_once(units, world):
    seen = []
    sizes = []
    for r in range(world):
        u0, u1 = ranks.unit_range(units, world, r)
        assert 0 <= u0 <= u1 <= units
        seen.extend(range(u0, u1))
        sizes.append(u1 - u0)
    assert seen == list(range(units))  # every unit once, in order
    assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        ranks.unit_range(units, world, world)


def test_unit_and_query_slices_are_contiguous_views():
    B, H, g, cap, d, nq = 2, 3, 2, 5, 4, 3
    K = torch.arange(B * H * cap * d, dtype=torch.float32).reshape(B, H, cap, d)
    Q = torch.arange(B * H * g * nq * d, dtype=torch.float32).reshape(B, H * g, nq, d)
    for u0, u1 in [(0, 6), (2, 5), (4, 6), (3, 3)]:
        ks = ranks.unit_slice(K, u0, u1)
        qs = ranks.query_slice(Q, g, u0, u1)
        assert ks.shape == (1, u1 - u0, cap, d) and ks.is_contiguous()
        assert qs.shape == (1, (u1 - u0) * g, nq, d) and qs.is_contiguous()
        for u in range(u0, u1):
            b, h = divmod(u, H)
            assert torch.equal(ks[0, u - u0], K[b, h])
            for j in range(g):  # query head h * g + j reads KV head h
                assert torch.equal(qs[0, (u - u0) * g + j], Q[b, h * g + j])


def _oracle_outputs(w, units, Qn, Kn, Vn):
    """The fp64 oracle's route + attention for the query heads of `units`: [len * g * nq, d]."""
    import oracle
    rows = []
    for u in units:
        b, h = divmod(u, w.kv_heads)
        ot = oracle.OracleTree(w.head_dim, w.leaf_block, w.branching).build(Kn[b, h], w.seq_len)
        for hq in range(h * w.group, (h + 1) * w.group):
            q64 = synth.to_f64(Qn[b, hq])
            leaves = ot.route(q64, w.beam)["leaves"]
            for i in range(q64.shape[0]):
                o, _ = oracle.attend(q64[i], Kn[b, h], Vn[b, h], w.seq_len, w.leaf_block, leaves[i], w.scale)
                rows.append(o)
    return torch.from_numpy(np.array(rows))


SPLIT_W = get("tiny_fp32").with_(batch=1, kv_heads=5, q_heads=10, seq_len=200, nq=3, needles=0, leaf_block=8)


def _split_worker(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    w = SPLIT_W
    Qn = synth.queries(w)
    Kn, Vn = synth.keys(w), synth.values(w)
    u0, u1 = ranks.unit_range(w.units, world, rank)
    local = _oracle_outputs(w, range(u0, u1), Qn, Kn, Vn)  # this rank's share (stand-in outputs)
    full = ranks.gather_units(local, w.units, world, rank, w.group * w.nq)
    torch.save(full, os.path.join(out_dir, f"gathered{rank}.pt"))
    dist.destroy_process_group()


def test_split_workload_gathers_in_unit_order(tmp_path):
    import torch.multiprocessing as mp
    mp.start_processes(_split_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    w = SPLIT_W
    ref = _oracle_outputs(w, range(w.units), synth.queries(w), synth.keys(w), synth.values(w))
    assert ref.shape == (w.units * w.group * w.nq, w.head_dim)
    for r in range(2):
        got = torch.load(tmp_path / f"gathered{r}.pt")
        assert torch.equal(got, ref)  # the 1-rank order, bit for bit
