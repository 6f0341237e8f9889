"""Shared helpers for the GPU parity tests: seeded inputs, oracle trees, comparisons."""
from __future__ import annotations

import numpy as np

import oracle
from tree_indexed_sparse_build_b200 import synth
from tree_indexed_sparse_build_b200.workloads import Workload


def torch_of(x: np.ndarray, device):
    return synth.to_torch(x, device)


def make_inputs(w: Workload, capacity: int | None = None, nq: int | None = None):
    """(Q, K, V) numpy arrays in storage types for workload w."""
    Q = synth.queries(w, nq=nq)
    K = synth.keys(w, capacity=capacity, Q=Q if w.needles else None)
    V = synth.values(w, capacity=capacity)
    return Q, K, V


def oracle_tree(w: Workload, K: np.ndarray, unit: int, N: int, summary: str = "f64") -> oracle.OracleTree:
    """The oracle's tree of one unit; summary "bf16" mirrors bf16-stored summaries."""
    b, h = divmod(unit, w.kv_heads)
    return oracle.OracleTree(w.head_dim, w.leaf_block, w.branching, summary=summary).build(K[b, h], N)


def summary_rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    """Largest per-node normwise relative error ||got - ref|| / ||ref||."""
    got = got.astype(np.float64)
    num = np.linalg.norm(got - ref, axis=-1)
    den = np.linalg.norm(ref, axis=-1)
    rel = np.where(den > 0, num / np.where(den > 0, den, 1.0), num)
    return float(rel.max()) if rel.size else 0.0


def out_to_f64(O) -> np.ndarray:
    import torch
    if O.dtype == torch.bfloat16:
        return O.float().cpu().numpy().astype(np.float64)
    return O.cpu().numpy().astype(np.float64)


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


class RouteTally:
    """Counts of a route comparison: well-conditioned queries (bit-exact), ill-conditioned
    queries (reported) and how many of those differ from the oracle's set."""

    def __init__(self):
        self.checked = self.ill = self.ill_mismatch = 0

    def rate(self) -> float:
        return self.ill_mismatch / max(self.checked + self.ill, 1)

    def __repr__(self):
        return (f"well-conditioned {self.checked} (bit-exact), ill-conditioned {self.ill}, "
                f"ill mismatches {self.ill_mismatch} (rate {self.rate():.2e})")


def route_unit_parity(w: Workload, ot: oracle.OracleTree, Q64: np.ndarray, idx: np.ndarray,
                      trace: np.ndarray | None, unit: int, tally: RouteTally, flat=None) -> None:
    """Compare one (batch, KV head) unit's routed leaves (and per-level survivors) with the
    oracle's beam descent.  Q64: fp64 queries [batch, q_heads, nq, d]; idx [batch, q_heads,
    nq, beam]; trace [batch, q_heads, nq, levels, beam] or None.  Well-conditioned queries
    must match exactly; the others must still be a valid leaf set (ascending, distinct, in
    range, min(beam, n0) of them) and are counted."""
    b, h = divmod(unit, w.kv_heads)
    g = w.group
    n0 = ot.levels[0].shape[0]
    flat = flat if flat is not None else ot.flat()
    for hq in range(h * g, (h + 1) * g):
        res = ot.route(Q64[b, hq], w.beam, flat=flat)
        ok = oracle.well_conditioned(res["bounds"])
        got = idx[b, hq]
        np.testing.assert_array_equal(got[ok], res["leaves"][ok])
        if trace is not None:
            np.testing.assert_array_equal(trace[b, hq][ok], res["survivors"][ok])
        tally.checked += int(ok.sum())
        for i in np.flatnonzero(~ok):
            tally.ill += 1
            valid = got[i][got[i] >= 0]
            assert len(valid) == min(w.beam, n0)
            assert (np.diff(valid) > 0).all() and valid.max() < n0 and valid.min() >= 0
            tally.ill_mismatch += int(not np.array_equal(got[i], res["leaves"][i]))


def attend_unit_parity(w: Workload, Q64: np.ndarray, K: np.ndarray, V: np.ndarray, N: int,
                       O: np.ndarray, idx: np.ndarray, unit: int) -> tuple[float, float]:
    """Worst (max-abs, relative L2) of one unit's outputs O (fp64 [batch, q_heads, nq, d])
    against the oracle's exact attention over the leaves the GPU selected (idx)."""
    b, h = divmod(unit, w.kv_heads)
    worst_abs = worst_rel = 0.0
    for hq in range(h * w.group, (h + 1) * w.group):
        for i in range(Q64.shape[2]):
            ref, _ = oracle.attend(Q64[b, hq, i], K[b, h], V[b, h], N, w.leaf_block,
                                   idx[b, hq, i].astype(np.int64), w.scale)
            worst_abs = max(worst_abs, float(np.abs(O[b, hq, i] - ref).max()))
            worst_rel = max(worst_rel, rel_l2(O[b, hq, i], ref))
    return worst_abs, worst_rel


def assert_attention_bar(w: Workload, worst_abs: float, worst_rel: float) -> None:
    """1e-5 max-abs for an fp32 cache with fp32 output, else 2e-2 relative L2."""
    if w.kv_dtype == "f32" and w.out_dtype == "f32":
        assert worst_abs <= 1e-5, f"max-abs {worst_abs}"
    else:
        assert worst_rel <= 2e-2, f"rel L2 {worst_rel}"
