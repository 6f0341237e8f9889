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
