"""The benchmark's algorithmic byte counts, against brute-force counts on routed trees.

The roofline's `achieved` figure divides these counts by kernel time, so they are pinned here:
bench.path_bytes (the union per (batch, KV head) of the summary rows scored and of the leaf
tokens attended, plus Q, indices and O) against a plain set count over the oracle's own
per-level candidates, and bench.level_counts / bench.append_bytes against the tree's
definition.  CPU only.
"""
from __future__ import annotations

import numpy as np
import pytest

import bench
import oracle
from tree_indexed_sparse_build_b200 import synth
from tree_indexed_sparse_build_b200.workloads import Workload


def _w(N, b, lb, beam, kvh, g, nq, d=16):
    return Workload(name="bytes", batch=2, kv_heads=kvh, q_heads=kvh * g, head_dim=d, seq_len=N, kv_dtype="f32",
                    branching=b, leaf_block=lb, beam=beam, nq=nq, out_dtype="f32", seed=77)


@pytest.mark.parametrize("N,b,lb,beam,kvh,g,nq", [(1000, 2, 16, 2, 1, 1, 5), (3001, 4, 7, 3, 2, 2, 3),
                                                   (5000, 8, 4, 8, 1, 4, 2), (777, 3, 5, 4, 2, 1, 4)])
def test_path_bytes_equal_brute_force_union(N, b, lb, beam, kvh, g, nq):
    w = _w(N, b, lb, beam, kvh, g, nq)
    Q = synth.queries(w)
    K = synth.keys(w)
    counts = bench.level_counts(N, lb, b)
    L = len(counts) - 1
    idx = np.empty((w.batch, w.q_heads, nq, beam), np.int64)
    trace = np.empty((w.batch, w.q_heads, nq, L, beam), np.int64)
    rows = toks = 0
    for bb in range(w.batch):
        for h in range(kvh):
            ot = oracle.OracleTree(w.head_dim, lb, b).build(K[bb, h], N)
            scored, attended = set(), set()
            for hq in range(h * g, (h + 1) * g):
                res = ot.route(synth.to_f64(Q[bb, hq]), beam)
                idx[bb, hq] = res["leaves"]
                trace[bb, hq] = res["survivors"]
                for i in range(nq):
                    # candidates of level l: every child of the survivors of level l + 1
                    surv = [0]  # the root
                    for li in range(L):
                        l = L - 1 - li
                        for s in surv:
                            for c in range(s * b, min(s * b + b, counts[l])):
                                scored.add((l, c))
                        surv = [int(x) for x in res["survivors"][i, li] if x >= 0]
                    for leaf in res["leaves"][i]:
                        if leaf >= 0:
                            attended.update(range(leaf * lb, min(leaf * lb + lb, N)))
            rows += len(scored)
            toks += len(attended)
    q = w.batch * w.q_heads * nq
    d, e = w.head_dim, 4
    pb = bench.path_bytes(idx, trace, counts, N, lb, b, d, e, g, 4)
    assert pb["route_bytes"] == rows * d * 4 + q * d * e + q * beam * 4
    assert pb["attend_bytes"] == toks * 2 * d * e + q * d * e + q * beam * 4 + q * d * 4
    # bf16 summaries halve the rows' part
    pb2 = bench.path_bytes(idx, trace, counts, N, lb, b, d, e, g, 4, sum_bytes=2)
    assert pb2["route_bytes"] == rows * d * 2 + q * d * e + q * beam * 4


@pytest.mark.parametrize("N,lb,b", [(1, 4, 2), (1024, 16, 2), (131073, 32, 16), (1048576, 4, 8), (266240, 16, 4)])
def test_level_counts_follow_the_tree_definition(N, lb, b):
    c = bench.level_counts(N, lb, b)
    assert c[0] == -(-N // lb) and c[-1] == 1
    assert len(c) - 1 == oracle.num_levels(c[0], b)
    for l in range(1, len(c)):
        assert c[l] == -(-c[l - 1] // b)


def test_append_bytes_one_leaf_path():
    # a one-token append at N = 1025 (leaf block 16, binary tree): the new leaf 64 holds one
    # token; every level above reads the existing children of the path node, and L + 1 rows
    # are written
    d, e, units = 8, 2, 3
    got = bench.append_bytes(1025, 16, 2, d, e, units, sum_bytes=4)
    c = bench.level_counts(1025, 16, 2)  # 65, 33, 17, 9, 5, 3, 2, 1
    L = len(c) - 1
    node, per = 64, 1 * d * e
    for l in range(1, L + 1):
        node //= 2
        per += (min(node * 2 + 2, c[l - 1]) - node * 2) * d * 4
    per += (L + 1) * d * 4
    assert got == per * units
