"""The benchmark's parity sample and its per-workload summary (CPU only).

bench.parity_sample compares one call's outputs with the fp64 oracle and reports, never
raises.  Fed the oracle's own results it must report a pass; fed a plausible mistake (a
wrong leaf on a well-conditioned query, a perturbed output, a perturbed summary) it must
report a failure.  config_summary must fit the few hundred characters that end the JSON line.
"""
from __future__ import annotations

import json

import numpy as np

import bench
import oracle
from tree_indexed_sparse_build_b200 import synth, workloads


def _oracle_outputs(w, Q, K, V, N):
    """The oracle's own leaves, survivors and outputs for every query of w (no GPU)."""
    Q64 = synth.to_f64(Q)
    B, Hq, nq, d = Q.shape
    idx = np.empty((B, Hq, nq, w.beam), np.int64)
    O = np.empty((B, Hq, nq, d), np.float64)
    trees = {}
    trace = None
    for u in range(w.units):
        b, h = divmod(u, w.kv_heads)
        trees[u] = oracle.OracleTree(w.head_dim, w.leaf_block, w.branching).build(K[b, h], N)
        if trace is None:
            trace = np.empty((B, Hq, nq, trees[u].L, w.beam), np.int64)
        for hq in range(h * w.group, (h + 1) * w.group):
            res = trees[u].route(Q64[b, hq], w.beam)
            idx[b, hq], trace[b, hq] = res["leaves"], res["survivors"]
            for i in range(nq):
                O[b, hq, i], _ = oracle.attend(Q64[b, hq, i], K[b, h], V[b, h], N, w.leaf_block,
                                               res["leaves"][i], w.scale)
    return idx, trace, O, trees


def _tiny():
    w = workloads.get("tiny_fp32")
    Q = synth.queries(w)
    K = synth.keys(w, Q=Q)
    V = synth.values(w)
    return w, Q, K, V


def test_oracle_results_pass():
    w, Q, K, V = _tiny()
    idx, tr, O, trees = _oracle_outputs(w, Q, K, V, w.seq_len)
    p = bench.parity_sample(w, Q, K, V, w.seq_len, idx, tr, O, [0],
                            gpu_levels=lambda u: trees[u].levels)
    assert p["pass"] and p["summaries_ok"] and p["summary_max_rel_err"] == 0.0
    assert p["queries"] == 16 and p["exact"] == p["well_conditioned"] > 0
    assert p["ill_mismatch"] == 0 and p["attn_max_abs"] < 1e-12
    assert bench.parity_brief(p).startswith("ok ")


def test_planted_mistakes_fail():
    w, Q, K, V = _tiny()
    idx, tr, O, trees = _oracle_outputs(w, Q, K, V, w.seq_len)
    res = trees[0].route(synth.to_f64(Q)[0, 0], w.beam)
    i = int(np.flatnonzero(oracle.well_conditioned(res["bounds"]))[0])
    n0 = trees[0].levels[0].shape[0]
    bad = idx.copy()  # a leaf replaced by one the query did not select
    bad[0, 0, i, 0] = next(x for x in range(n0) if x not in set(idx[0, 0, i].tolist()))
    bad[0, 0, i] = np.sort(bad[0, 0, i])
    p = bench.parity_sample(w, Q, K, V, w.seq_len, bad, None, O, [0])
    assert not p["pass"] and p["exact"] == p["well_conditioned"] - 1
    Ob = O.copy()
    Ob[0, 0, i, 3] += 2e-5  # beyond the fp32 bar of 1e-5 max-abs
    assert not bench.parity_sample(w, Q, K, V, w.seq_len, idx, tr, Ob, [0])["pass"]
    lv = [x.copy() for x in trees[0].levels]
    lv[2][1] *= 1.0 + 1e-5  # one node 1e-5 off: beyond the 1e-6 summary bar
    p = bench.parity_sample(w, Q, K, V, w.seq_len, idx, tr, O, [0], gpu_levels=lambda u: lv)
    assert not p["pass"] and not p["summaries_ok"]
    assert bench.parity_brief(p).startswith("FAIL")


def test_summary_fits_the_line_tail():
    par = {"pass": True, "exact": 3647, "well_conditioned": 3647, "ill_mismatch": 12, "ill_conditioned": 449,
           "attn_bar": "rel L2 2e-2", "attn_max_rel_l2": 2.17e-3, "attn_max_abs": 1e-3}
    small = {"qps": 1.23456e7, "ms": 0.0123456, "frac_of_peak": 0.123456, "keys_per_query": 512.0, "parity": par}
    one = {"qps": 3.1e7, "ms_per_step": 0.1234567, "frac_of_peak": 0.3456789, "keys_per_query": 32.0,
           "parity": par}
    line = {"value": 3.4e6, "ms_per_step": 0.0375, "roofline": {"frac": 0.216}, "keys_per_query": 512.0,
            "parity": par, "tiny_fp32": small, "gqa_32k": small,
            "ctx_1m": {"throughput": one, "single": one}, "ctx_1m_bf16_summaries": {"throughput": one, "single": one},
            "build_256k": {"build_gbs": 4570.123, "append_4096_ms": 0.0195, "qps": 4.0e7, "parity": par}}
    o = {k: 1234.5678 for k in ("tiny_fp32", "gqa_32k", "decode_128k", "deep_1m", "build_256k")}
    s = json.dumps({"configs": bench.config_summary(line, o, o)})
    assert len(s) < 1400, len(s)
    c = json.loads(s)["configs"]
    assert set(c) == {"tiny_fp32", "gqa_32k", "decode_128k", "deep_1m", "deep_1m_bf16sum", "build_256k"}
