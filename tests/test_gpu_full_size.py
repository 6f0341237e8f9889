"""Parity at the five benchmark workloads' exact shapes, through the C ABI, in the launch
configurations the benchmark times.

The small cases elsewhere reach every kernel variant, but not the launch plans that only
these sizes take: the 1M tree's six levels and 262,144 leaves in the narrow 4,096-query
launch, the 128K steps that deepen the tree (L 3 -> 4) on their first token, the 4,096-token
append that deepens the 256K tree (L 7 -> 8), and the GQA step at 32K.  Each test draws the
workload's seeded cache, runs the calls the benchmark runs, and compares against the fp64
oracle (ZHA abstract, page 5: a tree of recursively compressed key summaries over the KV
cache, traversed from the top down by each query, deepened as the cache grows, followed by a
final attention):

* summaries: per node ||S_gpu - S_64|| / ||S_64|| <= 1e-6 (fp32 storage), bit-exact against
  the oracle's bf16 tree (bf16 storage);
* leaves and per-level survivors: bit-exact on every query whose fp64 beam margins exceed
  1e-3 |score| at every level; the other queries must hold a valid leaf set, and how many of
  them differ is printed;
* attention over the leaves the GPU selected: 1e-5 max-abs (fp32 cache and output) or 2e-2
  relative L2 (bf16), against fp64.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from tests.helpers import (RouteTally, assert_attention_bar, attend_unit_parity, out_to_f64,
                           route_unit_parity, summary_rel_err)
from tree_indexed_sparse_build_b200 import synth, workloads

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from tree_indexed_sparse_build_b200 import zha
    zha.lib()
    return torch.device("cuda:0")


def _tdt(w):
    return torch.float32 if w.kv_dtype == "f32" else torch.bfloat16


def _odt(w):
    return torch.float32 if w.out_dtype == "f32" else torch.bfloat16


def _otree(w, Kn, unit, N, summary="f64"):
    b, h = divmod(unit, w.kv_heads)
    return oracle.OracleTree(w.head_dim, w.leaf_block, w.branching, summary=summary).build(Kn[b, h], N)


def _check_summaries(tree, ot, unit, summary="f64"):
    """Every level of one unit against the oracle's tree; returns the worst relative error."""
    assert tree.levels == ot.L
    worst = 0.0
    for lvl in range(ot.L + 1):
        assert tree.level_nodes(lvl) == ot.levels[lvl].shape[0]
        got = tree.level(lvl)[unit].float().cpu().numpy().astype(np.float64)
        if summary == "bf16":
            assert np.array_equal(got, ot.levels[lvl]), f"bf16 level {lvl} of unit {unit} differs"
        else:
            worst = max(worst, summary_rel_err(got, ot.levels[lvl]))
    assert worst <= 1e-6, f"unit {unit}: summary rel err {worst}"
    return worst


def _inputs(w, capacity=None, nq=None, units=None):
    Qn = synth.queries(w, nq=nq)
    Kn = synth.keys(w, capacity=capacity, Q=Qn if w.needles else None, units=units)
    Vn = synth.values(w, capacity=capacity, units=units)
    return Qn, Kn, Vn


def _decode_parity(w, tree, Qn, Kn, Vn, N, O, idx, tr, units, summary="f64", trees=None):
    """Routes (with survivors) and outputs of the given units against the oracle."""
    Q64 = synth.to_f64(Qn)
    idx_n = idx.cpu().numpy()
    tr_n = tr.cpu().numpy() if tr is not None else None
    O64 = out_to_f64(O)
    tally = RouteTally()
    worst_abs = worst_rel = 0.0
    for u in units:
        ot = trees[u] if trees is not None else _otree(w, Kn, u, N, summary)
        route_unit_parity(w, ot, Q64, idx_n, tr_n, u, tally)
        a, r = attend_unit_parity(w, Q64, Kn, Vn, N, O64, idx_n, u)
        worst_abs, worst_rel = max(worst_abs, a), max(worst_rel, r)
    assert tally.checked > 0
    assert_attention_bar(w, worst_abs, worst_rel)
    return tally, worst_abs, worst_rel


def test_tiny_fp32_full(dev):
    """1,024 fp32 tokens, binary tree of 16-token leaves (64 leaves, 6 levels), beam 2, 16
    queries, fp32 output: the stand-alone route + attention calls and the fused call."""
    from tree_indexed_sparse_build_b200 import zha
    w = workloads.get("tiny_fp32")
    Qn, Kn, Vn = _inputs(w)
    Q, K, V = (synth.to_torch(x, dev) for x in (Qn, Kn, Vn))
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, w.seq_len, _tdt(w))
    tree.build(K, w.seq_len)
    idx, _, tr = tree.route(Q, w.beam, trace=True)
    O = tree.attend(Q, K, V, idx, w.beam, w.scale, out_dtype=torch.float32)
    Of, idxf, _, trf = tree.decode(Q, K, V, w.beam, w.scale, out_dtype=torch.float32, trace=True)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert tree.levels == 6 and tree.level_nodes(0) == 64
    assert torch.equal(idxf, idx) and torch.equal(trf, tr)
    _check_summaries(tree, _otree(w, Kn, 0, w.seq_len), 0)
    for out in (O, Of):
        tally, a, r = _decode_parity(w, tree, Qn, Kn, Vn, w.seq_len, out, idx, tr, [0])
    assert (idx >= 0).sum().item() == w.nq * w.beam  # two leaves = 32 keys per query
    print(f"tiny_fp32: {tally}; attention max-abs {a:.2e}")
    tree.close()


def test_gqa_32k_full(dev):
    """8 x 8 KV heads x 32,768 bf16 tokens, 32 query heads (group 4), b 8, 64-token leaves (512
    leaves, 3 levels), beam 8, 16 needles per KV head: one decode step (zha_decode, one query
    per head) and the same through zha_route + zha_sparse_attn_decode; every unit checked."""
    from tree_indexed_sparse_build_b200 import zha
    w = workloads.get("gqa_32k")
    Qn, Kn, Vn = _inputs(w)
    Q, K, V = (synth.to_torch(x, dev) for x in (Qn, Kn, Vn))
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, w.seq_len, _tdt(w))
    tree.build(K, w.seq_len)
    O, idx, _, tr = tree.decode(Q, K, V, w.beam, w.scale, trace=True)
    ridx, _, rtr = tree.route(Q, w.beam, trace=True)
    O2 = tree.attend(Q, K, V, ridx, w.beam, w.scale)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert tree.levels == 3 and tree.level_nodes(0) == 512
    assert torch.equal(idx, ridx) and torch.equal(tr, rtr)
    trees = {u: _otree(w, Kn, u, w.seq_len) for u in range(w.units)}
    for u in (0, 27, w.units - 1):
        _check_summaries(tree, trees[u], u)
    units = range(w.units)
    tally, a, r = _decode_parity(w, tree, Qn, Kn, Vn, w.seq_len, O, idx, tr, units, trees=trees)
    _, a2, r2 = _decode_parity(w, tree, Qn, Kn, Vn, w.seq_len, O2, ridx, None, units, trees=trees)
    print(f"gqa_32k: {tally}; attention rel L2 fused {r:.2e}, two-call {r2:.2e}")
    tree.close()


def test_decode_128k_full(dev):
    """4 x 8 KV heads x 131,072 bf16 tokens with positional drift, 32 query heads, b 16,
    32-token leaves (4,096 leaves, 3 levels), beam 16: 64 zha_decode_step calls (append one
    token, route, attend), the benchmark's launch.  The first step deepens the tree to 4
    levels.  Summaries of units 0 and 31 after steps 1, 2 and 64 against oracle builds over
    the same tokens; every step's leaves, survivors and outputs of every unit against the
    oracle's tree appended step by step."""
    from tree_indexed_sparse_build_b200 import zha
    w = workloads.get("decode_128k")
    N, steps = w.seq_len, w.decode_steps
    cap = N + steps
    Kn = synth.keys(w, capacity=cap)
    Vn = synth.values(w, capacity=cap)
    K, V = synth.to_torch(Kn, dev), synth.to_torch(Vn, dev)
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, cap, _tdt(w))
    tree.build(K, N)
    assert tree.levels == 3
    trees = {u: _otree(w, Kn, u, N) for u in range(w.units)}
    total = RouteTally()
    worst_rel = 0.0
    for s in range(steps):
        n = N + s + 1
        Qn = synth.queries(w, step=s)
        O, idx, tr = tree.decode_step(K, V, n, synth.to_torch(Qn, dev), w.beam, w.scale, trace=True)
        torch.cuda.synchronize()
        assert tree.check() == zha.ZHA_OK
        assert tree.seq_len == n and tree.levels == 4
        for u in range(w.units):
            b, h = divmod(u, w.kv_heads)
            trees[u].append(Kn[b, h], n)
        if s in (0, 1, steps - 1):
            for u in (0, w.units - 1):
                _check_summaries(tree, _otree(w, Kn, u, n), u)
        tally, _, r = _decode_parity(w, tree, Qn, Kn, Vn, n, O, idx, tr, range(w.units), trees=trees)
        total.checked += tally.checked
        total.ill += tally.ill
        total.ill_mismatch += tally.ill_mismatch
        worst_rel = max(worst_rel, r)
    assert tree.level_nodes(0) == 4098
    print(f"decode_128k, {steps} steps: {total}; attention rel L2 {worst_rel:.2e}")
    tree.close()


@pytest.fixture(scope="module")
def deep_1m():
    """The 1M workload's seeded cache and its 64 queries per head (drawn once)."""
    w = workloads.get("deep_1m")
    Qn, Kn, Vn = _inputs(w, nq=workloads.THROUGHPUT_NQ)
    return w, Qn, Kn, Vn


@pytest.mark.parametrize("summary", ["f32", "bf16"])
def test_deep_1m_full(dev, deep_1m, summary):
    """1 x 8 KV heads x 1,048,576 bf16 tokens, 64 query heads (group 8), b 8, 4-token leaves
    (262,144 leaves, 6 levels), beam 8, 64 needles per KV head: the 4,096-query zha_decode (64
    queries per head: the narrow launch) and the single step (one query per head: the wide
    launch), over fp32- and bf16-stored summaries.  Summaries of units 0 and 7; every query's
    leaves, survivors and output."""
    from tree_indexed_sparse_build_b200 import zha
    w, Qn, Kn, Vn = deep_1m
    sdt = torch.bfloat16 if summary == "bf16" else torch.float32
    osum = "bf16" if summary == "bf16" else "f64"
    Q, K, V = (synth.to_torch(x, dev) for x in (Qn, Kn, Vn))
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, w.seq_len, _tdt(w),
                    summary_dtype=sdt)
    tree.build(K, w.seq_len)
    O, idx, _, tr = tree.decode(Q, K, V, w.beam, w.scale, trace=True)
    Q1 = Q[:, :, :1].contiguous()
    O1, idx1, _, tr1 = tree.decode(Q1, K, V, w.beam, w.scale, trace=True)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert tree.levels == 6 and tree.level_nodes(0) == 262144
    assert torch.equal(idx1, idx[:, :, :1]) and torch.equal(tr1, tr[:, :, :1])
    del K, V, Q
    tally = RouteTally()
    worst_rel = 0.0
    for u in range(w.units):
        ot = _otree(w, Kn, u, w.seq_len, osum)
        if u in (0, w.units - 1):
            _check_summaries(tree, ot, u, osum)
        t, _, r = _decode_parity(w, tree, Qn, Kn, Vn, w.seq_len, O, idx, tr, [u], trees={u: ot})
        _decode_parity(w, tree, Qn[:, :, :1], Kn, Vn, w.seq_len, O1, idx1, tr1, [u], trees={u: ot})
        tally.checked += t.checked
        tally.ill += t.ill
        tally.ill_mismatch += t.ill_mismatch
        worst_rel = max(worst_rel, r)
        del ot
    print(f"deep_1m ({summary} summaries): {tally}; attention rel L2 {worst_rel:.2e}")
    tree.close()


def test_build_256k_full(dev):
    """8 KV heads x 262,144 bf16 tokens, b 4, 16-token leaves (16,384 leaves, 7 levels): the
    build, one 4,096-token append (16,640 leaves, 8 levels), then 64 queries per head (2,048)
    through zha_decode and through zha_route + zha_sparse_attn_decode.  Every unit's
    summaries after the build and after the append; every query's leaves, survivors and
    output."""
    from tree_indexed_sparse_build_b200 import zha
    w = workloads.get("build_256k")
    N, cap = w.seq_len, w.capacity
    Qn, Kn, Vn = _inputs(w, capacity=cap)
    Q, K, V = (synth.to_torch(x, dev) for x in (Qn, Kn, Vn))
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, cap, _tdt(w))
    tree.build(K, N)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert tree.levels == 7 and tree.level_nodes(0) == 16384
    for u in range(w.units):
        _check_summaries(tree, _otree(w, Kn, u, N), u)
    tree.append(K, cap)
    O, idx, _, tr = tree.decode(Q, K, V, w.beam, w.scale, trace=True)
    ridx, _, rtr = tree.route(Q, w.beam, trace=True)
    O2 = tree.attend(Q, K, V, ridx, w.beam, w.scale)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert tree.levels == 8 and tree.level_nodes(0) == 16640
    assert torch.equal(idx, ridx) and torch.equal(tr, rtr)
    trees = {u: _otree(w, Kn, u, cap) for u in range(w.units)}
    for u in range(w.units):
        _check_summaries(tree, trees[u], u)
    units = range(w.units)
    tally, a, r = _decode_parity(w, tree, Qn, Kn, Vn, cap, O, idx, tr, units, trees=trees)
    _, _, r2 = _decode_parity(w, tree, Qn, Kn, Vn, cap, O2, ridx, None, units, trees=trees)
    print(f"build_256k: {tally}; attention rel L2 fused {r:.2e}, two-call {r2:.2e}")
    tree.close()
