"""Pins for the oracle's bf16-stored summaries.

The pages fix no storage precision for the summaries ("Subquadratic Attention with a
Hierarchical Tree-Structured Indexer", abstract: recursively compressed key summaries).
The reading pinned here: a stored node is its fp64 mean rounded to the nearest fp32 and
then to the nearest bf16 (ties to even both times), and a parent averages its children's
stored values.  Pins: a library conversion (numpy's fp32 cast followed by torch's bf16
cast) on random values, hand-worked ties and a hand-worked parent whose value tells the
stored-children rule from a token mean, a case that tells rounding through fp32 from
direct rounding, closed forms (constant keys), invariants (every value is a bf16, append
== rebuild exactly) and an error bound against the exact tree.
"""
import numpy as np
import pytest

import oracle
from tree_indexed_sparse_build_b200 import synth, workloads

torch = pytest.importorskip("torch")

U7, U8 = 2.0 ** -7, 2.0 ** -8  # bf16 spacing above 1, and half of it


def _f32(x):
    return np.ascontiguousarray(np.asarray(x, np.float32))


def test_round_bf16_equals_library_conversion():
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(20000) * np.exp2(rng.integers(-30, 30, 20000)),
        rng.standard_normal(2000) * 1e-39,  # fp32 subnormals
        [0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38],
    ])
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(x), ref)


def test_round_bf16_hand_values():
    x = np.array([1 + U8, 1 + 3 * U8, -(1 + U8), 1 + U8 + 2.0 ** -12, 1 + U8 + 2.0 ** -30])
    # ties go to the even neighbour (1.0; 1 + 2^-6); just above a tie rounds up; the last
    # value is above the tie in fp64 but lands on it in fp32, so it goes to 1.0
    np.testing.assert_array_equal(oracle.round_bf16(x), [1.0, 1 + 2 * U7, -1.0, 1 + U7, 1.0])


def test_leaf_means_round_ties_to_even():
    K = _f32([[1.0], [1 + U7], [1 + U7], [1 + 2 * U7]])
    t = oracle.OracleTree(1, 2, 2, summary="bf16").build(K, 4)
    # means 1 + 2^-8 and 1 + 3 2^-8 are ties: to 1.0 and 1 + 2^-6 (even mantissas)
    np.testing.assert_array_equal(t.levels[0][:, 0], [1.0, 1 + 2 * U7])


def test_parent_averages_stored_children():
    # x rounds up to 1 + 2^-7, y rounds up to 1 + 2^-6; their stored mean 1 + 3 2^-8 is a
    # tie and goes to 1 + 2^-6.  The token mean 1 + 2^-7 + 2^-12 would store 1 + 2^-7.
    x, y = 1 + U8 + 2.0 ** -12, 1 + U7 + U8 + 2.0 ** -12
    t = oracle.OracleTree(1, 1, 2, summary="bf16").build(_f32([[x], [y]]), 2)
    np.testing.assert_array_equal(t.levels[0][:, 0], [1 + U7, 1 + 2 * U7])
    assert t.levels[1][0, 0] == 1 + 2 * U7
    assert oracle.round_bf16(np.array([(x + y) / 2]))[0] == 1 + U7


def test_leaf_rounds_through_fp32():
    # mean = 1 + 2^-8 + 2^-23 / 3: above the bf16 tie, but its nearest fp32 is the tie itself
    K = _f32([[1 + U8], [1 + U8], [1 + U8 + 2.0 ** -23]])
    t = oracle.OracleTree(1, 3, 2, summary="bf16").build(K, 3)
    assert t.levels[0][0, 0] == 1.0


@pytest.mark.parametrize("c", [0.375, -2.5, 1 + U7])
def test_constant_keys_stay_exact(c):
    K = _f32(np.full((1000, 4), c))
    t = oracle.OracleTree(4, 7, 3, summary="bf16").build(K, 1000)
    for S in t.levels:
        assert (S == c).all()


def test_every_summary_is_a_bf16_value_within_the_rounding_bound():
    rng = np.random.default_rng(12)
    d, lb, b, N = 8, 5, 3, 4000
    K = _f32(rng.standard_normal((N, d)))
    tb = oracle.OracleTree(d, lb, b, summary="bf16").build(K, N)
    t64 = oracle.OracleTree(d, lb, b).build(K, N)
    M = float(np.abs(K).max())
    for lvl, (Sb, S64) in enumerate(zip(tb.levels, t64.levels)):
        f = Sb.astype(np.float32)
        assert (f.astype(np.float64) == Sb).all()
        assert not (f.view(np.uint32) & 0xFFFF).any()
        # each stored level adds at most half a bf16 unit (2^-8 relative, plus the fp32 step)
        assert np.abs(Sb - S64).max() <= (lvl + 1) * 2.0 ** -8 * M * 1.0001
    # far from the bound on random data: the levels are not simply the exact tree
    assert any((Sb != S64).any() for Sb, S64 in zip(tb.levels, t64.levels))


@pytest.mark.parametrize("lb,b", [(4, 2), (3, 3), (16, 4), (1, 5)])
def test_append_equals_rebuild_exactly(lb, b):
    rng = np.random.default_rng(40 + lb + b)
    d, cap = 6, 2500
    K = _f32(rng.standard_normal((cap, d)))
    t = oracle.OracleTree(d, lb, b, summary="bf16").build(K, 1)
    N = 1
    while N < cap:
        N = min(cap, N + int(rng.choice([1, 1, 2, 7, lb, b * lb + 3, 200])))
        t.append(K, N)
        ref = oracle.OracleTree(d, lb, b, summary="bf16").build(K, N)
        assert t.L == ref.L
        for a, r in zip(t.levels, ref.levels):
            np.testing.assert_array_equal(a, r)


def test_bf16_routing_agreement_is_reported():
    # the cost of bf16 storage to routing: the leaf sets of random queries under bf16 and
    # exact summaries (a 32K-token unit of the 32K workload's shape: b 8, 64-token leaves,
    # beam 8).  Not a pin: reported, with a loose floor.
    w = workloads.get("gqa_32k").with_(batch=1, kv_heads=1, q_heads=4, nq=64, needles=0)
    Kn = synth.keys(w)[0, 0]
    Q = synth.to_f64(synth.queries(w)[0]).reshape(-1, w.head_dim)
    t64 = oracle.OracleTree(w.head_dim, w.leaf_block, w.branching).build(Kn, w.seq_len)
    tb = oracle.OracleTree(w.head_dim, w.leaf_block, w.branching, summary="bf16").build(Kn, w.seq_len)
    a = t64.route(Q, w.beam)["leaves"]
    r = tb.route(Q, w.beam)["leaves"]
    same = (np.sort(a, 1) == np.sort(r, 1)).all(1).mean()
    overlap = np.mean([len(set(x) & set(y)) / w.beam for x, y in zip(a, r)])
    print(f"bf16 summaries: identical leaf sets {same:.3f}, mean overlap {overlap:.3f} over {len(Q)} queries")
    assert overlap > 0.5
