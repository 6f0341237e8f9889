"""Pins for the fp64 oracle, each against something other than the oracle itself.

Sources of the definitions: "Subquadratic Attention with a Hierarchical
Tree-Structured Indexer" (ZHA), abstract (recursively compressed key summaries,
top-down traversal, growing depth, final attention); "ALHR" news item,
technical features (static tree).  Pins used: a hand-worked tree
(tests/golden/hand_tree.json), closed forms (token means of full subtrees,
constant keys, q = 0 ties, single-token attention), exact append == rebuild,
brute-force subset enumeration of every beam step, a library sort on monotone
trees, a library softmax for beam >= n0, and planted needles.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy.special import softmax

import oracle
from tree_indexed_sparse_build_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_tree.json")


def _f32(x):
    return np.ascontiguousarray(np.asarray(x, np.float32))


# ---------------------------------------------------------------- hand-worked tree

@pytest.fixture(scope="module")
def hand():
    with open(GOLDEN) as f:
        return json.load(f)


def test_hand_tree_levels(hand):
    K = _f32(hand["K"])
    t = oracle.OracleTree(hand["d"], hand["leaf_block"], hand["branching"]).build(K, hand["N"])
    assert t.L == len(hand["levels"]) - 1
    for got, want in zip(t.levels, hand["levels"]):
        np.testing.assert_array_equal(got, np.asarray(want, np.float64))
    # unweighted mean of existing children, not the token mean
    assert not np.allclose(t.levels[-1][0], hand["token_mean"])


def test_hand_tree_routes(hand):
    K = _f32(hand["K"])
    t = oracle.OracleTree(hand["d"], hand["leaf_block"], hand["branching"]).build(K, hand["N"])
    for r in hand["routes"]:
        res = t.route(np.asarray([r["q"]], np.float64), r["beam"])
        leaves = res["leaves"][0]
        assert leaves[leaves >= 0].tolist() == r["leaves"]
        if "leaf_level_bounds" in r:
            np.testing.assert_array_equal(res["bounds"][0, -1], r["leaf_level_bounds"])


def test_hand_tree_attend(hand):
    K, V = _f32(hand["K"]), _f32(hand["V"])
    a = hand["attend"]
    t = oracle.OracleTree(hand["d"], hand["leaf_block"], hand["branching"]).build(K, hand["N"])
    q = np.asarray(a["q"], np.float64)
    leaves = t.route(q[None], a["beam"])["leaves"][0]
    scale = 1.0 / math.sqrt(a["scale_inv_sq"])
    o, ntok = oracle.attend(q, K, V, hand["N"], hand["leaf_block"], leaves, scale)
    assert ntok == len(a["tokens"])
    w = [math.exp(scale * s) for s in a["qk"]]
    want = sum(wi * np.asarray(hand["V"][tk], np.float64) for wi, tk in zip(w, a["tokens"])) / sum(w)
    np.testing.assert_allclose(o, want, rtol=1e-15, atol=1e-15)


def test_hand_tree_append(hand):
    K = _f32(hand["K"])
    ap = hand["append"]
    t = oracle.OracleTree(hand["d"], hand["leaf_block"], hand["branching"]).build(K, ap["from_N"])
    for got, want in zip(t.levels, ap["levels_at_from"]):
        np.testing.assert_array_equal(got, np.asarray(want, np.float64))
    t.append(K, ap["to_N"])
    assert t.L == len(hand["levels"]) - 1
    for got, want in zip(t.levels, hand["levels"]):
        np.testing.assert_array_equal(got, np.asarray(want, np.float64))


# ---------------------------------------------------------------- tree shape

@pytest.mark.parametrize("N,lb,b,n0,L", [
    (1024, 16, 2, 64, 6), (32768, 64, 8, 512, 3), (131072, 32, 16, 4096, 3),
    (1048576, 4, 8, 262144, 6), (262144, 16, 4, 16384, 7),
    (131072 + 64, 32, 16, 4098, 4), (262144 + 4096, 16, 4, 16640, 8),
    (1, 16, 2, 1, 1), (17, 16, 2, 2, 1), (33, 16, 2, 3, 2)])
def test_levels_and_leaves(N, lb, b, n0, L):
    assert oracle.num_leaves(N, lb) == n0
    assert oracle.num_levels(n0, b) == L


# ---------------------------------------------------------------- summaries

@pytest.mark.parametrize("lb,b,L", [(4, 2, 5), (3, 3, 3), (16, 4, 3), (1, 8, 2)])
def test_full_subtrees_equal_token_means(lb, b, L):
    rng = np.random.default_rng(1)
    d = 8
    N = lb * b ** L
    K = _f32(rng.standard_normal((N, d)))
    t = oracle.OracleTree(d, lb, b).build(K, N)
    assert t.L == L
    K64 = K.astype(np.float64)
    for lvl, S in enumerate(t.levels):
        span = lb * b ** lvl
        want = K64.reshape(N // span, span, d).mean(axis=1)
        np.testing.assert_allclose(S, want, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(t.levels[-1][0], K64.mean(axis=0), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("N", [1, 5, 97, 1000])
def test_constant_keys(N):
    d = 4
    c = np.array([0.5, -1.25, 3.0, 0.0], np.float32)
    K = np.tile(c, (N, 1))
    t = oracle.OracleTree(d, 7, 3).build(K, N)
    for S in t.levels:
        np.testing.assert_array_equal(S, np.tile(c.astype(np.float64), (S.shape[0], 1)))


def test_bf16_input_widening():
    # bf16 bit patterns of 1.0, -2.5, 0.15625 and the fp32 widening used by the oracle
    bits = np.array([[0x3F80, 0xC020, 0x3E20, 0x0000]], np.uint16)
    t = oracle.OracleTree(4, 1, 2).build(bits, 1)
    np.testing.assert_array_equal(t.levels[0][0], [1.0, -2.5, 0.15625, 0.0])


# ---------------------------------------------------------------- append

@pytest.mark.parametrize("lb,b", [(4, 2), (3, 3), (16, 4), (1, 5), (32, 16)])
def test_append_equals_rebuild(lb, b):
    rng = np.random.default_rng(2 + lb + b)
    d = 6
    cap = 3000
    K = _f32(rng.standard_normal((cap, d)))
    t = oracle.OracleTree(d, lb, b).build(K, 1)
    N = 1
    while N < cap:
        step = int(rng.choice([1, 1, 2, 7, lb, b * lb + 3, 200]))
        N = min(cap, N + step)
        t.append(K, N)
        ref = oracle.OracleTree(d, lb, b).build(K, N)
        assert t.L == ref.L
        for a, r in zip(t.levels, ref.levels):
            np.testing.assert_array_equal(a, r)


def test_append_dyadic_matches_token_means():
    # Dyadic inputs: every mean over a power-of-two count is exact in fp64, so the
    # appended tree's full subtrees equal the exact token means bit for bit.
    rng = np.random.default_rng(3)
    d, lb, b = 4, 4, 2
    cap = lb * b ** 6
    K = _f32(rng.integers(-8, 9, size=(cap, d)) / 8.0)
    t = oracle.OracleTree(d, lb, b).build(K, 5)
    for N in [6, 17, 64, 65, 200, cap]:
        t.append(K, N)
    K64 = K.astype(np.float64)
    for lvl, S in enumerate(t.levels):
        span = lb * b ** lvl
        np.testing.assert_array_equal(S, K64.reshape(cap // span, span, d).mean(axis=1))


# ---------------------------------------------------------------- routing

def _score(q, row):
    # q . row summed in index order, the same IEEE operations as the oracle's loop
    acc = 0.0
    for a, c in zip(q.tolist(), row.tolist()):
        acc += a * c
    return acc


def _closed_subsets(cands, scores, keep):
    """All keep-subsets whose every member beats every non-member under (score desc, index asc)."""
    out = []
    for sub in itertools.combinations(range(len(cands)), keep):
        s = set(sub)
        ok = all((scores[i] > scores[j]) or (scores[i] == scores[j] and cands[i] < cands[j])
                 for i in s for j in range(len(cands)) if j not in s)
        if ok:
            out.append(sorted(cands[i] for i in sub))
    return out


@pytest.mark.parametrize("b", [2, 3])
@pytest.mark.parametrize("kind", ["gauss", "ties"])
def test_route_bruteforce_each_level(b, kind):
    rng = np.random.default_rng(10 * b + (kind == "ties"))
    d = 3
    for trial in range(40):
        lb = int(rng.integers(1, 4))
        L = int(rng.integers(1, 5))
        n0 = int(rng.integers(b ** (L - 1) + 1, b ** L + 1))
        N = (n0 - 1) * lb + int(rng.integers(1, lb + 1))
        beam = int(rng.integers(1, 4))
        if kind == "ties":
            K = _f32(rng.integers(-1, 2, size=(N, d)))
            Q = rng.integers(-1, 2, size=(4, d)).astype(np.float64)
        else:
            K = _f32(rng.standard_normal((N, d)))
            Q = rng.standard_normal((4, d))
        t = oracle.OracleTree(d, lb, b).build(K, N)
        assert t.L == L
        res = t.route(Q, beam)
        for qi in range(Q.shape[0]):
            parents = [0]
            for li, lvl in enumerate(range(L - 1, -1, -1)):
                n = t.levels[lvl].shape[0]
                cands = [c for p in parents for c in range(b * p, min(b * p + b, n))]
                scores = [_score(Q[qi], t.levels[lvl][c]) for c in cands]
                keep = min(beam, len(cands))
                closed = _closed_subsets(cands, scores, keep)
                assert len(closed) == 1  # the (score, -index) order is total
                sv = res["survivors"][qi, li]
                assert sv[sv >= 0].tolist() == closed[0]
                assert res["ncand"][qi, li] == len(cands)
                if len(cands) > beam:
                    order = sorted(range(len(cands)), key=lambda i: (-scores[i], cands[i]))
                    assert res["bounds"][qi, li, 0] == scores[order[beam - 1]]
                    assert res["bounds"][qi, li, 1] == scores[order[beam]]
                else:
                    assert np.isnan(res["bounds"][qi, li]).all()
                parents = closed[0]
            lv = res["leaves"][qi]
            assert lv[lv >= 0].tolist() == parents


def test_q_zero_takes_leftmost_leaves_and_uniform_mean():
    rng = np.random.default_rng(4)
    d, lb, b, N, beam = 8, 5, 3, 203, 4
    K = _f32(rng.standard_normal((N, d)))
    V = _f32(rng.standard_normal((N, d)))
    t = oracle.OracleTree(d, lb, b).build(K, N)
    q = np.zeros(d)
    leaves = t.route(q[None], beam)["leaves"][0]
    assert leaves.tolist() == list(range(beam))
    o, ntok = oracle.attend(q, K, V, N, lb, leaves, 0.3)
    assert ntok == beam * lb
    np.testing.assert_allclose(o, V[:beam * lb].astype(np.float64).mean(axis=0), rtol=1e-13,
                               atol=1e-14)


@pytest.mark.parametrize("lb,b,N,beam", [(4, 2, 509, 3), (3, 4, 1000, 5), (16, 8, 4099, 8)])
def test_monotone_tree_is_global_top_b(lb, b, N, beam):
    rng = np.random.default_rng(5)
    d = 5
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    c = np.sort(rng.uniform(-3, 3, size=N))
    K = _f32(c[:, None] * u[None, :])
    t = oracle.OracleTree(d, lb, b).build(K, N)
    q = 2.0 * u.astype(np.float32).astype(np.float64)
    leaves = t.route(q[None], beam)["leaves"][0]
    leaf_scores = t.levels[0] @ q
    top = np.sort(np.argsort(-leaf_scores, kind="stable")[:beam])
    assert leaves.tolist() == top.tolist()


@pytest.mark.parametrize("lb,b,N", [(4, 2, 301), (1, 3, 50), (16, 16, 1000)])
def test_full_beam_is_dense_attention(lb, b, N):
    rng = np.random.default_rng(6)
    d = 16
    K = _f32(rng.standard_normal((N, d)))
    V = _f32(rng.standard_normal((N, d)))
    Q = rng.standard_normal((3, d))
    scale = d ** -0.5
    t = oracle.OracleTree(d, lb, b).build(K, N)
    n0 = t.levels[0].shape[0]
    res = t.route(Q, n0)
    for qi in range(3):
        assert sorted(res["leaves"][qi].tolist()) == list(range(n0))
        o, ntok = oracle.attend(Q[qi], K, V, N, lb, res["leaves"][qi], scale)
        assert ntok == N
        dn = oracle.dense(Q[qi], K, V, N, scale)
        np.testing.assert_allclose(o, dn, rtol=1e-12, atol=1e-13)
        p = softmax(scale * (K.astype(np.float64) @ Q[qi]))
        np.testing.assert_allclose(dn, p @ V.astype(np.float64), rtol=1e-12, atol=1e-13)


def test_single_token_attention_is_its_value():
    rng = np.random.default_rng(7)
    d, N = 8, 37
    K = _f32(rng.standard_normal((N, d)))
    V = _f32(rng.standard_normal((N, d)))
    t = oracle.OracleTree(d, 1, 2).build(K, N)
    q = rng.standard_normal(d)
    leaves = t.route(q[None], 1)["leaves"][0]
    o, ntok = oracle.attend(q, K, V, N, 1, leaves, 0.7)
    assert ntok == 1
    np.testing.assert_array_equal(o, V[leaves[0]].astype(np.float64))


# ---------------------------------------------------------------- append buffer

def test_buffered_attention_over_one_routed_leaf_and_the_rest_is_dense():
    # routed prefix = the first leaf (one leaf, kept whatever the query), buffer = every
    # later token: the union is the whole cache, so the result is a library softmax over all
    rng = np.random.default_rng(21)
    d, lb, N = 8, 4, 203
    K = _f32(rng.standard_normal((N, d)))
    V = _f32(rng.standard_normal((N, d)))
    q = rng.standard_normal(d)
    t = oracle.OracleTree(d, lb, 2).build(K, lb)
    leaves = t.route(q[None], 1)["leaves"][0]
    np.testing.assert_array_equal(leaves, [0])
    o, ntok = oracle.attend_buffered(q, K, V, leaves, lb, N, lb, 0.3)
    assert ntok == N
    w = softmax(0.3 * (K.astype(np.float64) @ q))
    np.testing.assert_allclose(o, w @ V.astype(np.float64), rtol=1e-12, atol=1e-14)


def test_buffered_attention_is_the_union_of_leaf_and_buffer_tokens():
    rng = np.random.default_rng(22)
    d, lb, b, n_routed, n_tokens = 6, 5, 3, 400, 437
    K = _f32(rng.standard_normal((n_tokens, d)))
    V = _f32(rng.standard_normal((n_tokens, d)))
    q = rng.standard_normal(d)
    t = oracle.OracleTree(d, lb, b).build(K, n_routed)
    leaves = t.route(q[None], 4)["leaves"][0]
    o, ntok = oracle.attend_buffered(q, K, V, leaves, n_routed, n_tokens, lb, 0.5)
    tok = np.concatenate([np.arange(l * lb, l * lb + lb) for l in leaves] + [np.arange(n_routed, n_tokens)])
    assert ntok == len(tok) == 4 * lb + 37
    w = softmax(0.5 * (K[tok].astype(np.float64) @ q))
    np.testing.assert_allclose(o, w @ V[tok].astype(np.float64), rtol=1e-12, atol=1e-14)
    # an empty buffer is the plain attention over the routed leaves
    o0, _ = oracle.attend_buffered(q, K, V, leaves, n_routed, n_routed, lb, 0.5)
    np.testing.assert_array_equal(o0, oracle.attend(q, K, V, n_routed, lb, leaves, 0.5)[0])


@pytest.mark.parametrize("lb,b,N", [(16, 2, 1024), (4, 8, 40000), (64, 8, 32768)])
def test_needle_on_quiet_background_is_retrieved(lb, b, N):
    rng = np.random.default_rng(8)
    d = 32
    K = _f32(1e-6 * rng.standard_normal((N, d)))
    q = rng.standard_normal(d)
    qhat = q / np.linalg.norm(q)
    for pos in rng.integers(0, N, size=5):
        Kp = K.copy()
        Kp[pos] = qhat
        t = oracle.OracleTree(d, lb, b).build(Kp, N)
        leaves = t.route(q[None], 1)["leaves"][0]
        assert leaves[0] == pos // lb


def test_route_pads_when_fewer_leaves_than_beam():
    rng = np.random.default_rng(9)
    d, lb, b, N = 4, 8, 4, 20  # 3 leaves
    K = _f32(rng.standard_normal((N, d)))
    t = oracle.OracleTree(d, lb, b).build(K, N)
    res = t.route(rng.standard_normal((2, d)), 5)
    assert (res["leaves"][:, :3] == np.arange(3)).all()
    assert (res["leaves"][:, 3:] == -1).all()


# ---------------------------------------------------------------- threshold descent
# Bounding spheres centered on the summaries ("Louver" explainer, index design): a leaf's
# radius covers its tokens, a parent's covers its children's spheres; a node is expanded
# iff q . c + ||q|| r >= tau, the surviving leaves' tokens are checked exactly.  Pinned
# against direct numpy geometry and a scan of all keys.

def _subtree_tokens(lvl, i, b, lb, N):
    span = lb * b ** lvl
    return i * span, min((i + 1) * span, N)


@pytest.mark.parametrize("b,lb,N", [(2, 4, 37), (3, 5, 200), (8, 16, 1000)])
def test_radii_bound_every_key_and_leaf_radius_is_farthest_token(b, lb, N):
    rng = np.random.default_rng(b * 100 + lb)
    d = 8
    K = rng.standard_normal((N, d)).astype(np.float32)
    t = oracle.OracleTree(d, lb, b).build(K, N)
    radii = t.radii(K)
    K64 = K.astype(np.float64)
    for lvl, (cent, rad) in enumerate(zip(t.levels, radii)):
        for i in range(cent.shape[0]):
            t0, t1 = _subtree_tokens(lvl, i, b, lb, N)
            far = np.linalg.norm(K64[t0:t1] - cent[i], axis=1).max()
            assert far <= rad[i] * (1 + 1e-12) + 1e-15
            if lvl == 0:
                assert rad[i] == pytest.approx(far, rel=1e-12, abs=1e-15)


def test_radii_hand_example():
    # keys (0,0), (4,0), (0,3), (0,3) with leaf block 2, b = 2:
    # leaf 0 = mean of (0,0), (4,0) = (2,0), radius 2; leaf 1 = (0,3), radius 0;
    # root = mean of leaves = (1, 1.5); radius = max(||(2,0)-(1,1.5)|| + 2, ||(0,3)-(1,1.5)|| + 0)
    #      = max(sqrt(3.25) + 2, sqrt(3.25)) = sqrt(3.25) + 2
    K = np.array([[0, 0], [4, 0], [0, 3], [0, 3]], np.float32)
    t = oracle.OracleTree(2, 2, 2).build(K, 4)
    r = t.radii(K)
    assert r[0].tolist() == [2.0, 0.0]
    assert r[1][0] == pytest.approx(np.sqrt(3.25) + 2.0, rel=1e-15)
    # tau = 2.5 with q = (1, 0): only (4,0) qualifies; leaf 1's sphere (x = 0) is pruned
    toks, tested = t.threshold(K, np.array([1.0, 0.0]), 2.5)
    assert toks.tolist() == [1]
    assert tested == 2  # the two leaves are tested, the root is not scored


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("b,lb,N", [(2, 1, 50), (2, 16, 1024), (3, 7, 500), (8, 4, 3000)])
def test_threshold_descent_equals_scan_of_all_keys(dt, b, lb, N):
    rng = np.random.default_rng(N + b)
    d = 16
    K32 = rng.standard_normal((N, d)).astype(np.float32)
    K = synth.round_to(K32.astype(np.float64), "bf16") if dt == "bf16" else K32
    Kf = synth.to_f64(K)
    t = oracle.OracleTree(d, lb, b).build(K, N)
    radii = t.radii(K)
    for trial in range(6):
        q = rng.standard_normal(d)
        s = np.sort(Kf @ q)
        # thresholds between neighbouring scores (never on one): none, all, a few, many
        taus = [s[-1] + 1.0, s[0] - 1.0] + [(s[-k] + s[-k - 1]) / 2 for k in (1, 5, N // 3)]
        for tau in taus:
            got, tested = t.threshold(K, q, tau, radii=radii)
            np.testing.assert_array_equal(got, oracle.threshold_brute(q, K, N, tau))
            assert tested <= sum(lv.shape[0] for lv in t.levels) - 1


def test_threshold_descent_prunes_clustered_keys():
    # 64 tight clusters of 16 keys (one per leaf) around spread-out centers: a query aimed
    # at one cluster with a threshold only that cluster reaches tests far fewer spheres
    # than the tree has nodes
    rng = np.random.default_rng(7)
    d, lb = 16, 16
    centers = rng.standard_normal((64, d)) * 10
    K = (np.repeat(centers, lb, axis=0) + 0.01 * rng.standard_normal((64 * lb, d))).astype(np.float32)
    t = oracle.OracleTree(d, lb, 2).build(K, K.shape[0])
    q = centers[17] / np.linalg.norm(centers[17])
    tau = q @ centers[17] - 0.5
    got, tested = t.threshold(K, q, tau)
    np.testing.assert_array_equal(got, oracle.threshold_brute(q, K, K.shape[0], tau))
    assert 17 * lb <= got.min() and got.max() < 18 * lb
    assert tested < 0.5 * sum(lv.shape[0] for lv in t.levels)
