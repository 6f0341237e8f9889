"""CUDA path (through the C ABI) against the fp64 oracle, on seeded inputs.

Bars: summaries within 1e-6 normwise relative error per node; leaf sets
bit-exact for every query whose fp64 beam margins exceed 1e-3 * |score| at all
levels (other queries: reported rate, and the GPU set must still be a valid
beam result shape); attention within 1e-5 max-abs (fp32 cache, fp32 output)
or 2e-2 relative L2 (bf16 cache, bf16 output) against fp64.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from tests.helpers import make_inputs, oracle_tree, out_to_f64, rel_l2, summary_rel_err, torch_of
from tree_indexed_sparse_build_b200 import synth
from tree_indexed_sparse_build_b200.workloads import Workload

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from tree_indexed_sparse_build_b200 import zha
    zha.lib()
    return torch.device("cuda:0")


def _wl(name, batch, kvh, qh, d, N, dt, b, lb, beam, nq, seed, out=None):
    return Workload(name=name, batch=batch, kv_heads=kvh, q_heads=qh, head_dim=d, seq_len=N,
                    kv_dtype=dt, branching=b, leaf_block=lb, beam=beam, nq=nq,
                    out_dtype=out or ("f32" if dt == "f32" else "bf16"), seed=seed)


# Small shapes that span several CTAs, ragged tails and every kernel variant.
CASES = [
    _wl("f32_d64_b2", 1, 1, 1, 64, 1000, "f32", 2, 16, 2, 16, 101),
    _wl("bf16_d128_b8_gqa", 2, 2, 8, 128, 5000, "bf16", 8, 64, 8, 1, 102),
    _wl("bf16_d128_b16_splits", 2, 2, 8, 128, 9000, "bf16", 16, 32, 16, 1, 103),
    _wl("bf16_d128_b8_lb4", 1, 2, 16, 128, 20001, "bf16", 8, 4, 8, 2, 104),
    _wl("bf16_d128_b4_nq", 1, 2, 4, 128, 3000, "bf16", 4, 16, 4, 8, 105),
    _wl("bf16_d64_b3", 1, 3, 3, 64, 777, "bf16", 3, 5, 3, 4, 106),
    _wl("f32_d128_b5", 2, 1, 2, 128, 1234, "f32", 5, 7, 6, 3, 107),
    _wl("f32_d64_b2_lb1", 1, 1, 2, 64, 300, "f32", 2, 1, 5, 4, 108),
    # > 2 queries per SM: one warp per query, several queries per CTA
    _wl("bf16_d128_narrow", 2, 2, 8, 128, 6000, "bf16", 8, 16, 8, 32, 111),
    _wl("f32_d64_narrow", 1, 2, 4, 64, 3000, "f32", 4, 8, 5, 80, 113),
    # enough queries that a few splits per query fill the GPU: merged inside a cluster
    _wl("bf16_d128_cluster", 4, 2, 8, 128, 9000, "bf16", 16, 32, 16, 4, 114),
    _wl("f32_d64_cluster", 2, 2, 8, 64, 3000, "f32", 4, 16, 8, 4, 115),
    # widest level (beam * b = 512 rows) too large to stage: register-batched route kernel
    _wl("bf16_d128_regpath", 1, 1, 2, 128, 20000, "bf16", 8, 4, 64, 2, 112),
    # many queries with short leaf lists (the 1M shape): narrow launch, attention fused
    _wl("bf16_d128_narrow_lb4", 1, 2, 16, 128, 20001, "bf16", 8, 4, 8, 32, 116),
    # odd number of queries (the last CTA is partly empty), d 64, one warp per query
    _wl("bf16_d64_narrow_odd", 1, 3, 3, 64, 2000, "bf16", 4, 8, 4, 101, 117),
]


def _tdt(w):
    return torch.float32 if w.kv_dtype == "f32" else torch.bfloat16


def _setup(w, dev, capacity=None, nq=None, summary_dtype=None):
    from tree_indexed_sparse_build_b200 import zha
    cap = capacity or w.seq_len
    Qn, Kn, Vn = make_inputs(w, capacity=cap, nq=nq)
    Q, K, V = torch_of(Qn, dev), torch_of(Kn, dev), torch_of(Vn, dev)
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, cap, _tdt(w),
                    summary_dtype=summary_dtype or torch.float32)
    return tree, (Qn, Kn, Vn), (Q, K, V)


def _check_levels(tree, w, Kn, N, units=None):
    torch.cuda.synchronize()
    worst = 0.0
    for u in (range(w.units) if units is None else units):
        ot = oracle_tree(w, Kn, u, N)
        assert tree.levels == ot.L
        for lvl in range(ot.L + 1):
            assert tree.level_nodes(lvl) == ot.levels[lvl].shape[0]
            got = tree.level(lvl)[u].cpu().numpy()
            worst = max(worst, summary_rel_err(got, ot.levels[lvl]))
    assert worst <= 1e-6, f"summary rel err {worst}"
    return worst


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_build_summaries(dev, w):
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev)
    tree.build(K, w.seq_len)
    _check_levels(tree, w, Kn, w.seq_len)
    assert tree.check() == 0


@pytest.mark.parametrize("w", CASES[:6], ids=lambda w: w.name)
def test_append_matches_rebuild_oracle(dev, w):
    cap = w.seq_len + 3 * w.leaf_block * w.branching + 17
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, capacity=cap)
    N = w.seq_len // 3
    tree.build(K, N)
    for step in [1, 1, 2, w.leaf_block, w.leaf_block * w.branching + 5, 1]:
        N = min(cap, N + step)
        tree.append(K, N)
        _check_levels(tree, w, Kn, N, units=[0, w.units - 1])
    # grow all the way to capacity (crosses at least one new level on small trees)
    tree.append(K, cap)
    _check_levels(tree, w, Kn, cap)


def test_append_grows_depth(dev):
    # 64 leaves of 16 = b^6 exactly full, then one token more: L 6 -> 7.
    w = _wl("grow", 1, 1, 1, 64, 1024, "f32", 2, 16, 2, 4, 109)
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, capacity=1024 + 40)
    tree.build(K, 1024)
    assert tree.levels == 6
    tree.append(K, 1025)
    assert tree.levels == 7
    _check_levels(tree, w, Kn, 1025)
    tree.append(K, 1064)
    _check_levels(tree, w, Kn, 1064)


def _route_compare(tree, w, Qn, Kn, idx, trace, N, units=None, summary="f64"):
    """Exact match on well-conditioned queries; returns (n_checked, n_ill, n_ill_mismatch).
    summary: the oracle's summary storage ("bf16" for trees with bf16 summaries)."""
    idx = idx.cpu().numpy()
    trace = trace.cpu().numpy() if trace is not None else None
    g = w.group
    checked = ill = ill_bad = 0
    for u in (range(w.units) if units is None else units):
        b, h = divmod(u, w.kv_heads)
        ot = oracle_tree(w, Kn, u, N, summary=summary)
        flat = ot.flat()
        for hq in range(h * g, h * g + g):
            q64 = synth.to_f64(Qn[b, hq])
            res = ot.route(q64, w.beam, flat=flat)
            ok = oracle.well_conditioned(res["bounds"])
            got = idx[b, hq]
            for i in range(q64.shape[0]):
                if ok[i]:
                    np.testing.assert_array_equal(got[i], res["leaves"][i])
                    if trace is not None:
                        np.testing.assert_array_equal(trace[b, hq, i], res["survivors"][i])
                    checked += 1
                else:
                    ill += 1
                    valid = got[i][got[i] >= 0]
                    assert len(valid) == min(w.beam, ot.levels[0].shape[0])
                    assert (np.diff(valid) > 0).all() and valid.max() < ot.levels[0].shape[0]
                    ill_bad += int(not np.array_equal(got[i], res["leaves"][i]))
    return checked, ill, ill_bad


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_route_matches_oracle(dev, w):
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev)
    tree.build(K, w.seq_len)
    idx, sc, tr = tree.route(Q, w.beam, scores=True, trace=True)
    checked, ill, bad = _route_compare(tree, w, Qn, Kn, idx, tr, w.seq_len)
    assert checked > 0
    # queries whose beam boundary is within the margin rule are only reported
    print(f"{w.name}: well-conditioned {checked}, ill {ill}, ill mismatches {bad}")
    # leaf scores are q . S0[leaf] in fp32
    idx_n = idx.cpu().numpy()
    sc_n = sc.cpu().numpy()
    u0 = oracle_tree(w, Kn, 0, w.seq_len)
    q0 = synth.to_f64(Qn[0, 0])
    for i in range(q0.shape[0]):
        lv = idx_n[0, 0, i][idx_n[0, 0, i] >= 0]
        ref = u0.levels[0][lv] @ q0[i]
        np.testing.assert_allclose(sc_n[0, 0, i][:len(lv)], ref, rtol=1e-4, atol=1e-4)


def _attend_check(w, Qn, Kn, Vn, O, leaves, N):
    got = out_to_f64(O)
    worst_abs = worst_rel = 0.0
    for b in range(w.batch):
        for hq in range(w.q_heads):
            h = hq // w.group
            q64 = synth.to_f64(Qn[b, hq])
            for i in range(q64.shape[0]):
                ref, _ = oracle.attend(q64[i], Kn[b, h], Vn[b, h], N, w.leaf_block,
                                       leaves[b, hq, i], w.scale)
                worst_abs = max(worst_abs, float(np.abs(got[b, hq, i] - ref).max()))
                worst_rel = max(worst_rel, rel_l2(got[b, hq, i], ref))
    if w.kv_dtype == "f32" and w.out_dtype == "f32":
        assert worst_abs <= 1e-5, f"max-abs {worst_abs}"
    else:
        assert worst_rel <= 2e-2, f"rel L2 {worst_rel}"
    return worst_abs, worst_rel


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_attend_on_oracle_leaves(dev, w):
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev)
    tree.build(K, w.seq_len)
    leaves = np.empty((w.batch, w.q_heads, Qn.shape[2], w.beam), np.int64)
    for u in range(w.units):
        b, h = divmod(u, w.kv_heads)
        ot = oracle_tree(w, Kn, u, w.seq_len)
        for hq in range(h * w.group, (h + 1) * w.group):
            leaves[b, hq] = ot.route(synth.to_f64(Qn[b, hq]), w.beam)["leaves"]
    idx = torch.from_numpy(leaves.astype(np.int32)).to(dev)
    odt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    O = tree.attend(Q, K, V, idx, w.beam, w.scale, out_dtype=odt)
    torch.cuda.synchronize()
    assert tree.check() == 0
    _attend_check(w, Qn, Kn, Vn, O, leaves, w.seq_len)


@pytest.mark.parametrize("w", CASES[:4], ids=lambda w: w.name)
def test_full_beam_equals_dense(dev, w):
    # beam >= n0 keeps every leaf, so the sparse path must equal dense attention.
    w = w.with_(seq_len=min(w.seq_len, 600))
    n0 = -(-w.seq_len // w.leaf_block)
    if n0 > 1024 or n0 * w.branching > 4096:
        pytest.skip("beam bound")
    w = w.with_(beam=n0)
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev)
    tree.build(K, w.seq_len)
    idx, _, _ = tree.route(Q, w.beam)
    assert (torch.sort(idx, dim=-1).values == torch.arange(n0, device=dev, dtype=torch.int32)).all()
    odt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    O = tree.attend(Q, K, V, idx, w.beam, w.scale, out_dtype=odt)
    got = out_to_f64(O)
    for b in range(w.batch):
        for hq in range(w.q_heads):
            q64 = synth.to_f64(Qn[b, hq])
            for i in range(q64.shape[0]):
                ref = oracle.dense(q64[i], Kn[b, hq // w.group], Vn[b, hq // w.group], w.seq_len,
                                   w.scale)
                if w.out_dtype == "f32":
                    assert np.abs(got[b, hq, i] - ref).max() <= 1e-5
                else:
                    assert rel_l2(got[b, hq, i], ref) <= 2e-2


def test_single_token_and_padding(dev):
    from tree_indexed_sparse_build_b200 import zha
    w = _wl("one", 1, 1, 1, 64, 1, "f32", 2, 4, 3, 2, 110)
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, capacity=8)
    tree.build(K, 1)
    assert tree.levels == 1
    idx, _, _ = tree.route(Q, 3)
    assert idx.cpu().numpy().tolist() == [[[[0, -1, -1], [0, -1, -1]]]]
    O = tree.attend(Q, K, V, idx, 3, w.scale, out_dtype=torch.float32)
    np.testing.assert_array_equal(O.cpu().numpy()[0, 0], np.tile(Vn[0, 0, 0], (2, 1)))
    assert tree.check() == zha.ZHA_OK


def test_bad_leaf_index_is_reported(dev):
    from tree_indexed_sparse_build_b200 import zha
    w = CASES[0]
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev)
    tree.build(K, w.seq_len)
    idx, _, _ = tree.route(Q, w.beam)
    idx[0, 0, 0, 0] = 10_000_000
    O = tree.attend(Q, K, V, idx, w.beam, w.scale, out_dtype=torch.float32)
    assert tree.check() == zha.ZHA_ERR_DEVICE
    assert torch.isfinite(O).all()
    assert tree.check() == zha.ZHA_OK  # the word was cleared


def test_host_errors_leave_tree_usable(dev):
    from tree_indexed_sparse_build_b200 import zha
    w = CASES[1]
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev)
    with pytest.raises(zha.ZhaError) as e:
        tree.build(K, w.seq_len + 1)
    assert e.value.status == zha.ZHA_ERR_CAPACITY
    with pytest.raises(zha.ZhaError) as e:
        tree.route(Q, w.beam)  # empty tree
    assert e.value.status == zha.ZHA_ERR_INVALID_ARG
    tree.build(K, w.seq_len)
    with pytest.raises(zha.ZhaError) as e:
        tree.append(K, w.seq_len - 1)
    assert e.value.status == zha.ZHA_ERR_INVALID_ARG
    with pytest.raises(zha.ZhaError):
        tree.route(Q, 0)
    with pytest.raises(zha.ZhaError) as e:
        tree.route(Q, 1024)  # beam * b > 4096
    assert e.value.status == zha.ZHA_ERR_UNSUPPORTED
    Q3 = Q[:, :3].contiguous()
    with pytest.raises(zha.ZhaError):  # 3 heads % 2 kv heads
        zha.zha_route(tree.handle, Q3, w.beam, torch.empty(Q3.shape[:3] + (w.beam,), dtype=torch.int32, device=dev))
    with pytest.raises(ValueError):  # a leaf-index buffer too small for the queries: refused
        zha.zha_route(tree.handle, Q, w.beam, torch.empty(1, dtype=torch.int32, device=dev))
    idx, _, _ = tree.route(Q[:, :, :0].contiguous(), w.beam)  # nq == 0 is a no-op
    assert idx.numel() == 0
    idx, _, _ = tree.route(Q, w.beam)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK


@pytest.mark.parametrize("kv", ["f32", "bf16"])
def test_largest_beam_keeps_every_leaf(dev, kv):
    # beam 1024 with beam * b = 4096 (the limits): a tree of 1,000 leaves keeps them all, so
    # routing returns every leaf in order (then -1) and attention equals dense attention over
    # the whole cache.  The levels above the leaves are kept whole; the 1,000 leaf rows are
    # too many to stage, so they are scored by the register route and attended by a second
    # launch
    from tree_indexed_sparse_build_b200 import zha
    w = _wl(f"beam1024_{kv}", 1, 1, 2, 64, 3000, kv, 4, 3, 1024, 2, 118)
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev)
    tree.build(K, w.seq_len)
    n0 = tree.level_nodes(0)
    assert n0 == 1000
    idx, _, _ = tree.route(Q, w.beam)
    expect = torch.cat([torch.arange(n0, dtype=torch.int32), torch.full((w.beam - n0,), -1, dtype=torch.int32)])
    assert (idx.cpu() == expect).all()
    odt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    O, didx = tree.decode(Q, K, V, w.beam, w.scale, out_dtype=odt)[:2]
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert torch.equal(didx, idx)
    got = out_to_f64(O)
    for hq in range(w.q_heads):
        q64 = synth.to_f64(Qn[0, hq])
        for i in range(q64.shape[0]):
            ref = oracle.dense(q64[i], Kn[0, 0], Vn[0, 0], w.seq_len, w.scale)
            if kv == "f32":
                assert np.abs(got[0, hq, i] - ref).max() <= 1e-5
            else:
                assert rel_l2(got[0, hq, i], ref) <= 2e-2
