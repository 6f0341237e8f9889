"""Bounding-sphere radii and threshold (halfspace) descent through the C ABI.

The set of tokens with q . k >= tau is fixed by the keys alone, so the GPU's descent must
return exactly the oracle's scan of all keys (bit-exact index lists; thresholds are
placed between neighbouring fp64 scores, never on one).  The radii are checked as
geometry: every stored radius bounds every key of its subtree around the GPU's own (fp32)
center, leaf radii are the farthest token, and radii maintained through appends and
decode steps equal a fresh recomputation bit for bit.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from tests.helpers import make_inputs, torch_of
from tests.test_gpu_parity import _wl
from tree_indexed_sparse_build_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from tree_indexed_sparse_build_b200 import zha
    zha.lib()
    return torch.device("cuda:0")


def _setup(w, dev, nq, capacity=None, summary_dtype=None):
    from tree_indexed_sparse_build_b200 import zha
    cap = capacity or w.seq_len
    Qn, Kn, Vn = make_inputs(w, capacity=cap, nq=nq)
    Q, K, V = torch_of(Qn, dev), torch_of(Kn, dev), torch_of(Vn, dev)
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, cap,
                    torch.float32 if w.kv_dtype == "f32" else torch.bfloat16,
                    summary_dtype=summary_dtype or torch.float32)
    return tree, (Qn, Kn, Vn), (Q, K, V)


def _check_radii(w, tree, Kn, N, units=None):
    radii = tree._radii.view(w.units, -1).cpu().numpy().astype(np.float64)
    for u in (range(w.units) if units is None else units):
        b, h = divmod(u, w.kv_heads)
        K64 = synth.to_f64(Kn[b, h, :N])
        for lvl in range(tree.levels + 1):
            cent = tree.level(lvl)[u].float().cpu().numpy().astype(np.float64)
            off = tree.level_offset(lvl)
            rad = radii[u, off:off + cent.shape[0]]
            span = w.leaf_block * w.branching ** lvl
            for i in range(cent.shape[0]):
                far = np.linalg.norm(K64[i * span:min((i + 1) * span, N)] - cent[i], axis=1).max()
                assert far <= rad[i], (lvl, i, far, rad[i])
                if lvl == 0:
                    assert rad[i] <= far * (1 + 1e-6) + 1e-12


SHAPES = [
    (_wl("th_f32_d64_b2", 1, 1, 2, 64, 1000, "f32", 2, 16, 2, 1, 301), 8),
    (_wl("th_bf16_d128_b8", 2, 2, 8, 128, 5000, "bf16", 8, 16, 8, 1, 302), 4),
    (_wl("th_bf16_d128_b16_lb32", 1, 2, 4, 128, 20000, "bf16", 16, 32, 16, 1, 303), 8),
    (_wl("th_f32_d128_b4_lb1", 1, 1, 1, 128, 3000, "f32", 4, 1, 4, 1, 304), 16),
]


@pytest.mark.parametrize("w,nq", SHAPES, ids=lambda x: getattr(x, "name", str(x)))
def test_radii_bound_subtrees(dev, w, nq):
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, nq)
    tree.build(K, w.seq_len)
    tree.attach_radii(K)
    torch.cuda.synchronize()
    _check_radii(w, tree, Kn, w.seq_len, units=[0, w.units - 1])


@pytest.mark.parametrize("w,nq", SHAPES, ids=lambda x: getattr(x, "name", str(x)))
def test_threshold_equals_scan_of_all_keys(dev, w, nq):
    from tree_indexed_sparse_build_b200 import zha
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, nq)
    tree.build(K, w.seq_len)
    tree.attach_radii(K)
    N = w.seq_len
    # thresholds per query between neighbouring scores: the 1st, 10th and 100th largest
    taus = {}
    for k in (1, 10, 100):
        tau = np.empty((w.batch, w.q_heads, nq), np.float32)
        for b in range(w.batch):
            for hq in range(w.q_heads):
                s = synth.to_f64(Kn[b, hq // w.group, :N]) @ synth.to_f64(Qn[b, hq]).T  # [N, nq]
                s = np.sort(s, axis=0)
                tau[b, hq] = ((s[-k] + s[-k - 1]) / 2).astype(np.float32)
        taus[k] = tau
    for k, tau in taus.items():
        toks, cnt, st = tree.threshold(K, Q, torch.from_numpy(tau).to(dev), 256, stats=True)
        torch.cuda.synchronize()
        assert tree.check() == zha.ZHA_OK
        toks, cnt, st = toks.cpu().numpy(), cnt.cpu().numpy(), st.cpu().numpy()
        nodes = sum(tree.level_nodes(lvl) for lvl in range(tree.levels))
        for b in range(w.batch):
            for hq in range(w.q_heads):
                q64 = synth.to_f64(Qn[b, hq])
                for i in range(nq):
                    ref = oracle.threshold_brute(q64[i], Kn[b, hq // w.group], N, float(tau[b, hq, i]))
                    assert cnt[b, hq, i] == len(ref)
                    np.testing.assert_array_equal(toks[b, hq, i, :len(ref)], ref)
                    assert (toks[b, hq, i, len(ref):] == -1).all()
                    assert st[b, hq, i, 0] <= nodes and st[b, hq, i, 1] >= len(ref)


def test_threshold_truncation_and_extremes(dev):
    w, nq = SHAPES[1]
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, nq)
    tree.build(K, w.seq_len)
    tree.attach_radii(K)
    shape = (w.batch, w.q_heads, nq)
    lo = torch.full(shape, -1e30, dtype=torch.float32, device=dev)  # every token
    hi = torch.full(shape, 1e30, dtype=torch.float32, device=dev)   # none
    toks, cnt, _ = tree.threshold(K, Q, hi, 8)
    assert (cnt == 0).all() and (toks == -1).all()
    toks, cnt, _ = tree.threshold(K, Q, lo, 8)
    assert (cnt == w.seq_len).all()
    assert (toks == torch.arange(8, device=dev, dtype=torch.int32)).all()  # the first 8, ascending


def test_threshold_frontier_overflow_is_reported_per_query(dev):
    # 20,000 single-token leaves and a threshold every key passes: the leaf level keeps
    # more than 8,192 nodes, so the descent stops with count -1 for that query only
    w = _wl("th_overflow", 1, 1, 1, 64, 20000, "f32", 8, 1, 8, 2, 305)
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, 2)
    tree.build(K, w.seq_len)
    tree.attach_radii(K)
    tau = torch.tensor([[[-1e30, 1e30]]], dtype=torch.float32, device=dev)
    toks, cnt, _ = tree.threshold(K, Q, tau, 16)
    assert cnt.cpu().tolist() == [[[-1, 0]]]
    assert (toks == -1).all()


@pytest.mark.parametrize("sdt", ["f32", "bf16"])
def test_radii_follow_appends_and_decode_steps(dev, sdt):
    # radii kept current by append and zha_decode_step equal a fresh computation bit for bit
    # (fp32 and bf16 summaries: the centers are the stored summaries either way)
    w = _wl("th_grow", 1, 2, 4, 64, 1024, "f32", 2, 16, 2, 1, 306)
    cap = 1024 + 80
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, 1, capacity=cap,
                                           summary_dtype=torch.bfloat16 if sdt == "bf16" else None)
    tree.build(K, 700)
    tree.attach_radii(K)
    for n in (701, 703, 760, 1024, 1025):  # crosses leaves and adds a level
        tree.append(K, n)
    for n in (1026, 1027):
        tree.decode_step(K, V, n, Q, w.beam, w.scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    kept = tree._radii.clone()
    tree.attach_radii(K)
    torch.cuda.synchronize()
    assert torch.equal(kept, tree._radii)
    _check_radii(w, tree, Kn, 1027)


def test_threshold_prunes_clustered_keys_exactly(dev):
    # keys clustered in leaf blocks: most spheres miss the halfspace, and the found set is
    # still exactly the scan of all keys
    from tree_indexed_sparse_build_b200 import zha
    w = _wl("th_clustered", 1, 2, 8, 128, 8192, "bf16", 8, 64, 8, 4, 307)
    Qn = synth.queries(w)
    Kn = synth.clustered_keys(w, 0.1)
    Q, K = torch_of(Qn, dev), torch_of(Kn, dev)
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, w.seq_len, torch.bfloat16)
    tree.build(K, w.seq_len)
    tree.attach_radii(K)
    tau = np.empty((1, w.q_heads, 4), np.float32)
    for hq in range(w.q_heads):
        s = np.sort(synth.to_f64(Kn[0, hq // w.group]) @ synth.to_f64(Qn[0, hq]).T, axis=0)
        tau[0, hq] = ((s[-64] + s[-65]) / 2).astype(np.float32)
    toks, cnt, st = tree.threshold(K, Q, torch.from_numpy(tau).to(dev), 128, stats=True)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    toks, cnt, st = toks.cpu().numpy(), cnt.cpu().numpy(), st.cpu().numpy()
    for hq in range(w.q_heads):
        for i in range(4):
            ref = oracle.threshold_brute(synth.to_f64(Qn[0, hq, i]), Kn[0, hq // w.group], w.seq_len,
                                         float(tau[0, hq, i]))
            assert cnt[0, hq, i] == len(ref) == 64
            np.testing.assert_array_equal(toks[0, hq, i, :64], ref)
    assert st[..., 1].mean() < 0.25 * w.seq_len  # most leaves pruned
