"""Trees with bf16-stored summaries, through the C ABI, against the oracle's bf16 mode.

The stored value of a node is fixed by its children's stored values alone (the fp64 mean,
rounded to fp32 and then to bf16, ties to even), and both sides sum in the same order, so
every summary the GPU stores -- built, appended (one-launch path kernel and level passes),
or written by the fused decode step -- must equal the oracle's bit for bit.  Routing
(staged and register kernels, fused decode, causal prefixes) uses the parity bars of the
fp32 trees against the oracle's bf16 tree: exact leaf sets and survivors on queries whose
fp64 margins exceed 1e-3 |score|; attention within 1e-5 max-abs (fp32 cache and output) or
2e-2 relative L2.  Threshold descent stays exact (a scan of all keys).
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from tests.helpers import oracle_tree
from tests.test_gpu_parity import CASES, _attend_check, _route_compare, _setup, _wl
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


def _odt(w):
    return torch.float32 if w.out_dtype == "f32" else torch.bfloat16


def _bit_exact(tree, w, Kn, N, units=None):
    torch.cuda.synchronize()
    for u in (range(w.units) if units is None else units):
        ot = oracle_tree(w, Kn, u, N, summary="bf16")
        assert tree.levels == ot.L
        for lvl in range(ot.L + 1):
            got = tree.level(lvl)[u].float().cpu().numpy().astype(np.float64)
            np.testing.assert_array_equal(got, ot.levels[lvl], err_msg=f"unit {u} level {lvl}")


# fp32 and bf16 caches, d 64 and 128, b 2 .. 16, ragged tails, wide / narrow / register routes
S16_CASES = [CASES[i] for i in (0, 1, 2, 3, 5, 6, 8, 12, 13, 14)]


@pytest.mark.parametrize("w", S16_CASES, ids=lambda w: w.name)
def test_build_is_bit_exact(dev, w):
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, summary_dtype=torch.bfloat16)
    tree.build(K, w.seq_len)
    _bit_exact(tree, w, Kn, w.seq_len, units=[0, w.units - 1])
    assert tree.check() == 0


@pytest.mark.parametrize("w", [CASES[i] for i in (0, 1, 2, 5, 6)], ids=lambda w: w.name)
def test_appends_are_bit_exact(dev, w):
    # small appends take the one-launch path kernel, wide ones the level passes
    cap = w.seq_len + 3 * w.leaf_block * w.branching + 17
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, capacity=cap, summary_dtype=torch.bfloat16)
    N = w.seq_len // 3
    tree.build(K, N)
    for step in [1, 1, 2, w.leaf_block, w.leaf_block * w.branching + 5, 1, 20 * w.leaf_block]:
        N = min(cap, N + step)
        tree.append(K, N)
        _bit_exact(tree, w, Kn, N, units=[0, w.units - 1])
    tree.append(K, cap)
    _bit_exact(tree, w, Kn, cap)


@pytest.mark.parametrize("w", S16_CASES, ids=lambda w: w.name)
def test_route_and_decode_match_oracle(dev, w):
    from tree_indexed_sparse_build_b200 import zha
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, summary_dtype=torch.bfloat16)
    tree.build(K, w.seq_len)
    idx, sc, tr = tree.route(Q, w.beam, scores=True, trace=True)
    checked, ill, bad = _route_compare(tree, w, Qn, Kn, idx, tr, w.seq_len, summary="bf16")
    assert checked > 0
    # leaf scores are q . S0[leaf] over the stored bf16 summaries
    idx_n, sc_n = idx.cpu().numpy(), sc.cpu().numpy()
    u0 = oracle_tree(w, Kn, 0, w.seq_len, summary="bf16")
    q0 = synth.to_f64(Qn[0, 0])
    for i in range(q0.shape[0]):
        lv = idx_n[0, 0, i][idx_n[0, 0, i] >= 0]
        np.testing.assert_allclose(sc_n[0, 0, i][:len(lv)], u0.levels[0][lv] @ q0[i], rtol=1e-4, atol=1e-4)
    O, didx, dsc, dtr = tree.decode(Q, K, V, w.beam, w.scale, out_dtype=_odt(w), scores=True, trace=True)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert torch.equal(didx, idx) and torch.equal(dtr, tr)
    assert torch.equal(dsc.nan_to_num(-7.0), sc.nan_to_num(-7.0))
    _attend_check(w, Qn, Kn, Vn, O, idx.cpu().numpy().astype(np.int64), w.seq_len)
    print(f"{w.name}: well-conditioned {checked}, ill {ill} ({bad} differ)")


@pytest.mark.parametrize("w", [CASES[i] for i in (0, 1, 2, 4, 6, 13)], ids=lambda w: w.name)
def test_decode_steps_are_bit_exact(dev, w):
    # zha_decode_step over bf16 summaries: the fused append's path rows (and the two-launch
    # form's) equal the oracle's bf16 tree after every step; the outputs equal
    # append + decode on a twin tree
    from tree_indexed_sparse_build_b200 import zha
    cap = w.seq_len + 3 * w.leaf_block + 8
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, capacity=cap, summary_dtype=torch.bfloat16)
    twin = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, cap,
                    torch.float32 if w.kv_dtype == "f32" else torch.bfloat16, summary_dtype=torch.bfloat16)
    N = w.seq_len - 5
    tree.build(K, N)
    twin.build(K, N)
    for step in (1, 1, 3, w.leaf_block, 1):
        N = min(cap, N + step)
        twin.append(K, N)
        O_ref, idx_ref, _ = twin.decode(Q, K, V, w.beam, w.scale, out_dtype=_odt(w))
        O, idx = tree.decode_step(K, V, N, Q, w.beam, w.scale, out_dtype=_odt(w))
        torch.cuda.synchronize()
        assert tree.check() == zha.ZHA_OK and twin.check() == zha.ZHA_OK
        assert torch.equal(idx, idx_ref)
        assert torch.equal(O.float().nan_to_num(7.0), O_ref.float().nan_to_num(7.0))
        _bit_exact(tree, w, Kn, N, units=[0, w.units - 1])
    checked, _, _ = _route_compare(tree, w, Qn, Kn, idx, None, N, units=[0, w.units - 1], summary="bf16")
    assert checked > 0
    _attend_check(w, Qn, Kn, Vn, O, idx.cpu().numpy().astype(np.int64), N)


def test_decode_step_grows_depth_bit_exact(dev):
    w = _wl("grow_s16", 1, 1, 2, 64, 1024, "f32", 2, 16, 2, 4, 109)
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, capacity=1024 + 40, summary_dtype=torch.bfloat16)
    tree.build(K, 1024)
    for N in (1025, 1026, 1040, 1041):
        tree.decode_step(K, V, N, Q, w.beam, w.scale, out_dtype=torch.float32)
        assert tree.levels == 7
        _bit_exact(tree, w, Kn, N)


@pytest.mark.parametrize("which", [0, 2, 3])
def test_causal_routing_over_bf16_prefix_trees(dev, which):
    from tests.test_gpu_causal import CAUSAL, _check, _positions
    from tests.test_gpu_causal import _setup as causal_setup
    from tree_indexed_sparse_build_b200 import zha
    w, nq = CAUSAL[which]
    tree, (Qn, Kn, Vn), (Q, K, V) = causal_setup(w, dev, nq, summary_dtype=torch.bfloat16)
    pos = _positions(w, nq, w.seed + 7)
    pos_d = torch.from_numpy(pos).to(dev)
    O, idx = tree.decode_causal(Q, pos_d, K, V, w.beam, w.scale, out_dtype=_odt(w))
    ridx, tr = tree.route_causal(K, Q, pos_d, w.beam, trace=True)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert torch.equal(idx, ridx)
    _check(w, tree, Qn, Kn, Vn, pos, idx, tr, O, summary="bf16")


@pytest.mark.parametrize("which", [0, 1])
def test_threshold_over_bf16_centers_is_exact(dev, which):
    from tests.test_gpu_threshold import SHAPES, _check_radii
    from tests.test_gpu_threshold import _setup as th_setup
    from tree_indexed_sparse_build_b200 import zha
    w, nq = SHAPES[which]
    tree, (Qn, Kn, Vn), (Q, K, V) = th_setup(w, dev, nq, summary_dtype=torch.bfloat16)
    tree.build(K, w.seq_len)
    tree.attach_radii(K)
    torch.cuda.synchronize()
    _check_radii(w, tree, Kn, w.seq_len, units=[0])
    N = w.seq_len
    tau = np.empty((w.batch, w.q_heads, nq), np.float32)
    for b in range(w.batch):
        for hq in range(w.q_heads):
            s = np.sort(synth.to_f64(Kn[b, hq // w.group, :N]) @ synth.to_f64(Qn[b, hq]).T, axis=0)
            tau[b, hq] = ((s[-10] + s[-11]) / 2).astype(np.float32)
    toks, cnt, _ = tree.threshold(K, Q, torch.from_numpy(tau).to(dev), 64, stats=True)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    toks, cnt = toks.cpu().numpy(), cnt.cpu().numpy()
    for b in range(w.batch):
        for hq in range(w.q_heads):
            q64 = synth.to_f64(Qn[b, hq])
            for i in range(nq):
                ref = oracle.threshold_brute(q64[i], Kn[b, hq // w.group], N, float(tau[b, hq, i]))
                assert cnt[b, hq, i] == len(ref) == 10
                np.testing.assert_array_equal(toks[b, hq, i, :10], ref)
