"""Calls with many queries (narrow launches: several queries per SM) through the C ABI.

Routing is per query, so the leaf sets, per-level survivors and leaf scores of a call with
more than 1,000 queries must equal, bit for bit, those of the same queries routed a few
at a time (wide launches: one query per CTA); they must also equal the oracle's on every
sampled query whose fp64 margins exceed 1e-3 |score|.  zha_decode over the same batch
selects the same leaves, and its outputs are checked against the oracle (1e-5 max-abs for
fp32 K/V and output, 2e-2 relative L2 otherwise).  Shapes cover fp32 / bf16 K/V and
summaries, d 64 / 128, ragged tails, levels kept whole, decodes fused in one launch and
decodes that take two, and q stored in the other precision than K/V.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from tests.helpers import make_inputs, oracle_tree, out_to_f64, rel_l2, torch_of
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


def _w(name, batch, kvh, qh, d, N, kv, b, lb, beam, nq, seed):
    return Workload(name=name, batch=batch, kv_heads=kvh, q_heads=qh, head_dim=d, seq_len=N, kv_dtype=kv,
                    branching=b, leaf_block=lb, beam=beam, nq=nq, out_dtype="f32" if kv == "f32" else "bf16",
                    seed=seed)


# (workload, summary dtype)
CASES = [
    (_w("batch_deep_bf16", 1, 2, 16, 128, 20001, "bf16", 8, 4, 8, 80, 201), "f32"),
    (_w("batch_deep_bf16_s16", 1, 2, 16, 128, 20001, "bf16", 8, 4, 8, 80, 202), "bf16"),
    # the leaves' tokens do not fit the narrow launch's stages: route, then attention
    (_w("batch_f32_d64", 2, 2, 4, 64, 6000, "f32", 4, 16, 5, 160, 203), "f32"),
    (_w("batch_f32_d128_b5", 1, 3, 6, 128, 3001, "f32", 5, 7, 6, 210, 204), "bf16"),
    (_w("batch_bf16_d64_wide_beam", 1, 1, 4, 64, 1000, "bf16", 2, 1, 64, 300, 205), "f32"),
    (_w("batch_large", 1, 1, 8, 64, 3000, "bf16", 4, 8, 4, 700, 206), "f32"),
]


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _tree(w, sdt, dev):
    from tree_indexed_sparse_build_b200 import zha
    tdt = torch.float32 if w.kv_dtype == "f32" else torch.bfloat16
    return zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, w.seq_len, tdt,
                    summary_dtype=torch.bfloat16 if sdt == "bf16" else torch.float32)


def _few_at_a_time(tree, Q, beam, step=8):
    # the same queries in calls of at most 2 x SMs queries (wide launches)
    outs = []
    for s in range(0, Q.shape[2], step):
        outs.append(tree.route(Q[:, :, s:s + step].contiguous(), beam, scores=True, trace=True))
    return tuple(torch.cat([o[i] for o in outs], dim=2) for i in range(3))


def _sample(w, k=6):
    rng = np.random.default_rng(w.seed)
    units = sorted({0, w.units - 1})
    return [(u, int(hq), int(i)) for u in units
            for hq, i in zip(rng.integers(0, w.group, k) + (u % w.kv_heads) * w.group, rng.integers(0, w.nq, k))]


@pytest.mark.parametrize("w,sdt", CASES, ids=lambda c: c.name if hasattr(c, "name") else c)
def test_batch_route_equals_few_at_a_time_and_oracle(dev, w, sdt):
    from tree_indexed_sparse_build_b200 import zha
    assert w.batch * w.q_heads * w.nq > 2 * _sms(), "the call must take a narrow launch"
    assert w.batch * w.q_heads * 8 <= 2 * _sms(), "the slices must take wide launches"
    Qn, Kn, Vn = make_inputs(w)
    Q, K = torch_of(Qn, dev), torch_of(Kn, dev)
    tree = _tree(w, sdt, dev)
    tree.build(K, w.seq_len)
    idx, sc, tr = tree.route(Q, w.beam, scores=True, trace=True)
    idx2, sc2, tr2 = _few_at_a_time(tree, Q, w.beam)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert torch.equal(idx, idx2)
    assert torch.equal(tr, tr2)
    assert torch.equal(torch.nan_to_num(sc, nan=-7.0), torch.nan_to_num(sc2, nan=-7.0))
    idx_n, tr_n = idx.cpu().numpy(), tr.cpu().numpy()
    checked = 0
    summary = "bf16" if sdt == "bf16" else "f64"
    trees = {}
    for u, hq, i in _sample(w):
        bb = u // w.kv_heads
        if u not in trees:
            trees[u] = oracle_tree(w, Kn, u, w.seq_len, summary=summary)
        res = trees[u].route(synth.to_f64(Qn[bb, hq, i:i + 1]), w.beam)
        if oracle.well_conditioned(res["bounds"])[0]:
            np.testing.assert_array_equal(idx_n[bb, hq, i], res["leaves"][0])
            np.testing.assert_array_equal(tr_n[bb, hq, i], res["survivors"][0])
            checked += 1
    assert checked > 0
    tree.close()


@pytest.mark.parametrize("w,sdt", CASES, ids=lambda c: c.name if hasattr(c, "name") else c)
def test_batch_decode_matches_oracle(dev, w, sdt):
    from tree_indexed_sparse_build_b200 import zha
    Qn, Kn, Vn = make_inputs(w)
    Q, K, V = torch_of(Qn, dev), torch_of(Kn, dev), torch_of(Vn, dev)
    tree = _tree(w, sdt, dev)
    tree.build(K, w.seq_len)
    odt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    O, didx, dsc, dtr = tree.decode(Q, K, V, w.beam, w.scale, out_dtype=odt, scores=True, trace=True)
    idx, sc, tr = tree.route(Q, w.beam, scores=True, trace=True)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert torch.equal(didx, idx) and torch.equal(dtr, tr)
    assert torch.equal(torch.nan_to_num(dsc, nan=-7.0), torch.nan_to_num(sc, nan=-7.0))
    got, idx_n = out_to_f64(O), idx.cpu().numpy()
    worst = 0.0
    for u, hq, i in _sample(w, 10):
        bb, h = divmod(u, w.kv_heads)
        ref, _ = oracle.attend(synth.to_f64(Qn[bb, hq, i]), Kn[bb, h], Vn[bb, h], w.seq_len, w.leaf_block,
                               idx_n[bb, hq, i].astype(np.int64), w.scale)
        if w.out_dtype == "f32":
            worst = max(worst, float(np.abs(got[bb, hq, i] - ref).max()))
        else:
            worst = max(worst, rel_l2(got[bb, hq, i], ref))
    assert worst <= (1e-5 if w.out_dtype == "f32" else 2e-2), worst
    assert torch.isfinite(O.float()).all()
    tree.close()


@pytest.mark.parametrize("kv,nq", [("f32", 80), ("f32", 2), ("bf16", 80), ("bf16", 2)])
def test_q_in_the_other_precision(dev, kv, nq):
    # q stored in bf16 over fp32 K/V (and in fp32 over bf16 K/V), in a narrow launch (nq 80)
    # and a wide one (nq 2), against the oracle on q as stored
    from tree_indexed_sparse_build_b200 import zha
    w = _w(f"mixq_{kv}", 1, 2, 16, 128, 9000, kv, 8, 8, 8, nq, 207)
    Qn, Kn, Vn = make_inputs(w)
    Qx = synth.round_to(synth.to_f64(Qn), "bf16") if kv == "f32" else synth.to_f64(Qn).astype(np.float32)
    Q, K, V = torch_of(Qx, dev), torch_of(Kn, dev), torch_of(Vn, dev)
    tree = _tree(w, "f32", dev)
    tree.build(K, w.seq_len)
    odt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    O, idx, _ = tree.decode(Q, K, V, w.beam, w.scale, out_dtype=odt)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    got, idx_n = out_to_f64(O), idx.cpu().numpy()
    worst, checked = 0.0, 0
    ot = {}
    for u, hq, i in _sample(w, 8):
        bb, h = divmod(u, w.kv_heads)
        q64 = synth.to_f64(Qx[bb, hq, i])
        if u not in ot:
            ot[u] = oracle_tree(w, Kn, u, w.seq_len)
        res = ot[u].route(q64[None], w.beam)
        if oracle.well_conditioned(res["bounds"])[0]:
            np.testing.assert_array_equal(idx_n[bb, hq, i], res["leaves"][0])
            checked += 1
        ref, _ = oracle.attend(q64, Kn[bb, h], Vn[bb, h], w.seq_len, w.leaf_block, idx_n[bb, hq, i].astype(np.int64),
                               w.scale)
        worst = max(worst, float(np.abs(got[bb, hq, i] - ref).max()) if w.out_dtype == "f32"
                    else rel_l2(got[bb, hq, i], ref))
    assert checked > 0
    assert worst <= (1e-5 if w.out_dtype == "f32" else 2e-2), worst
    tree.close()
