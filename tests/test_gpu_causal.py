"""Causal (per-position) routing through the C ABI against the fp64 oracle.

Query i of every head routes over the tree of tokens 0 .. positions[i]; the oracle builds
that prefix tree from scratch (its own depth, node counts and right edge) and routes over
it.  Bars as in the other parity tests: leaf sets and per-level survivors bit-exact on
queries whose fp64 beam margins exceed 1e-3 |score| at every level; attention over the
leaves' tokens inside the prefix within 1e-5 max-abs (fp32) or 2e-2 relative L2 (bf16).
Also: the keys read per query over a 1,024-token causal pass (the pages' statistic is
about 30 with learned routing against 512 for dense attention; here it follows from beam
and leaf block alone).
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from tests.helpers import make_inputs, out_to_f64, rel_l2, torch_of
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


def _positions(w, nq, seed):
    rng = np.random.default_rng(seed)
    pos = rng.integers(0, w.seq_len, size=nq).astype(np.int64)
    pos[:3] = [0, w.seq_len - 1, min(w.leaf_block, w.seq_len - 1)]  # first, last, a leaf edge
    return pos


def _setup(w, dev, nq, summary_dtype=None):
    from tree_indexed_sparse_build_b200 import zha
    Qn, Kn, Vn = make_inputs(w, nq=nq)
    Q, K, V = torch_of(Qn, dev), torch_of(Kn, dev), torch_of(Vn, dev)
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, w.seq_len,
                    torch.float32 if w.kv_dtype == "f32" else torch.bfloat16,
                    summary_dtype=summary_dtype or torch.float32)
    tree.build(K, w.seq_len)
    return tree, (Qn, Kn, Vn), (Q, K, V)


def _check(w, tree, Qn, Kn, Vn, pos, idx, tr, O=None, summary="f64"):
    idx, tr = idx.cpu().numpy(), tr.cpu().numpy()
    got_o = out_to_f64(O) if O is not None else None
    L = tree.levels
    checked = ill = 0
    worst = 0.0
    for b in range(w.batch):
        for hq in range(w.q_heads):
            h = hq // w.group
            q64 = synth.to_f64(Qn[b, hq])
            for i, p in enumerate(pos):
                n = int(p) + 1
                ot = oracle.OracleTree(w.head_dim, w.leaf_block, w.branching, summary=summary).build(Kn[b, h], n)
                res = ot.route(q64[i:i + 1], w.beam)
                if oracle.well_conditioned(res["bounds"])[0]:
                    np.testing.assert_array_equal(idx[b, hq, i], res["leaves"][0])
                    Lq = ot.L
                    assert (tr[b, hq, i, :L - Lq] == -1).all()
                    np.testing.assert_array_equal(tr[b, hq, i, L - Lq:], res["survivors"][0])
                    checked += 1
                else:
                    ill += 1
                    valid = idx[b, hq, i][idx[b, hq, i] >= 0]
                    assert len(valid) == min(w.beam, ot.levels[0].shape[0])
                    assert (np.diff(valid) > 0).all() and valid.max() < ot.levels[0].shape[0]
                if got_o is not None:
                    ref, _ = oracle.attend(q64[i], Kn[b, h], Vn[b, h], n, w.leaf_block,
                                           idx[b, hq, i].astype(np.int64), w.scale)
                    if w.kv_dtype == "f32" and w.out_dtype == "f32":
                        worst = max(worst, float(np.abs(got_o[b, hq, i] - ref).max()))
                    else:
                        worst = max(worst, rel_l2(got_o[b, hq, i], ref))
    assert checked > 0
    if got_o is not None:
        assert worst <= (1e-5 if (w.kv_dtype == "f32" and w.out_dtype == "f32") else 2e-2), worst
    return checked, ill


CAUSAL = [
    # wide launch (few queries), bf16, 4-token leaves
    (_wl("causal_wide_bf16", 1, 2, 4, 128, 5000, "bf16", 8, 4, 8, 1, 201), 16),
    # narrow, one warp per query, fp32, binary tree (the pages' 1,024-token setting)
    (_wl("causal_narrow_f32", 1, 1, 1, 64, 1024, "f32", 2, 16, 2, 1, 202), 400),
    # narrow warp groups, bf16, deeper tree
    (_wl("causal_groups_bf16", 1, 2, 16, 128, 20001, "bf16", 8, 4, 8, 1, 203), 32),
    # narrow, 64-token leaves: the attention streams 512 tokens through 8 stages
    (_wl("causal_many_stages", 1, 2, 16, 128, 9000, "bf16", 8, 64, 8, 1, 205), 32),
]


@pytest.mark.parametrize("w,nq", CAUSAL, ids=lambda x: getattr(x, "name", str(x)))
def test_route_causal_matches_oracle(dev, w, nq):
    from tree_indexed_sparse_build_b200 import zha
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, nq)
    pos = _positions(w, nq, w.seed)
    pos_d = torch.from_numpy(pos).to(dev)
    idx, tr = tree.route_causal(K, Q, pos_d, w.beam, trace=True)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    checked, ill = _check(w, tree, Qn, Kn, Vn, pos, idx, tr)
    print(f"{w.name}: well-conditioned {checked}, ill {ill}")


@pytest.mark.parametrize("w,nq", CAUSAL, ids=lambda x: getattr(x, "name", str(x)))
def test_decode_causal_matches_oracle(dev, w, nq):
    from tree_indexed_sparse_build_b200 import zha
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, nq)
    pos = _positions(w, nq, w.seed + 1)
    pos_d = torch.from_numpy(pos).to(dev)
    odt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    O, idx = tree.decode_causal(Q, pos_d, K, V, w.beam, w.scale, out_dtype=odt)
    ridx, tr = tree.route_causal(K, Q, pos_d, w.beam, trace=True)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert torch.equal(idx, ridx)
    _check(w, tree, Qn, Kn, Vn, pos, idx, tr, O)


def test_causal_full_prefix_equals_route(dev):
    # position N - 1 for every query: the prefix is the whole cache, so causal routing must
    # give zha_route's result exactly
    w = CAUSAL[0][0]
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, 16)
    pos_d = torch.full((16,), w.seq_len - 1, dtype=torch.int64, device=dev)
    idx, tr = tree.route_causal(K, Q, pos_d, w.beam, trace=True)
    ridx, _, rtr = tree.route(Q, w.beam, trace=True)
    assert torch.equal(idx, ridx) and torch.equal(tr, rtr)


def test_causal_keys_read_per_query(dev):
    # every position of a 1,024-token cache (binary tree, 16-token leaves, beam 2): keys read
    # per query = tokens of the selected leaves inside the prefix; at most 2 x 16 = 32
    w = _wl("causal_1024", 1, 1, 1, 64, 1024, "f32", 2, 16, 2, 1, 204)
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, 1024)
    pos = np.arange(1024, dtype=np.int64)
    idx, _ = tree.route_causal(K, Q, torch.from_numpy(pos).to(dev), w.beam)
    idx = idx.cpu().numpy()[0, 0].astype(np.int64)
    tok = np.where(idx >= 0, np.minimum((idx + 1) * 16, pos[:, None] + 1) - idx * 16, 0).sum(axis=1)
    assert tok.max() <= 32 and (tok >= np.minimum(pos + 1, 17)).all()
    dense = (pos + 1).mean()
    assert dense == 512.5
    print(f"keys read per query: {tok.mean():.2f} (dense causal: {dense})")


def test_causal_bad_position_is_reported(dev):
    from tree_indexed_sparse_build_b200 import zha
    w = CAUSAL[0][0]
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, 16)
    pos = np.full(16, 10, np.int64)
    pos[3] = w.seq_len  # outside the tree
    idx, _ = tree.route_causal(K, Q, torch.from_numpy(pos).to(dev), w.beam)
    assert tree.check() == zha.ZHA_ERR_DEVICE
    got = idx.cpu().numpy()
    assert (got[:, :, 3] == -1).all()
    assert (got[:, :, 0] >= 0).any()
    assert tree.check() == zha.ZHA_OK
