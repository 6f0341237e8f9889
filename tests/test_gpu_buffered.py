"""Decode with an append buffer (zha_decode_buffered) through the C ABI against the oracle.

Each query routes over the tree of the first n_routed tokens and attends over its leaves'
tokens and every buffered token n_routed .. n_tokens - 1.  Bars as in the other parity
tests: leaf sets and survivors bit-exact on queries whose fp64 margins exceed 1e-3 |score|
(the oracle's tree of the first n_routed tokens); attention within 1e-5 max-abs (fp32 cache
and output) or 2e-2 relative L2 against oracle.attend_buffered over the GPU's leaves.
The commit of the buffer (zha_tree_append on a second stream) may run while decodes with
the old n_routed are in flight: their outputs must not change at all.
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


def _odt(w):
    return torch.float32 if w.out_dtype == "f32" else torch.bfloat16


def _setup(w, dev, nq, cap, summary_dtype=None):
    from tree_indexed_sparse_build_b200 import zha
    Qn, Kn, Vn = make_inputs(w, capacity=cap, nq=nq)
    Q, K, V = torch_of(Qn, dev), torch_of(Kn, dev), torch_of(Vn, dev)
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, cap,
                    torch.float32 if w.kv_dtype == "f32" else torch.bfloat16,
                    summary_dtype=summary_dtype or torch.float32)
    return tree, (Qn, Kn, Vn), (Q, K, V)


def _check(w, Qn, Kn, Vn, n_routed, n_tokens, idx, tr, O, summary="f64"):
    idx, tr, got = idx.cpu().numpy(), tr.cpu().numpy(), out_to_f64(O)
    checked = 0
    worst = 0.0
    for b in range(w.batch):
        for h in range(w.kv_heads):
            ot = oracle.OracleTree(w.head_dim, w.leaf_block, w.branching, summary=summary).build(Kn[b, h], n_routed)
            L = tr.shape[3]
            for hq in range(h * w.group, (h + 1) * w.group):
                q64 = synth.to_f64(Qn[b, hq])
                res = ot.route(q64, w.beam)
                ok = oracle.well_conditioned(res["bounds"])
                for i in range(q64.shape[0]):
                    if ok[i]:
                        np.testing.assert_array_equal(idx[b, hq, i], res["leaves"][i])
                        assert (tr[b, hq, i, :L - ot.L] == -1).all()
                        np.testing.assert_array_equal(tr[b, hq, i, L - ot.L:], res["survivors"][i])
                        checked += 1
                    ref, ntok = oracle.attend_buffered(q64[i], Kn[b, h], Vn[b, h], idx[b, hq, i], n_routed,
                                                       n_tokens, w.leaf_block, w.scale)
                    if w.kv_dtype == "f32" and w.out_dtype == "f32":
                        worst = max(worst, float(np.abs(got[b, hq, i] - ref).max()))
                    else:
                        worst = max(worst, rel_l2(got[b, hq, i], ref))
    assert checked > 0
    assert worst <= (1e-5 if (w.kv_dtype == "f32" and w.out_dtype == "f32") else 2e-2), worst


BUF = [
    # wide (few queries), bf16, 16-token leaves
    (_wl("buf_wide_bf16", 1, 2, 4, 128, 4096, "bf16", 8, 16, 8, 1, 401), 4),
    # narrow, fp32, binary tree, one warp per query
    (_wl("buf_narrow_f32", 1, 1, 1, 64, 1024, "f32", 2, 16, 2, 1, 402), 300),
    # narrow warp groups, bf16, 4-token leaves (the 1M geometry)
    (_wl("buf_narrow_lb4", 1, 2, 16, 128, 20000, "bf16", 8, 4, 8, 1, 403), 24),
]


@pytest.mark.parametrize("w,nq", BUF, ids=lambda x: getattr(x, "name", str(x)))
def test_buffered_decode_matches_oracle(dev, w, nq):
    from tree_indexed_sparse_build_b200 import zha
    lb = w.leaf_block
    n_routed = (w.seq_len // 2) // lb * lb
    cap = w.seq_len
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, nq, cap)
    tree.build(K, n_routed)
    for buf in (0, 1, lb - 1, 3 * lb + 5, 300, cap - n_routed):
        n_tokens = n_routed + buf
        O, idx, tr = tree.decode_buffered(Q, K, V, n_routed, n_tokens, w.beam, w.scale, out_dtype=_odt(w),
                                          trace=True)
        torch.cuda.synchronize()
        assert tree.check() == zha.ZHA_OK
        _check(w, Qn, Kn, Vn, n_routed, n_tokens, idx, tr, O)
    # an empty buffer is the causal decode at position n_routed - 1
    pos = torch.full((nq,), n_routed - 1, dtype=torch.int64, device=dev)
    Oc, idxc = tree.decode_causal(Q, pos, K, V, w.beam, w.scale, out_dtype=_odt(w))
    O0, idx0 = tree.decode_buffered(Q, K, V, n_routed, n_routed, w.beam, w.scale, out_dtype=_odt(w))
    assert torch.equal(idx0, idxc) and torch.equal(O0, Oc)


def test_buffered_decode_over_bf16_summaries(dev):
    from tree_indexed_sparse_build_b200 import zha
    w, nq = BUF[2]
    n_routed, n_tokens = 12000, 12345
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, nq, w.seq_len, summary_dtype=torch.bfloat16)
    tree.build(K, n_routed)
    O, idx, tr = tree.decode_buffered(Q, K, V, n_routed, n_tokens, w.beam, w.scale, trace=True)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    _check(w, Qn, Kn, Vn, n_routed, n_tokens, idx, tr, O, summary="bf16")


@pytest.mark.parametrize("w,nq", [BUF[0], BUF[2]], ids=lambda x: getattr(x, "name", str(x)))
def test_commit_on_a_second_stream_leaves_decodes_unchanged(dev, w, nq):
    # decodes with the old n_routed, launched while the buffer's commit (an append on another
    # stream, no ordering between the two) runs, read nothing the commit writes: their
    # outputs equal those of the same decodes before the commit, bit for bit
    from tree_indexed_sparse_build_b200 import zha
    lb = w.leaf_block
    n_routed = (w.seq_len // 2) // lb * lb
    n_tokens = n_routed + 20 * lb + 3
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, nq, w.seq_len)
    tree.build(K, n_routed)
    ref = [tree.decode_buffered(Q, K, V, n_routed, n_tokens, w.beam, w.scale, out_dtype=_odt(w))
           for _ in range(1)][0]
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    with torch.cuda.stream(s1):
        for k in range(6):
            if k == 1:
                tree.append(K, n_tokens, stream=s2)  # the commit, unordered with s1
            outs.append(tree.decode_buffered(Q, K, V, n_routed, n_tokens, w.beam, w.scale, out_dtype=_odt(w),
                                             stream=s1))
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    for O, idx in outs:
        assert torch.equal(idx, ref[1]) and torch.equal(O, ref[0])
    # after the commit, a decode over the committed tree (empty buffer when n_tokens ends a
    # leaf; else the partial leaf stays buffered) matches the oracle
    assert tree.seq_len == n_tokens
    n2 = n_tokens // lb * lb
    O2, idx2, tr2 = tree.decode_buffered(Q, K, V, n2, n_tokens, w.beam, w.scale, out_dtype=_odt(w), trace=True)
    torch.cuda.synchronize()
    _check(w, Qn, Kn, Vn, n2, n_tokens, idx2, tr2, O2)


def test_buffered_host_errors(dev):
    from tree_indexed_sparse_build_b200 import zha
    w, nq = BUF[0]
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, nq, w.seq_len)
    tree.build(K, 1600)
    for n_routed, n_tokens, status in ((1601, 1700, zha.ZHA_ERR_INVALID_ARG),  # not a leaf boundary
                                       (1616, 1700, zha.ZHA_ERR_INVALID_ARG),  # beyond the tree
                                       (0, 10, zha.ZHA_ERR_INVALID_ARG),       # nothing routed
                                       (1600, 1599, zha.ZHA_ERR_INVALID_ARG),  # tokens before the prefix end
                                       (1600, w.seq_len + 1, zha.ZHA_ERR_CAPACITY)):
        with pytest.raises(zha.ZhaError) as e:
            tree.decode_buffered(Q, K, V, n_routed, n_tokens, w.beam, w.scale)
        assert e.value.status == status
    O, idx = tree.decode_buffered(Q, K, V, 1600, 1600, w.beam, w.scale)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
