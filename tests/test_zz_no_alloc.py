"""Attention for callers that cannot allocate device memory.

Some callers can neither allocate device memory nor hand the library a scratch
buffer: an operator hook that only receives its input and output pointers, or a
code path where cudaMalloc is not allowed.  zha_sparse_attn_decode_noalloc serves
them from a fixed array inside the library.  These tests call it through the C
ABI and check that two calls in a row give the outputs of zha_sparse_attn_decode
(caller scratch) and of the fp64 oracle's attention over the same leaves, within the
tolerances the parity tests use, and that a shape whose partials do not fit the array is
refused.  The file is collected last.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from tree_indexed_sparse_build_b200 import synth
from tree_indexed_sparse_build_b200.workloads import Workload

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from tree_indexed_sparse_build_b200 import zha
    zha.lib()
    return torch.device("cuda:0"), zha


def _setup(w: Workload, dev, zha, host=False):
    dt = torch.float32 if w.kv_dtype == "f32" else torch.bfloat16
    Kn, Vn = synth.keys(w), synth.values(w)
    K = synth.to_torch(Kn, dev)
    V = synth.to_torch(Vn, dev)
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, w.seq_len, dt)
    tree.build(K, w.seq_len)
    return (tree, K, V, Kn, Vn) if host else (tree, K, V)


@pytest.mark.parametrize("kv_dtype", ["bf16", "f32"])
def test_noalloc_matches_caller_scratch_twice(kv_dtype):
    dev, zha = _need_gpu()
    # few queries, 16 leaves of 32 tokens each: every query's leaves are split over more
    # CTAs than a cluster holds, so their partials go through the fixed array
    w = Workload(name="noalloc", batch=1, kv_heads=2, q_heads=8,
                 head_dim=128, seq_len=9000, kv_dtype=kv_dtype, branching=16, leaf_block=32,
                 beam=16, nq=1, seed=0x2A0F0)
    tree, K, V, Kn, Vn = _setup(w, dev, zha, host=True)
    # the shape splits each query's leaves, so the partials do go through the fixed array
    assert 0 < zha.zha_attn_scratch_bytes(tree.handle, w.q_heads, 1, w.beam) <= \
        zha.zha_noalloc_scratch_capacity()
    odt = torch.float32 if kv_dtype == "f32" else torch.bfloat16
    for call in range(2):
        Qn = synth.queries(w, step=call)
        Q = synth.to_torch(Qn, dev)
        idx, _, _ = tree.route(Q, w.beam)
        ref = tree.attend(Q, K, V, idx, w.beam, w.scale, out_dtype=odt)
        got = torch.full_like(ref, float("nan"))
        zha.zha_sparse_attn_decode_noalloc(tree.handle, Q, K, V, idx, w.beam, w.scale, got)
        torch.cuda.synchronize()
        assert tree.check() == zha.ZHA_OK
        g = got.float().cpu().numpy().astype(np.float64)
        r = ref.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all()
        if kv_dtype == "f32":
            assert np.abs(g - r).max() <= 1e-5
        else:
            rel = np.linalg.norm(g - r, axis=-1) / np.linalg.norm(r, axis=-1)
            assert rel.max() <= 2e-2
        # and against the fp64 oracle's exact attention over the same leaves
        leaves = idx.cpu().numpy().astype(np.int64)
        for hq in range(w.q_heads):
            h = hq // w.group
            q64 = synth.to_f64(Qn[0, hq])
            ref64, _ = oracle.attend(q64[0], Kn[0, h], Vn[0, h], w.seq_len, w.leaf_block, leaves[0, hq, 0], w.scale)
            if kv_dtype == "f32":
                assert np.abs(g[0, hq, 0] - ref64).max() <= 1e-5
            else:
                assert np.linalg.norm(g[0, hq, 0] - ref64) / np.linalg.norm(ref64) <= 2e-2
    tree.close()


def test_noalloc_refuses_partials_beyond_capacity():
    dev, zha = _need_gpu()
    # 36 queries with 16 leaves of 64 tokens each: sixteen splits per query whose partials
    # (36 x 16 x 130 fp32) exceed the fixed array
    w = Workload(name="noalloc_big", batch=1, kv_heads=4, q_heads=36, head_dim=128,
                 seq_len=4096, kv_dtype="bf16", branching=16, leaf_block=64, beam=16, nq=1,
                 seed=0x2A0F1)
    tree, K, V = _setup(w, dev, zha)
    if zha.zha_attn_scratch_bytes(tree.handle, w.q_heads, 1, w.beam) <= \
            zha.zha_noalloc_scratch_capacity():
        pytest.skip("this device's split plan fits the fixed array")
    Q = synth.to_torch(synth.queries(w), dev)
    idx, _, _ = tree.route(Q, w.beam)
    O = torch.empty((1, w.q_heads, 1, 128), dtype=torch.bfloat16, device=dev)
    assert zha.zha_attn_scratch_bytes(tree.handle, w.q_heads, 1, w.beam) > 0
    with pytest.raises(zha.ZhaError) as e:
        zha.zha_sparse_attn_decode_noalloc(tree.handle, Q, K, V, idx, w.beam, w.scale, O)
    assert e.value.status == zha.ZHA_ERR_CAPACITY
    tree.close()
