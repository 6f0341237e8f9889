"""The Python binding refuses output and index buffers of the wrong type or size.

The C calls take plain pointers and cannot see buffer sizes, so the binding checks every
buffer it hands over against the sizes that follow from Q's shape (and beam, max_tokens)
before any library call.  CPU only: the checks run before the device-tensor check.
"""
from __future__ import annotations

import pytest

torch = pytest.importorskip("torch")

from tree_indexed_sparse_build_b200 import zha  # noqa: E402

B, HQ, NQ, D, BEAM = 1, 2, 3, 64, 4


def _q(dtype=torch.float32):
    return torch.zeros((B, HQ, NQ, D), dtype=dtype)


def _idx(n=B * HQ * NQ * BEAM, dtype=torch.int32):
    return torch.zeros(n, dtype=dtype)


def test_route_leaf_index_buffer():
    with pytest.raises(ValueError, match="leaf_idx: 5 elements"):
        zha.zha_route(None, _q(), BEAM, _idx(5))
    with pytest.raises(ValueError, match="leaf_idx: dtype torch.int64"):
        zha.zha_route(None, _q(), BEAM, _idx(dtype=torch.int64))
    with pytest.raises(ValueError, match="leaf_score"):
        zha.zha_route(None, _q(), BEAM, _idx(), torch.zeros(3, dtype=torch.float32))


def test_decode_output_buffer():
    K = V = torch.zeros(1)
    with pytest.raises(ValueError, match="O: dtype torch.float16"):
        zha.zha_decode(None, _q(), BEAM, K, V, 0.1, _idx(), torch.zeros((B, HQ, NQ, D), dtype=torch.float16))
    with pytest.raises(ValueError, match="O: 8 elements"):
        zha.zha_decode(None, _q(), BEAM, K, V, 0.1, _idx(), torch.zeros(8, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="leaf_idx"):
        zha.zha_sparse_attn_decode(None, _q(), K, V, _idx(7), BEAM, 0.1, torch.zeros((B, HQ, NQ, D)))
    with pytest.raises(ValueError, match="leaf_idx"):
        zha.zha_decode_step(None, K, V, 10, _q(), BEAM, 0.1, _idx(7), torch.zeros((B, HQ, NQ, D)))
    with pytest.raises(ValueError, match="O:"):
        zha.zha_decode_buffered(None, _q(), BEAM, K, V, 8, 9, 0.1, _idx(), torch.zeros(1))


def test_causal_positions_and_threshold_buffers():
    K = V = torch.zeros(1)
    with pytest.raises(ValueError, match="positions: dtype torch.int32"):
        zha.zha_route_causal(None, K, _q(), torch.zeros(NQ, dtype=torch.int32), BEAM, _idx())
    with pytest.raises(ValueError, match="positions: 2 elements"):
        zha.zha_decode_causal(None, _q(), torch.zeros(2, dtype=torch.int64), BEAM, K, V, 0.1, _idx(),
                              torch.zeros((B, HQ, NQ, D)))
    tau = torch.zeros((B, HQ, NQ), dtype=torch.float32)
    count = torch.zeros((B, HQ, NQ), dtype=torch.int32)
    with pytest.raises(ValueError, match="tau: dtype torch.float64"):
        zha.zha_threshold_route(None, K, _q(), tau.double(), 8, torch.zeros((B, HQ, NQ, 8), dtype=torch.int32), count)
    with pytest.raises(ValueError, match="tokens: 24 elements"):
        zha.zha_threshold_route(None, K, _q(), tau, 8, torch.zeros((B, HQ, NQ, 4), dtype=torch.int32), count)
    with pytest.raises(ValueError, match="stats"):
        zha.zha_threshold_route(None, K, _q(), tau, 8, torch.zeros((B, HQ, NQ, 8), dtype=torch.int32), count,
                                torch.zeros(5, dtype=torch.int32))


def test_right_sizes_reach_the_device_check():
    # sizes and types right: the next refusal is the binding's device-tensor check
    with pytest.raises(ValueError, match="device tensors"):
        zha.zha_route(None, _q(), BEAM, _idx(), torch.zeros(B * HQ * NQ * BEAM, dtype=torch.float32))


# Q, K and V against the tree's geometry.  No tree can be created without a GPU, so the
# binding's desc getter is replaced by a fixed geometry: batch 2, 2 KV heads, d 64,
# capacity 16 tokens, bf16 caches.
TREE = zha.zha_tree_desc(2, 2, 64, 4, 4, 16, zha.ZHA_BF16, zha.ZHA_F32)
HANDLE = object()


@pytest.fixture()
def fake_tree(monkeypatch):
    monkeypatch.setattr(zha, "zha_tree_get_desc", lambda h: TREE)


def _cache(dtype=torch.bfloat16, n=2 * 2 * 16 * 64):
    return torch.zeros(n, dtype=dtype)


def _q2(b=2, hq=4, nq=3, d=64, dtype=torch.bfloat16):
    return torch.zeros((b, hq, nq, d), dtype=dtype)


def _out(q):
    return torch.zeros(q.shape, dtype=torch.bfloat16)


def _ix(q, beam=BEAM):
    return torch.zeros(q.shape[:3] + (beam,), dtype=torch.int32)


def test_query_must_fit_the_tree(fake_tree):
    for bad in (_q2(b=1), _q2(b=3), _q2(d=128)):
        with pytest.raises(ValueError, match="does not fit the tree"):
            zha.zha_route(HANDLE, bad, BEAM, _ix(bad))
        with pytest.raises(ValueError, match="does not fit the tree"):
            zha.zha_decode(HANDLE, bad, BEAM, _cache(), _cache(), 0.1, _ix(bad), _out(bad))
        with pytest.raises(ValueError, match="does not fit the tree"):
            zha.zha_sparse_attn_decode_noalloc(HANDLE, bad, _cache(), _cache(), _ix(bad), BEAM, 0.1, _out(bad))
    flat = torch.zeros((2, 4, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="expected \\[batch, q_heads, nq, head_dim\\]"):
        zha.zha_route(HANDLE, flat, BEAM, torch.zeros(2 * 4 * BEAM, dtype=torch.int32))
    with pytest.raises(ValueError, match="Q: dtype torch.float16"):
        q = _q2(dtype=torch.float16)
        zha.zha_route(HANDLE, q, BEAM, _ix(q))


def test_caches_must_fit_the_tree(fake_tree):
    q = _q2()
    for K, V, what in ((_cache(torch.float32), _cache(), "K: dtype"), (_cache(n=100), _cache(), "K: 100"),
                       (_cache(), _cache(n=2 * 2 * 17 * 64), "V: 4352"), (_cache(), _cache(torch.float32), "V: dtype")):
        with pytest.raises(ValueError, match=what):
            zha.zha_decode(HANDLE, q, BEAM, K, V, 0.1, _ix(q), _out(q))
        with pytest.raises(ValueError, match=what):
            zha.zha_decode_step(HANDLE, K, V, 10, q, BEAM, 0.1, _ix(q), _out(q))
        with pytest.raises(ValueError, match=what):
            zha.zha_sparse_attn_decode(HANDLE, q, K, V, _ix(q), BEAM, 0.1, _out(q))
        with pytest.raises(ValueError, match=what):
            zha.zha_decode_buffered(HANDLE, q, BEAM, K, V, 4, 9, 0.1, _ix(q), _out(q))
    with pytest.raises(ValueError, match="K: 100"):
        zha.zha_tree_build(HANDLE, _cache(n=100), 8)
    with pytest.raises(ValueError, match="K: dtype"):
        zha.zha_tree_append(HANDLE, _cache(torch.float32), 8)
    with pytest.raises(ValueError, match="K: 100"):
        zha.zha_route_causal(HANDLE, _cache(n=100), q, torch.zeros(3, dtype=torch.int64), BEAM, _ix(q))


def test_fitting_buffers_reach_the_device_check(fake_tree):
    q = _q2()
    with pytest.raises(ValueError, match="device tensors"):
        zha.zha_decode(HANDLE, q, BEAM, _cache(), _cache(), 0.1, _ix(q), _out(q))
    with pytest.raises(ValueError, match="device tensors"):
        zha.zha_tree_build(HANDLE, _cache(), 8)
