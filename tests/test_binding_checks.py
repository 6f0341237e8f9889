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
