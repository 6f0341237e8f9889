"""The benchmark's workloads: their shapes, and the tree sizes those shapes imply.

Each workload is named by what it is; the test fixes its dimensions (so an edit that would
change what the benchmark measures fails here) and checks the leaf and level counts that
follow from the tree's definition (leaves = ceil(N / leaf block); L = the smallest L >= 1
with b^L >= leaves).  CPU only.
"""
from __future__ import annotations

import pytest

import bench
import oracle
from tree_indexed_sparse_build_b200 import workloads

# name: (batch, kv heads, q heads, d, N, K/V type, b, leaf block, beam, leaves, levels)
EXPECTED = {
    "tiny_fp32": (1, 1, 1, 64, 1024, "f32", 2, 16, 2, 64, 6),
    "gqa_32k": (8, 8, 32, 128, 32768, "bf16", 8, 64, 8, 512, 3),
    "decode_128k": (4, 8, 32, 128, 131072, "bf16", 16, 32, 16, 4096, 3),
    "deep_1m": (1, 8, 64, 128, 1048576, "bf16", 8, 4, 8, 262144, 6),
    "build_256k": (1, 8, 32, 128, 262144, "bf16", 4, 16, 4, 16384, 7),
}


@pytest.mark.parametrize("name", sorted(EXPECTED))
def test_workload_shape_and_tree(name):
    w = workloads.get(name)
    B, kvh, qh, d, N, kv, b, lb, beam, leaves, levels = EXPECTED[name]
    assert (w.batch, w.kv_heads, w.q_heads, w.head_dim, w.seq_len, w.kv_dtype) == (B, kvh, qh, d, N, kv)
    assert (w.branching, w.leaf_block, w.beam) == (b, lb, beam)
    counts = bench.level_counts(w.seq_len, w.leaf_block, w.branching)
    assert counts[0] == leaves and counts[-1] == 1
    assert len(counts) - 1 == levels == oracle.num_levels(leaves, b)
    assert w.q_heads % w.kv_heads == 0


def test_workload_extras():
    # tiny: 4 planted needles, at most beam x leaf block = 32 keys read per query, 16 queries
    t = workloads.get("tiny_fp32")
    assert t.needles == 4 and t.beam * t.leaf_block == 32 and t.nq == 16 and t.out_dtype == "f32"
    assert workloads.get("gqa_32k").needles == 16
    d = workloads.get("decode_128k")
    assert d.decode_steps == 64 and d.drift
    assert workloads.get("deep_1m").needles == 64
    assert workloads.THROUGHPUT_NQ == 64
    s = workloads.get("build_256k")
    assert s.append_tokens == 4096 and s.nq == 64
