"""The seeded input generator: determinism, counter addressing, RNE rounding, recipes."""
import ctypes

import numpy as np
import pytest

from tree_indexed_sparse_build_b200 import synth, workloads


def test_counter_addressing_and_determinism():
    a = synth.normal(7, 1, 0, 5000)
    b = synth.normal(7, 1, 1234, 100)
    np.testing.assert_array_equal(a[1234:1334], b)
    np.testing.assert_array_equal(a, synth.normal(7, 1, 0, 5000))
    assert not np.array_equal(a, synth.normal(7, 2, 0, 5000))
    assert not np.array_equal(a, synth.normal(8, 1, 0, 5000))


def test_thread_count_does_not_change_values():
    lib = synth._load()
    n = 300_000
    outs = []
    for th in (1, 3, 8):
        o = np.empty(n, np.float64)
        lib.synth_normal_f64(11, 3, 99, n, 0.0, 1.0, o.ctypes.data_as(ctypes.c_void_p), th)
        outs.append(o)
    np.testing.assert_array_equal(outs[0], outs[1])
    np.testing.assert_array_equal(outs[0], outs[2])


def test_normal_moments():
    x = synth.normal(1, 1, 0, 1 << 20)
    assert abs(x.mean()) < 5e-3
    assert abs(x.std() - 1.0) < 5e-3
    assert abs(np.mean(x ** 4) - 3.0) < 0.05


def _nearest_bf16(x):
    # Brute force: the two bf16 neighbours around x by truncation, nearest wins, ties to even.
    f = np.float32(x)
    bits = int(np.array([f], np.float32).view(np.uint32)[0])
    lo = bits & 0xFFFF0000
    best = None
    for cand in (lo - 0x10000, lo, lo + 0x10000):
        v = float(np.array([cand & 0xFFFFFFFF], np.uint32).view(np.float32)[0])
        err = abs(v - x)
        key = (err, (cand >> 16) & 1)
        if best is None or key < best[0]:
            best = (key, (cand >> 16) & 0xFFFF)
    return best[1]


def test_bf16_rounding_is_nearest_even_from_fp64():
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.standard_normal(3000) * 10 ** rng.uniform(-3, 3, 3000),
                         # exact ties between two bf16 values, and values a hair off a tie
                         [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8),
                          1.0 + 2 ** -8 + 2 ** -40, 1.0 + 2 ** -8 - 2 ** -40]])
    got = synth.round_to(xs, "bf16")
    want = np.array([_nearest_bf16(x) for x in xs], np.uint16)
    np.testing.assert_array_equal(got, want)
    # 1 + 2^-8 + 2^-40 rounds up although its fp32 rounding lands on the tie
    assert got[-2] == 0x3F81


def test_workload_recipes_small():
    w = workloads.get("tiny_fp32")
    Q = synth.queries(w)
    K = synth.keys(w, Q=Q)
    V = synth.values(w)
    assert Q.shape == (1, 1, 16, 64) and Q.dtype == np.float32
    assert K.shape == (1, 1, 1024, 64) and V.shape == K.shape
    nd = synth.needles(w, Q)[0]
    assert len(nd) == 4 and len({p for p, _, _ in nd}) == 4
    for i, (p, hq, qi) in enumerate(nd):
        assert hq == 0 and qi == i
        q = Q[0, 0, qi].astype(np.float64)
        cos = float(K[0, 0, p].astype(np.float64) @ q) / (np.linalg.norm(q) * 3.0)
        assert cos > 0.9  # 3 q_hat + N(0, 0.1^2) noise
    # capacity does not change drawn values
    K2 = synth.keys(w, capacity=1100, Q=Q)
    np.testing.assert_array_equal(K2[:, :, :1024], K)


def test_bf16_queries_prefix_independent_of_nq():
    w = workloads.get("deep_1m").with_(batch=1, kv_heads=1, q_heads=2)
    a = synth.queries(w, nq=1)
    b = synth.queries(w, nq=5)
    np.testing.assert_array_equal(a[:, :, 0], b[:, :, 0])
    assert a.dtype == np.uint16


def test_drift_keys_match_formula():
    w = workloads.get("decode_128k").with_(batch=1, kv_heads=1)
    K = synth.keys(w, capacity=300)
    A, P, phi = synth._drift_params(w, 0)
    x = synth.normal(w.seed, synth.STREAM_K, 0, 300 * 128).reshape(300, 128)
    t = np.arange(300.0)[:, None]
    x = x + 0.5 * (np.sin(2 * np.pi * t / P[None] + phi[None]) @ A.reshape(128, 8).T)
    np.testing.assert_array_equal(K[0, 0], synth.round_to(x, "bf16"))


def test_clustered_keys_are_seeded_blocks_around_centers():
    from tree_indexed_sparse_build_b200.workloads import Workload
    w = Workload(name="c", batch=1, kv_heads=2, q_heads=2, head_dim=16, seq_len=100, kv_dtype="f32",
                 branching=2, leaf_block=8, beam=2)
    a = synth.clustered_keys(w, 0.1)
    assert np.array_equal(a, synth.clustered_keys(w, 0.1))
    x = a[0, 1].astype(np.float64)
    blocks = [x[i:i + 8] for i in range(0, 100, 8)]
    within = max(np.linalg.norm(blk - blk.mean(0), axis=1).max() for blk in blocks)
    between = np.linalg.norm(blocks[0].mean(0) - blocks[1].mean(0))
    assert within < 1.0 < between
