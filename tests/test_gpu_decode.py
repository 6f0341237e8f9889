"""zha_decode (route + attention in one launch) through the C ABI.

The fused call must select exactly the leaves zha_route selects (same arithmetic, so
bit-exact, scores included), match the fp64 oracle's leaf sets on well-conditioned
queries, and give attention within the parity bars against the oracle's attention
over the leaves it used: 1e-5 max-abs (fp32 cache and output), 2e-2 relative L2 (bf16).
"""
from __future__ import annotations

import numpy as np
import pytest

from tests.helpers import out_to_f64
from tests.test_gpu_parity import CASES, _attend_check, _route_compare, _setup, _wl

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


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_decode_matches_route_and_oracle(dev, w):
    from tree_indexed_sparse_build_b200 import zha
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev)
    tree.build(K, w.seq_len)
    ridx, rsc, rtr = tree.route(Q, w.beam, scores=True, trace=True)
    l0 = tree.launches
    O, idx, sc, tr = tree.decode(Q, K, V, w.beam, w.scale, out_dtype=_odt(w), scores=True, trace=True)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert torch.equal(idx, ridx)
    assert torch.equal(tr, rtr)
    assert torch.equal(sc.nan_to_num(-7.0), rsc.nan_to_num(-7.0))
    checked, ill, bad = _route_compare(tree, w, Qn, Kn, idx, tr, w.seq_len)
    assert checked > 0
    _attend_check(w, Qn, Kn, Vn, O, idx.cpu().numpy().astype(np.int64), w.seq_len)
    launches = tree.launches - l0
    # one launch whenever the plan fuses (the wide cases and the short-leaf narrow one)
    if w.name in ("f32_d64_b2", "bf16_d128_b16_splits", "bf16_d128_narrow_lb4"):
        assert launches == 1
    print(f"{w.name}: launches {launches}, well-conditioned {checked}, ill {ill} ({bad} differ)")


@pytest.mark.parametrize("w", [CASES[2], CASES[4], CASES[9]], ids=lambda w: w.name)
def test_decode_steps_after_appends(dev, w):
    # decode steps interleaved with one-token appends, as in generation
    from tree_indexed_sparse_build_b200 import zha
    cap = w.seq_len + 40
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, capacity=cap)
    N = w.seq_len
    tree.build(K, N)
    for step in range(3):
        N += 1 + 7 * step
        tree.append(K, N)
        O, idx, _ = tree.decode(Q, K, V, w.beam, w.scale, out_dtype=_odt(w))
        torch.cuda.synchronize()
        assert tree.check() == zha.ZHA_OK
        checked, _, _ = _route_compare(tree, w, Qn, Kn, idx, None, N, units=[0, w.units - 1])
        assert checked > 0
        _attend_check(w, Qn, Kn, Vn, O, idx.cpu().numpy().astype(np.int64), N)


def test_decode_single_token_and_padding(dev):
    from tree_indexed_sparse_build_b200 import zha
    w = _wl("one", 1, 1, 1, 64, 1, "f32", 2, 4, 3, 2, 110)
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, capacity=8)
    tree.build(K, 1)
    O, idx, sc = tree.decode(Q, K, V, 3, w.scale, out_dtype=torch.float32, scores=True)
    assert idx.cpu().numpy().tolist() == [[[[0, -1, -1], [0, -1, -1]]]]
    assert torch.isnan(sc[..., 1:]).all()
    np.testing.assert_array_equal(O.cpu().numpy()[0, 0], np.tile(Vn[0, 0, 0], (2, 1)))
    assert tree.check() == zha.ZHA_OK


def test_decode_host_errors(dev):
    from tree_indexed_sparse_build_b200 import zha
    w = CASES[1]
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev)
    with pytest.raises(zha.ZhaError) as e:
        tree.decode(Q, K, V, w.beam, w.scale)  # empty tree
    assert e.value.status == zha.ZHA_ERR_INVALID_ARG
    tree.build(K, w.seq_len)
    with pytest.raises(zha.ZhaError) as e:
        tree.decode(Q, K, V, 1024, w.scale)  # beam * b > 4096
    assert e.value.status == zha.ZHA_ERR_UNSUPPORTED
    O = torch.empty((w.batch, w.q_heads, 1, w.head_dim), dtype=torch.bfloat16, device=dev)
    with pytest.raises(zha.ZhaError) as e:
        zha.zha_decode(tree.handle, Q, w.beam, K, V, float("nan"),
                       torch.empty(Q.shape[:3] + (w.beam,), dtype=torch.int32, device=dev), O)
    assert e.value.status == zha.ZHA_ERR_INVALID_ARG
    O2, idx, _ = tree.decode(Q, K, V, w.beam, w.scale)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert torch.isfinite(out_to_f64_t(O2)).all()


def out_to_f64_t(O):
    return torch.from_numpy(out_to_f64(O))


def _twins(w, dev, cap):
    """Two identical trees over the same seeded cache (capacity cap)."""
    from tree_indexed_sparse_build_b200 import zha
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, capacity=cap)
    twin = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, cap,
                    torch.float32 if w.kv_dtype == "f32" else torch.bfloat16)
    return tree, twin, (Qn, Kn, Vn), (Q, K, V)


def _same_summaries(a, b):
    assert a.levels == b.levels
    for lvl in range(a.levels + 1):
        assert a.level_nodes(lvl) == b.level_nodes(lvl)
        assert torch.equal(a.level(lvl), b.level(lvl)), f"level {lvl} differs"


STEP_CASES = [CASES[0], CASES[1], CASES[2], CASES[4], CASES[6], CASES[10], CASES[13]]


@pytest.mark.parametrize("w", STEP_CASES, ids=lambda w: w.name)
def test_decode_step_equals_append_then_decode(dev, w):
    # zha_decode_step(new N) == zha_tree_append(new N) + zha_decode: bit-identical summaries,
    # leaves and outputs; one launch when the new tokens fall into one leaf (wide launches)
    from tree_indexed_sparse_build_b200 import zha
    cap = w.seq_len + 3 * w.leaf_block + 8
    tree, twin, (Qn, Kn, Vn), (Q, K, V) = _twins(w, dev, cap)
    N = w.seq_len - 5
    tree.build(K, N)
    twin.build(K, N)
    wide = w.batch * w.q_heads * Qn.shape[2] <= 2 * torch.cuda.get_device_properties(dev).multi_processor_count
    for step in (1, 1, 3, w.leaf_block, 1):
        N = min(cap, N + step)
        one_leaf = (tree.seq_len // w.leaf_block) == ((N - 1) // w.leaf_block)
        twin.append(K, N)
        O_ref, idx_ref, _ = twin.decode(Q, K, V, w.beam, w.scale, out_dtype=_odt(w))
        l0 = tree.launches
        O, idx = tree.decode_step(K, V, N, Q, w.beam, w.scale, out_dtype=_odt(w))
        torch.cuda.synchronize()
        assert tree.check() == zha.ZHA_OK and twin.check() == zha.ZHA_OK
        assert tree.seq_len == N
        _same_summaries(tree, twin)
        assert torch.equal(idx, idx_ref)
        assert torch.equal(O.float().nan_to_num(7.0), O_ref.float().nan_to_num(7.0))
        if one_leaf and wide:
            assert tree.launches - l0 == 1
    checked, _, _ = _route_compare(tree, w, Qn, Kn, idx, None, N, units=[0, w.units - 1])
    assert checked > 0
    _attend_check(w, Qn, Kn, Vn, O, idx.cpu().numpy().astype(np.int64), N)


def test_decode_step_grows_depth(dev):
    # 64 full leaves of 16 = b^6; one more token starts leaf 64 under a new root (L 6 -> 7)
    w = _wl("grow", 1, 1, 2, 64, 1024, "f32", 2, 16, 2, 4, 109)
    tree, twin, (Qn, Kn, Vn), (Q, K, V) = _twins(w, dev, 1024 + 40)
    tree.build(K, 1024)
    twin.build(K, 1024)
    for N in (1025, 1026, 1040, 1041):
        twin.append(K, N)
        O_ref, idx_ref, _ = twin.decode(Q, K, V, w.beam, w.scale, out_dtype=torch.float32)
        O, idx, tr = tree.decode_step(K, V, N, Q, w.beam, w.scale, out_dtype=torch.float32, trace=True)
        torch.cuda.synchronize()
        assert tree.levels == 7
        _same_summaries(tree, twin)
        assert torch.equal(idx, idx_ref) and torch.equal(O, O_ref)
        checked, _, _ = _route_compare(tree, w, Qn, Kn, idx, tr, N)
        assert checked > 0
        _attend_check(w, Qn, Kn, Vn, O, idx.cpu().numpy().astype(np.int64), N)


def test_decode_step_host_errors_leave_tree_unchanged(dev):
    from tree_indexed_sparse_build_b200 import zha
    w = CASES[1]
    tree, (Qn, Kn, Vn), (Q, K, V) = _setup(w, dev, capacity=w.seq_len + 4)
    tree.build(K, w.seq_len)
    for bad_n, status in ((w.seq_len - 1, zha.ZHA_ERR_INVALID_ARG),
                          (w.seq_len + 5, zha.ZHA_ERR_CAPACITY)):
        with pytest.raises(zha.ZhaError) as e:
            tree.decode_step(K, V, bad_n, Q, w.beam, w.scale)
        assert e.value.status == status
        assert tree.seq_len == w.seq_len
    with pytest.raises(zha.ZhaError) as e:
        tree.decode_step(K, V, w.seq_len + 1, Q, 1024, w.scale)  # beam * b > 4096
    assert e.value.status == zha.ZHA_ERR_UNSUPPORTED
    assert tree.seq_len == w.seq_len
    O, idx = tree.decode_step(K, V, w.seq_len + 1, Q, w.beam, w.scale)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK and tree.seq_len == w.seq_len + 1
