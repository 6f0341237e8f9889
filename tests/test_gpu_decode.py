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
