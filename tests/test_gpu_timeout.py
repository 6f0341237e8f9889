"""Bounded device waits that run out, on purpose and safely.

Every kernel that waits for its own bulk copies bounds the wait; when it runs out the kernel
records ZHA_ERR_TIMEOUT in the tree's error word, waits for the copies it issued (with the
default bound of about a second), marks the affected queries' outputs as lost (leaf indices
-1, O NaN) and returns.  Nothing traps and nothing waits without a bound.  These tests lower
the first bound to one SM clock cycle (zha_tree_set_wait_limit), so the wait for copies that
were issued a moment before gives up, and check:

* zha_tree_check reports ZHA_ERR_TIMEOUT (and clears the word);
* every query's result is either marked lost or equal to a normal run's;
* with the bound restored the same call on the same context succeeds and matches the
  normal run bit for bit.

Right before each call under the lowered bound the L2 cache is flushed, so the copies come
from DRAM and are still in flight at the first check (from L2 they can land first).

Which kernels wait: the staged route kernel (every level's rows and the attention's stages
arrive by bulk copies; it runs the causal and buffered calls, and any shape the other
kernels do not take), the stand-alone attention, the append kernel, and the CTA-per-query
kernel's fused append path.  The warp-per-query and CTA-per-query kernels otherwise load
straight into registers and have no copy to wait for.
"""
from __future__ import annotations

import pytest

from tests.helpers import make_inputs, torch_of
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


# 2 units x 8 query heads, one query each: a wide launch (one query per CTA)
W = Workload(name="timeout", batch=1, kv_heads=2, q_heads=8, head_dim=128, seq_len=6000, kv_dtype="bf16",
             branching=8, leaf_block=16, beam=8, nq=1, seed=131)
# The CTA-per-query kernel waits for the fused append's path after scoring the first level
# (19 leaves here), so the path must still be in flight then: 320-token fp32 leaves make its
# token copy about 160 KB, several thousand cycles behind the first level's rows.
W_PATH = Workload(name="timeout_path", batch=1, kv_heads=2, q_heads=8, head_dim=128, seq_len=6071, kv_dtype="f32",
                  branching=8, leaf_block=320, beam=4, nq=1, seed=132)


def _setup(dev, capacity=None, w=W):
    from tree_indexed_sparse_build_b200 import zha
    cap = capacity or w.seq_len
    Qn, Kn, Vn = make_inputs(w, capacity=cap)
    Q, K, V = torch_of(Qn, dev), torch_of(Kn, dev), torch_of(Vn, dev)
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, cap,
                    torch.float32 if w.kv_dtype == "f32" else torch.bfloat16)
    return tree, Q, K, V


def _flush_l2(dev):
    torch.empty(512 << 20, dtype=torch.uint8, device=dev).zero_()


def _lost_or_equal(idx, O, idx_ref, O_ref):
    """Per query: marked lost (O all NaN; its leaves -1 when the route itself gave up, else
    the reference's) or equal to the reference run.  Returns how many were lost."""
    idx, O = idx.reshape(-1, idx.shape[-1]).cpu(), O.reshape(-1, O.shape[-1]).float().cpu()
    idx_ref, O_ref = idx_ref.reshape(idx.shape).cpu(), O_ref.reshape(O.shape).float().cpu()
    lost = 0
    for i in range(idx.shape[0]):
        if torch.isnan(O[i]).all():
            lost += 1
            assert (idx[i] == -1).all() or torch.equal(idx[i], idx_ref[i]), f"query {i}"
        else:
            assert torch.equal(idx[i], idx_ref[i]) and torch.equal(O[i], O_ref[i]), f"query {i}"
    return lost


def test_staged_route_and_decode_time_out_and_recover(dev):
    # the causal calls run the staged kernel; every query at the last position routes over
    # the whole tree
    from tree_indexed_sparse_build_b200 import zha
    tree, Q, K, V = _setup(dev)
    tree.build(K, W.seq_len)
    pos = torch.full((W.nq,), W.seq_len - 1, dtype=torch.int64, device=dev)
    O_ref, idx_ref = tree.decode_causal(Q, pos, K, V, W.beam, W.scale)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK

    zha.zha_tree_set_wait_limit(tree.handle, 1)
    _flush_l2(dev)
    O, idx = tree.decode_causal(Q, pos, K, V, W.beam, W.scale)
    _flush_l2(dev)
    ridx, _ = tree.route_causal(K, Q, pos, W.beam)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_ERR_TIMEOUT
    assert tree.check() == zha.ZHA_OK  # the word was cleared
    assert _lost_or_equal(idx, O, idx_ref, O_ref) > 0
    rlost = sum(int((ridx.reshape(-1, W.beam)[i] == -1).all()) for i in range(ridx.numel() // W.beam))
    assert rlost > 0

    zha.zha_tree_set_wait_limit(tree.handle, 0)
    O2, idx2 = tree.decode_causal(Q, pos, K, V, W.beam, W.scale)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert torch.equal(idx2, idx_ref) and torch.equal(O2, O_ref)
    tree.close()


def test_register_kernels_do_not_wait(dev):
    # the plain route and decode of this shape load rows straight into registers: a lowered
    # bound changes nothing
    from tree_indexed_sparse_build_b200 import zha
    tree, Q, K, V = _setup(dev)
    tree.build(K, W.seq_len)
    O_ref, idx_ref, _ = tree.decode(Q, K, V, W.beam, W.scale)
    ridx_ref, _, _ = tree.route(Q, W.beam)
    torch.cuda.synchronize()
    zha.zha_tree_set_wait_limit(tree.handle, 1)
    _flush_l2(dev)
    O, idx, _ = tree.decode(Q, K, V, W.beam, W.scale)
    _flush_l2(dev)
    ridx, _, _ = tree.route(Q, W.beam)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert torch.equal(idx, idx_ref) and torch.equal(O, O_ref) and torch.equal(ridx, ridx_ref)
    zha.zha_tree_set_wait_limit(tree.handle, 0)
    tree.close()


def test_standalone_attention_times_out_and_recovers(dev):
    from tree_indexed_sparse_build_b200 import zha
    tree, Q, K, V = _setup(dev)
    tree.build(K, W.seq_len)
    idx, _, _ = tree.route(Q, W.beam)
    O_ref = tree.attend(Q, K, V, idx, W.beam, W.scale)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK

    zha.zha_tree_set_wait_limit(tree.handle, 1)
    _flush_l2(dev)
    O = tree.attend(Q, K, V, idx, W.beam, W.scale)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_ERR_TIMEOUT
    Of, Orf = O.reshape(-1, W.head_dim).float().cpu(), O_ref.reshape(-1, W.head_dim).float().cpu()
    nan_rows = torch.isnan(Of).any(dim=1)
    assert nan_rows.any()
    assert torch.equal(Of[~nan_rows], Orf[~nan_rows])

    zha.zha_tree_set_wait_limit(tree.handle, 0)
    O2 = tree.attend(Q, K, V, idx, W.beam, W.scale)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert torch.equal(O2, O_ref)
    tree.close()


def test_append_and_fused_step_time_out_and_recover(dev):
    from tree_indexed_sparse_build_b200 import zha
    N = W.seq_len - 40
    tree, Q, K, V = _setup(dev)
    ref, _, _, _ = _setup(dev)
    ref.build(K, N + 1)

    # the one-leaf append kernel (path staged with one bulk copy round)
    tree.build(K, N)
    zha.zha_tree_set_wait_limit(tree.handle, 1)
    _flush_l2(dev)
    tree.append(K, N + 1)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_ERR_TIMEOUT
    zha.zha_tree_set_wait_limit(tree.handle, 0)
    tree.build(K, N + 1)  # the summaries the failed append was writing are rebuilt
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    for lvl in range(tree.levels + 1):
        assert torch.equal(tree.level(lvl), ref.level(lvl))

    tree.close()
    ref.close()

    # the fused decode step (append path + route + attention in one launch, CTA-per-query
    # kernel: the path's copies are its one wait)
    w = W_PATH
    N = w.seq_len - 1  # the last leaf holds 310 tokens; the step appends the 311th
    tree, Q, K, V = _setup(dev, w=w)
    ref, _, _, _ = _setup(dev, w=w)
    ref.build(K, N)
    l0 = ref.launches
    O_ref, idx_ref = ref.decode_step(K, V, N + 1, Q, w.beam, w.scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ref.launches - l0 == 1  # fused
    tree.build(K, N)
    zha.zha_tree_set_wait_limit(tree.handle, 1)
    _flush_l2(dev)
    # the query and the first scored level (the leaves) back in L2, the path's tokens not:
    # the route's first rows then arrive long before the path's 160 KB of tokens
    warm = float(Q.sum()) + float(tree.level(0).sum())
    assert warm == warm
    O, idx = tree.decode_step(K, V, N + 1, Q, w.beam, w.scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_ERR_TIMEOUT
    assert _lost_or_equal(idx, O, idx_ref, O_ref) > 0
    zha.zha_tree_set_wait_limit(tree.handle, 0)
    tree.build(K, N)
    O2, idx2 = tree.decode_step(K, V, N + 1, Q, w.beam, w.scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    assert torch.equal(idx2, idx_ref) and torch.equal(O2, O_ref)
    tree.close()
    ref.close()


def test_wait_limit_arguments(dev):
    from tree_indexed_sparse_build_b200 import zha
    tree, Q, K, V = _setup(dev)
    with pytest.raises(zha.ZhaError) as e:
        zha.zha_tree_set_wait_limit(tree.handle, -1)
    assert e.value.status == zha.ZHA_ERR_INVALID_ARG
    with pytest.raises(zha.ZhaError):
        zha.zha_tree_set_wait_limit(None, 5)
    tree.close()
