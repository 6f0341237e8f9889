"""Seeded random shapes through the C ABI against the oracle.

Each case draws a tree geometry (branching 2-16, leaf block 1-64, beam up to 32 with
beam * branching <= 512), head size 64 or 128, K/V in fp32 or bf16, summaries in fp32 or
bf16, a cache length and a query count (so launches fall on both the wide and the narrow
side), then builds, appends in a few steps and runs zha_route, zha_decode and
zha_decode_step.  Bars as in the other parity tests: summaries within 1e-6 normwise (fp32
summaries) or bit-exact with the oracle's bf16 tree; leaf sets and survivors bit-exact on
queries whose fp64 margins exceed 1e-3 |score|; zha_decode selecting zha_route's leaves
exactly; attention within 1e-5 max-abs (fp32 cache and output) or 2e-2 relative L2.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from tests.helpers import make_inputs, oracle_tree, out_to_f64, rel_l2, summary_rel_err, torch_of
from tree_indexed_sparse_build_b200 import synth
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


def _case(seed: int):
    rng = np.random.default_rng(seed)
    b = int(rng.choice([2, 3, 4, 5, 8, 16]))
    lb = int(rng.choice([1, 2, 4, 7, 16, 32, 64]))
    beam = int(rng.integers(1, min(32, 512 // b) + 1))
    d = int(rng.choice([64, 128]))
    kvh = int(rng.integers(1, 3))
    group = int(rng.choice([1, 2, 4]))
    batch = int(rng.integers(1, 3))
    N = int(rng.integers(max(lb * 2, 20), 6000))
    nq = int(rng.choice([1, 2, 5, 16, 40]))
    kv = str(rng.choice(["f32", "bf16"]))
    sdt = str(rng.choice(["f32", "bf16"]))
    w = Workload(name=f"rand{seed}", batch=batch, kv_heads=kvh, q_heads=kvh * group, head_dim=d, seq_len=N,
                 kv_dtype=kv, branching=b, leaf_block=lb, beam=beam, nq=nq,
                 out_dtype="f32" if kv == "f32" else "bf16", seed=0x3B000 + seed)
    return w, sdt


CASES = list(range(24))


@pytest.mark.parametrize("seed", CASES)
def test_random_shape_matches_oracle(dev, seed):
    from tree_indexed_sparse_build_b200 import zha
    w, sdt = _case(seed)
    summary = "bf16" if sdt == "bf16" else "f64"
    cap = w.seq_len + 2 * w.leaf_block + 3
    Qn, Kn, Vn = make_inputs(w, capacity=cap)
    Q, K, V = torch_of(Qn, dev), torch_of(Kn, dev), torch_of(Vn, dev)
    tdt = torch.float32 if w.kv_dtype == "f32" else torch.bfloat16
    odt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, cap, tdt,
                    summary_dtype=torch.bfloat16 if sdt == "bf16" else torch.float32)
    N = w.seq_len - 3
    tree.build(K, N)
    for N in (w.seq_len - 2, w.seq_len):
        tree.append(K, N)
    # decode steps: into the next leaf, then up to the capacity
    for N in sorted({min(w.seq_len + w.leaf_block - w.seq_len % w.leaf_block + 1, cap), cap}):
        O_s, idx_s = tree.decode_step(K, V, N, Q, w.beam, w.scale, out_dtype=odt)
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK

    units = [0, w.units - 1]
    for u in units:
        ot = oracle_tree(w, Kn, u, N, summary=summary)
        assert tree.levels == ot.L
        for lvl in range(ot.L + 1):
            got = tree.level(lvl)[u].float().cpu().numpy().astype(np.float64)
            if sdt == "bf16":
                np.testing.assert_array_equal(got, ot.levels[lvl], err_msg=f"level {lvl}")
            else:
                assert summary_rel_err(got, ot.levels[lvl]) <= 1e-6

    idx, _, tr = tree.route(Q, w.beam, trace=True)
    O, didx = tree.decode(Q, K, V, w.beam, w.scale, out_dtype=odt)[:2]
    torch.cuda.synchronize()
    assert torch.equal(didx, idx), "zha_decode selected other leaves than zha_route"
    assert torch.equal(idx_s, idx), "the decode step selected other leaves than zha_route"
    idx_n, tr_n, got = idx.cpu().numpy(), tr.cpu().numpy(), out_to_f64(O)
    checked = 0
    worst = 0.0
    for u in units:
        bb, h = divmod(u, w.kv_heads)
        ot = oracle_tree(w, Kn, u, N, summary=summary)
        for hq in range(h * w.group, (h + 1) * w.group):
            q64 = synth.to_f64(Qn[bb, hq])
            res = ot.route(q64, w.beam)
            ok = oracle.well_conditioned(res["bounds"])
            for i in range(q64.shape[0]):
                if ok[i]:
                    np.testing.assert_array_equal(idx_n[bb, hq, i], res["leaves"][i])
                    np.testing.assert_array_equal(tr_n[bb, hq, i], res["survivors"][i])
                    checked += 1
                ref, _ = oracle.attend(q64[i], Kn[bb, h], Vn[bb, h], N, w.leaf_block,
                                       idx_n[bb, hq, i].astype(np.int64), w.scale)
                if w.kv_dtype == "f32" and w.out_dtype == "f32":
                    worst = max(worst, float(np.abs(got[bb, hq, i] - ref).max()))
                else:
                    worst = max(worst, rel_l2(got[bb, hq, i], ref))
    assert checked > 0
    assert worst <= (1e-5 if (w.kv_dtype == "f32" and w.out_dtype == "f32") else 2e-2), worst
    tree.close()


@pytest.mark.parametrize("seed", CASES[:12])
def test_random_shape_causal_and_buffered(dev, seed):
    # causal routing at random positions, and the append-buffer decode over a committed prefix
    from tree_indexed_sparse_build_b200 import zha
    w, sdt = _case(seed)
    summary = "bf16" if sdt == "bf16" else "f64"
    Qn, Kn, Vn = make_inputs(w)
    Q, K, V = torch_of(Qn, dev), torch_of(Kn, dev), torch_of(Vn, dev)
    tdt = torch.float32 if w.kv_dtype == "f32" else torch.bfloat16
    odt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, w.seq_len, tdt,
                    summary_dtype=torch.bfloat16 if sdt == "bf16" else torch.float32)
    n_routed = max(w.leaf_block, (w.seq_len // 2) // w.leaf_block * w.leaf_block)
    tree.build(K, n_routed)
    rng = np.random.default_rng(1000 + seed)
    pos = rng.integers(0, n_routed, size=w.nq).astype(np.int64)
    try:
        cidx, ctr = tree.route_causal(K, Q, torch.from_numpy(pos).to(dev), w.beam, trace=True)
        Ob, bidx = tree.decode_buffered(Q, K, V, n_routed, w.seq_len, w.beam, w.scale, out_dtype=odt)
    except zha.ZhaError as e:  # a level too wide for the staged kernel: the call says so
        assert e.status == zha.ZHA_ERR_UNSUPPORTED
        pytest.skip("shape outside the staged kernel")
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK
    cidx, ctr, bidx, got = cidx.cpu().numpy(), ctr.cpu().numpy(), bidx.cpu().numpy(), out_to_f64(Ob)
    checked = 0
    worst = 0.0
    for u in (0, w.units - 1):
        bb, h = divmod(u, w.kv_heads)
        otb = oracle.OracleTree(w.head_dim, w.leaf_block, w.branching, summary=summary).build(Kn[bb, h], n_routed)
        for hq in range(h * w.group, (h + 1) * w.group):
            q64 = synth.to_f64(Qn[bb, hq])
            resb = otb.route(q64, w.beam)
            okb = oracle.well_conditioned(resb["bounds"])
            for i in range(q64.shape[0]):
                # causal: the tree of the prefix 0 .. pos[i]
                ot = oracle.OracleTree(w.head_dim, w.leaf_block, w.branching, summary=summary).build(
                    Kn[bb, h], int(pos[i]) + 1)
                res = ot.route(q64[i:i + 1], w.beam)
                if oracle.well_conditioned(res["bounds"])[0]:
                    np.testing.assert_array_equal(cidx[bb, hq, i], res["leaves"][0])
                    L = ctr.shape[3]
                    np.testing.assert_array_equal(ctr[bb, hq, i, L - ot.L:], res["survivors"][0])
                    checked += 1
                # buffered: routed over the first n_routed tokens, the rest attended
                if okb[i]:
                    np.testing.assert_array_equal(bidx[bb, hq, i], resb["leaves"][i])
                ref, _ = oracle.attend_buffered(q64[i], Kn[bb, h], Vn[bb, h], bidx[bb, hq, i], n_routed, w.seq_len,
                                                w.leaf_block, w.scale)
                if w.kv_dtype == "f32" and w.out_dtype == "f32":
                    worst = max(worst, float(np.abs(got[bb, hq, i] - ref).max()))
                else:
                    worst = max(worst, rel_l2(got[bb, hq, i], ref))
    assert checked > 0
    assert worst <= (1e-5 if (w.kv_dtype == "f32" and w.out_dtype == "f32") else 2e-2), worst
    tree.close()
