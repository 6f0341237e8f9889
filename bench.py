#!/usr/bin/env python
"""Benchmark of tree-indexed sparse decode attention on B200.

Default (one GPU): the 128K decode workload -- batch 4, 8 KV heads, 32 query
heads, d = 128, bf16 cache of 131,072 tokens, b = 16, leaf block 32, beam 16.
A step is one decode step over the whole batch: append one token to every
(batch, KV head) tree (ancestor recompression, depth growth on the first
step), route one query per query head, attend.  Each step is replayed from its
own CUDA graph with graph-captured events around each call; an L2 flush
(512 MiB memset) runs between steps, outside the events.  The same JSON line
also carries the 1M-token throughput figures (64 queries per head) and the
256K build / append figures.

``--impl reference`` times the fp64 oracle instead (host cores, bounded sample).

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode queries/sec at 128K and 1M ctx; route+attend HBM GB/s vs B200 peak"
UNIT = "queries/s"
FALLBACK_HBM_GBS = 6650.0
FLUSH_BYTES = 512 << 20


# ----------------------------------------------------------------------------- helpers

def levels_for(n0: int, b: int) -> int:
    if n0 <= 0:
        return 0
    L, span = 1, b
    while span < n0:
        span *= b
        L += 1
    return L


def level_counts(N: int, lb: int, b: int) -> list[int]:
    n0 = -(-N // lb)
    L = levels_for(n0, b)
    out, n = [], n0
    for _ in range(L + 1):
        out.append(n)
        n = -(-n // b)
    return out


def append_bytes(N_new: int, lb: int, b: int, d: int, kv_bytes: int, units: int, sum_bytes: int = 4) -> int:
    """Algorithmic bytes of a one-leaf append that ends at N_new tokens: per unit, the
    touched leaf's tokens and, at every level above, the stored children of the path node
    are read; the L + 1 path rows (sum_bytes an element) are written."""
    counts = level_counts(N_new, lb, b)
    L = len(counts) - 1
    leaf = (N_new - 1) // lb
    per_unit = (N_new - leaf * lb) * d * kv_bytes
    node = leaf
    for lvl in range(1, L + 1):
        node //= b
        per_unit += (min(node * b + b, counts[lvl - 1]) - node * b) * d * sum_bytes
    per_unit += (L + 1) * d * sum_bytes
    return per_unit * units


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def path_bytes(idx, trace, counts, N, lb, b, d, kv_bytes, g, out_bytes, sum_bytes=4):
    """Algorithmic bytes of one route call and one attend call, plus per-query counts.

    Bytes are the union per (batch, KV head) of distinct summary rows scored (sum_bytes an
    element: 4 for fp32 summaries, 2 for bf16) and of distinct leaf-token K/V rows attended,
    plus Q in, indices and O out.
    """
    B, Hq, nq, beam = idx.shape
    L = trace.shape[3]
    Hkv = Hq // g
    route_rows = 0
    attend_tokens = 0
    scored = []
    keys = []
    ar = np.arange(b)
    for bb in range(B):
        for h in range(Hkv):
            tr = trace[bb, h * g:(h + 1) * g].reshape(-1, L, beam)
            lv = idx[bb, h * g:(h + 1) * g].reshape(-1, beam)
            nqq = tr.shape[0]
            per_q = np.full(nqq, counts[L - 1], np.int64)
            route_rows += counts[L - 1]
            for li in range(1, L):
                l = L - 1 - li
                s = tr[:, li - 1, :].astype(np.int64)
                ch = s[:, :, None] * b + ar[None, None, :]
                ok = (s[:, :, None] >= 0) & (ch < counts[l])
                per_q += ok.reshape(nqq, -1).sum(axis=1)
                route_rows += np.unique(ch[ok]).size
            scored.append(per_q)
            valid = lv >= 0
            tok = np.where(valid, np.minimum((lv.astype(np.int64) + 1) * lb, N) - lv.astype(np.int64) * lb, 0)
            keys.append(tok.sum(axis=1))
            u = np.unique(lv[valid])
            attend_tokens += int((np.minimum((u + 1) * lb, N) - u * lb).sum())
    q = B * Hq * nq
    route_b = route_rows * d * sum_bytes + q * d * kv_bytes + q * beam * 4
    attend_b = attend_tokens * 2 * d * kv_bytes + q * d * kv_bytes + q * beam * 4 + q * d * out_bytes
    return {"route_bytes": int(route_b), "attend_bytes": int(attend_b),
            "summaries_per_query": float(np.concatenate(scored).mean()),
            "keys_per_query": float(np.concatenate(keys).mean())}


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples: list[tuple[int, int]] = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                if not uuid.startswith("GPU-"):
                    uuid = "GPU-" + uuid
                self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = int(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.ok = True
        except Exception as e:  # NVML absent: report no clocks rather than fail the bench
            self.err = str(e)

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                              getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
        while not self._stop.is_set():
            try:
                mhz = int(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                rs = int(get_reasons(self.h)) if get_reasons else 0
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": getattr(self, "max_mhz", None), "reasons": [],
                    "samples": 0}
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        names = sorted(v for k, v in self.REASONS.items() if bits & k and k != 0x1)
        return {"sm_mhz": float(statistics.median(mhz)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(mhz)}


def kernel_traffic(kernel: str):
    """dram bytes per launch recorded from an ncu capture, if the kernel source is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel)
        srcs = rec["source"] if isinstance(rec["source"], list) else [rec["source"]]
        h = hashlib.sha256()
        for name in srcs:  # the kernel's source files, hashed in the listed order
            with open(os.path.join(ROOT, "tree_indexed_sparse_build_b200", "csrc", name), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["sha256"]:
            return None
        return rec["dram_bytes_per_launch"]
    except Exception:
        return None


# ----------------------------------------------------------------------------- our arm

def _graph_events(n):
    import torch
    return [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n)]


def run_decode(w, W, K, rank, dev, flush, sampler_factory, eager=False, mode="step", summary_dtype=None,
               e2e=True):
    """128K decode steps: append 1 token + route + attend, one CUDA graph per step.

    mode "step": one zha_decode_step launch per step (append, route and attention fused);
    "decode": zha_tree_append then zha_decode; "two_call": zha_tree_append, zha_route,
    zha_sparse_attn_decode.  Timed pass (the bench value): steps W .. W+K-1, each graph
    bracketed by a start and an end event only.  Kernel pass (per-call times for the
    roofline): steps W+K .. W+2K-1, with an event after the append as well in the modes that
    launch it separately (extra graph nodes between the kernels cost a few microseconds,
    which is why they stay out of the timed pass).
    """
    import torch
    from tree_indexed_sparse_build_b200 import ranks, synth, zha

    summary_dtype = summary_dtype or torch.float32
    sum_bytes = 2 if summary_dtype == torch.bfloat16 else 4
    N, cap = w.seq_len, w.seq_len + W + 2 * K
    w = w.with_(seed=ranks.rank_seed(w.seed, rank))
    Qs = np.stack([synth.queries(w, step=s) for s in range(W + 2 * K)])
    Kn = synth.keys(w, capacity=cap)
    Vn = synth.values(w, capacity=cap)
    Kd, Vd, Qd = synth.to_torch(Kn, dev), synth.to_torch(Vn, dev), synth.to_torch(Qs, dev)
    B, Hq, nq, d, beam = w.batch, w.q_heads, 1, w.head_dim, w.beam
    tree = zha.Tree(B, w.kv_heads, d, w.branching, w.leaf_block, cap, torch.bfloat16,
                    summary_dtype=summary_dtype)
    tree.build(Kd, N)
    scratch = tree.scratch_for(Hq, nq, beam, dev)
    idx = torch.empty((2 * K, B, Hq, nq, beam), dtype=torch.int32, device=dev)
    O = torch.empty((2 * K, B, Hq, nq, d), dtype=torch.bfloat16, device=dev)
    Ls = [levels_for(-(-(N + W + s + 1) // w.leaf_block), w.branching) for s in range(2 * K)]
    traces = [torch.empty((B, Hq, nq, Ls[s], beam), dtype=torch.int32, device=dev)
              for s in range(2 * K)]
    Ow = torch.empty((B, Hq, nq, d), dtype=torch.bfloat16, device=dev)
    Iw = torch.empty((B, Hq, nq, beam), dtype=torch.int32, device=dev)
    for s in range(W):
        zha.zha_decode_step(tree.handle, Kd, Vd, N + s + 1, Qd[s], beam, w.scale, Iw, Ow)
    torch.cuda.synchronize()

    def decode_call(new_n, Q, ix, out, tr, e=None):
        """The step's calls; e: record an event between the append and the rest."""
        if mode == "step":
            zha.zha_decode_step(tree.handle, Kd, Vd, new_n, Q, beam, w.scale, ix, out, None, tr)
            return
        zha.zha_tree_append(tree.handle, Kd, new_n)
        if e is not None:
            e.record()
        if mode == "two_call":
            zha.zha_route(tree.handle, Q, beam, ix, None, tr)
            zha.zha_sparse_attn_decode(tree.handle, Q, Kd, Vd, ix, beam, w.scale, out, scratch)
        else:
            zha.zha_decode(tree.handle, Q, beam, Kd, Vd, w.scale, ix, out, None, tr)

    def one_step(s, e):
        """Step W+s; e = [start, end] or [start, after append, end]."""
        st = W + s
        e[0].record()
        decode_call(N + st + 1, Qd[st], idx[s], O[s], traces[s], e[1] if len(e) == 3 else None)
        e[-1].record()

    def make(nev):
        if eager:  # same launches without graphs (for profilers that cannot replay graph nodes)
            return [torch.cuda.Event(enable_timing=True) for _ in range(nev)]
        return _graph_events(nev)

    # timed pass
    l0 = tree.launches
    outer, graphs = [], []
    cap_stream = torch.cuda.Stream()
    if eager:
        outer = [make(2) for _ in range(K)]
        with sampler_factory() as smp:
            for s in range(K):
                flush.zero_()
                one_step(s, outer[s])
            torch.cuda.synchronize()
    else:
        for s in range(K):
            e = make(2)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap_stream, capture_error_mode="thread_local"):
                one_step(s, e)
            graphs.append(g)
            outer.append(e)
        torch.cuda.synchronize()
        with sampler_factory() as smp:
            for s in range(K):
                flush.zero_()
                graphs[s].replay()
            torch.cuda.synchronize()
    launches = (tree.launches - l0) / K
    t_step = np.array([outer[s][0].elapsed_time(outer[s][1]) for s in range(K)])

    # kernel pass
    n_in = 2 if mode == "step" else 3
    inner, graphs2 = [], []
    if eager:
        inner = [make(n_in) for _ in range(K)]
        for s in range(K):
            flush.zero_()
            one_step(K + s, inner[s])
        torch.cuda.synchronize()
    else:
        for s in range(K):
            e = make(n_in)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap_stream, capture_error_mode="thread_local"):
                one_step(K + s, e)
            graphs2.append(g)
            inner.append(e)
        torch.cuda.synchronize()
        for s in range(K):
            flush.zero_()
            graphs2[s].replay()
        torch.cuda.synchronize()
    if mode == "step":  # one launch: append, route and attention together
        t_dec = np.array([inner[s][0].elapsed_time(inner[s][1]) for s in range(K)])
        t_app = np.zeros(K)
    else:
        t_app = np.array([inner[s][0].elapsed_time(inner[s][1]) for s in range(K)])
        t_dec = np.array([inner[s][1].elapsed_time(inner[s][2]) for s in range(K)])
    assert tree.check() == zha.ZHA_OK, "device error word set during the timed steps"

    idx_n, tr_n = idx.cpu().numpy(), [t.cpu().numpy() for t in traces]
    acc = {"route_bytes": 0, "attend_bytes": 0, "summaries_per_query": 0.0, "keys_per_query": 0.0,
           "append_bytes": 0}
    for s in range(K, 2 * K):  # the kernel pass's calls, whose times the roofline uses
        Nst = N + W + s + 1
        acc["append_bytes"] += append_bytes(Nst, w.leaf_block, w.branching, d, 2, w.units, sum_bytes) / K
        pb = path_bytes(idx_n[s], tr_n[s], level_counts(Nst, w.leaf_block, w.branching), Nst,
                        w.leaf_block, w.branching, d, 2, w.group, 2, sum_bytes=sum_bytes)
        for k in pb:
            acc[k] += pb[k] / K
    del graphs, graphs2
    # the last kernel-pass step (tokens N + W + 2K) against the oracle, first and last unit
    sl = 2 * K - 1
    par = parity_sample(w, Qs[W + sl], Kn, Vn, N + W + sl + 1, idx_n[sl], tr_n[sl], O[sl].float().cpu().numpy(),
                        (0, w.units - 1), summary="bf16" if sum_bytes == 2 else "f64")
    res = {"parity": par, "step_ms": t_step, "append_ms": t_app, "decode_ms": t_dec,
           "queries_per_step": B * Hq * nq, "launches_per_step": launches, "clocks": smp.summary(),
           **acc}
    if not e2e:
        tree.close()
        return res

    # End to end through the public API: per step, H2D of the new K/V rows and the query
    # from pinned memory, append + route + attend, D2H of the output, synchronize.  Measured
    # twice: each step's calls issued eagerly, and each step's calls (copies included)
    # captured in one CUDA graph per step, as a serving loop would replay them (the value
    # reported as e2e).
    # host staging step-major ([step, batch, kv_heads, d]), so a step's rows are one contiguous
    # pinned block (graph capture copies only from pinned, contiguous host memory)
    hk = torch.from_numpy(np.ascontiguousarray(np.moveaxis(Kn[:, :, N:N + W + K], 2, 0))).view(
        torch.bfloat16).pin_memory()
    hv = torch.from_numpy(np.ascontiguousarray(np.moveaxis(Vn[:, :, N:N + W + K], 2, 0))).view(
        torch.bfloat16).pin_memory()
    hq = torch.from_numpy(Qs).view(torch.bfloat16).pin_memory()
    ho = torch.empty((K, B, Hq, nq, d), dtype=torch.bfloat16).pin_memory()
    qbuf = torch.empty((B, Hq, nq, d), dtype=torch.bfloat16, device=dev)
    obuf = torch.empty((B, Hq, nq, d), dtype=torch.bfloat16, device=dev)
    ibuf = torch.empty((B, Hq, nq, beam), dtype=torch.int32, device=dev)

    # the step's K and V rows go straight into the caches' strided rows with one 2-D copy each
    # (B * H rows of d elements; the caches' row pitch is the capacity); torch's copy_ of a
    # strided destination would stage through a temporary and a copy kernel
    try:
        from cuda.bindings import runtime as cudart
    except Exception:  # no CUDA Python bindings: torch's copies
        cudart = None

    def h2d_rows(dst_cache, src_host, pos):
        if cudart is None:
            dst_cache[:, :, pos].copy_(src_host, non_blocking=True)
            return
        esz = dst_cache.element_size()
        err, = cudart.cudaMemcpy2DAsync(dst_cache[:, :, pos].data_ptr(), cap * d * esz, src_host.data_ptr(),
                                        d * esz, d * esz, B * w.kv_heads,
                                        cudart.cudaMemcpyKind.cudaMemcpyHostToDevice,
                                        torch.cuda.current_stream().cuda_stream)
        if err != cudart.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaMemcpy2DAsync: {err}")

    def e2e_calls(s, out_slot):
        pos = N + s
        h2d_rows(Kd, hk[s], pos)
        h2d_rows(Vd, hv[s], pos)
        qbuf.copy_(hq[s], non_blocking=True)
        decode_call(pos + 1, qbuf, ibuf, obuf, None)
        if out_slot is not None:
            ho[out_slot].copy_(obuf, non_blocking=True)

    def timed_e2e(run):
        for s in range(W):
            run(s, None)
            torch.cuda.current_stream().synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for s in range(K):
            run(W + s, s)
            torch.cuda.current_stream().synchronize()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / K

    tree.build(Kd, N)
    res["e2e_eager_ms_per_step"] = timed_e2e(e2e_calls)
    if not eager:
        tree.build(Kd, N)  # the same starting tree; the graphs replay the same steps
        egraphs = []
        for s in range(W + K):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap_stream, capture_error_mode="thread_local"):
                e2e_calls(s, s - W if s >= W else None)
            egraphs.append(g)
        res["e2e_ms_per_step"] = timed_e2e(lambda s, slot: egraphs[s].replay())
        del egraphs
    else:
        res["e2e_ms_per_step"] = res["e2e_eager_ms_per_step"]
    # the copies put exactly the seeded rows into the caches
    want = torch.from_numpy(np.ascontiguousarray(Kn[:, :, N:N + W + K])).to(dev).view(torch.bfloat16)
    assert torch.equal(Kd[:, :, N:N + W + K], want), "e2e K rows differ from the seeded ones"
    res["h2d_bytes_per_step"] = int(2 * B * w.kv_heads * d * 2 + B * Hq * nq * d * 2)
    res["d2h_bytes_per_step"] = int(B * Hq * nq * d * 2)
    # parity spot check of the last e2e output against the graph run is not meaningful
    # (different steps); correctness is covered by the -m gpu tests.
    tree.close()
    return res


def run_decode_split(w, W, K, rank, world, dev, flush):
    """128K decode steps of ONE workload split over the ranks by (batch, KV head) unit: rank r
    decodes units ranks.unit_range(units, world, r) (its K/V rows and queries are contiguous
    slices of the full tensors, run as a tree set of batch 1) and the step's outputs are
    all-gathered into unit order on every rank.  A step = zha_decode_step on the rank's units
    (one CUDA graph) + the all-gather, bracketed by events on the same stream; L2 flushed
    between steps.  Returns the rank's per-step times and a parity sample of its first unit."""
    import torch
    from tree_indexed_sparse_build_b200 import ranks, synth, zha

    N, cap = w.seq_len, w.seq_len + W + K
    u0, u1 = ranks.unit_range(w.units, world, rank)
    nl, g, d, beam = u1 - u0, w.group, w.head_dim, w.beam
    Qs = np.stack([synth.queries(w, step=s) for s in range(W + K)])  # [steps, B, Hq, 1, d]
    Kn = synth.keys(w, capacity=cap, units=list(range(u0, u1)))
    Vn = synth.values(w, capacity=cap, units=list(range(u0, u1)))
    Kl = ranks.unit_slice(torch.from_numpy(Kn), u0, u1).contiguous().view(torch.bfloat16).to(dev)
    Vl = ranks.unit_slice(torch.from_numpy(Vn), u0, u1).contiguous().view(torch.bfloat16).to(dev)
    Ql = torch.stack([ranks.query_slice(torch.from_numpy(Qs[s]), g, u0, u1) for s in range(W + K)]).contiguous()
    Ql = Ql.view(torch.bfloat16).to(dev)  # [steps, 1, nl * g, 1, d]
    tree = zha.Tree(1, nl, d, w.branching, w.leaf_block, cap, torch.bfloat16)
    tree.build(Kl, N)
    O = torch.empty((W + K, 1, nl * g, 1, d), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((W + K, 1, nl * g, 1, beam), dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream()
    graphs = []
    for s in range(W + K):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream, capture_error_mode="thread_local"):
            zha.zha_decode_step(tree.handle, Kl, Vl, N + s + 1, Ql[s], beam, w.scale, idx[s], O[s])
        graphs.append(gr)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms, full = [], None
    for s in range(W + K):
        flush.zero_()
        torch.cuda.synchronize()
        ranks.barrier(world)
        e0.record()
        graphs[s].replay()
        full = ranks.gather_units(O[s].reshape(nl * g, d), w.units, world, rank, g)
        e1.record()
        torch.cuda.synchronize()
        if s >= W:
            ms.append(e0.elapsed_time(e1))
    assert tree.check() == zha.ZHA_OK, "device error word set during the split decode steps"
    assert full.shape == (w.units * g, d)
    s_last = W + K - 1
    par = parity_sample(w.with_(batch=1, kv_heads=nl, q_heads=nl * g), Ql[s_last].view(torch.uint16).cpu().numpy(),
                        ranks.unit_slice(torch.from_numpy(Kn), u0, u1).numpy(),
                        ranks.unit_slice(torch.from_numpy(Vn), u0, u1).numpy(), N + s_last + 1,
                        idx[s_last].cpu().numpy(), None, O[s_last].float().cpu().numpy(), (0,))
    del graphs
    tree.close()
    return {"step_ms": np.array(ms), "units": [u0, u1], "parity": par}


def run_buffered(w, W, K, rank, dev, flush, buf_leaves=2, eager=False):
    """128K decode steps with an append buffer: each step writes one token into the buffer
    (tokens after the committed prefix) and runs zha_decode_buffered; when buf_leaves full
    leaves have accumulated, the step also commits them (zha_tree_append on a second stream,
    forked from the step and joined at its end, so the commit overlaps that step's decode).
    One CUDA graph per step (eager: the same launches without graphs), start and end events
    on the decode stream around the fork and the join; L2 flushed between steps."""
    import torch
    from tree_indexed_sparse_build_b200 import ranks, synth, zha

    lb = w.leaf_block
    N, cap = w.seq_len, w.seq_len + W + K
    w = w.with_(seed=ranks.rank_seed(w.seed, rank))
    Qs = np.stack([synth.queries(w, step=s) for s in range(W + K)])
    Kd = synth.to_torch(synth.keys(w, capacity=cap), dev)
    Vd = synth.to_torch(synth.values(w, capacity=cap), dev)
    Qd = synth.to_torch(Qs, dev)
    B, Hq, d, beam = w.batch, w.q_heads, w.head_dim, w.beam
    tree = zha.Tree(B, w.kv_heads, d, w.branching, lb, cap, torch.bfloat16)
    tree.build(Kd, N)
    torch.cuda.synchronize()
    O = torch.empty((W + K, B, Hq, 1, d), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((W + K, B, Hq, 1, beam), dtype=torch.int32, device=dev)
    main, side = torch.cuda.Stream(), torch.cuda.Stream()
    plan, n_routed, commits = [], N, 0
    for s in range(W + K):  # (tokens after this step's write, routed prefix, commit target or None)
        n_tok = N + s + 1
        full = (n_tok - n_routed) // lb
        target = n_routed + buf_leaves * lb if full >= buf_leaves else None
        plan.append((n_tok, n_routed, target))
        if target is not None:
            n_routed = target
    def step(s, e):
        n_tok, nr, target = plan[s]
        e[0].record(main)
        if target is not None:
            side.wait_stream(main)
            zha.zha_tree_append(tree.handle, Kd, target, side)
        zha.zha_decode_buffered(tree.handle, Qd[s], beam, Kd, Vd, nr, n_tok, w.scale, idx[s], O[s],
                                None, None, main)
        if target is not None:
            main.wait_stream(side)
        e[1].record(main)

    graphs, evs = [], []
    l0 = tree.launches
    if eager:
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in plan]
        runs = [(lambda s=s: step(s, evs[s])) for s in range(len(plan))]
        with torch.cuda.stream(main):  # the step's launches, outside any graph
            for s in range(W):
                runs[s]()
        torch.cuda.synchronize()
        launches = (tree.launches - l0) / W if W else 0.0
    else:
        for s in range(len(plan)):
            e = _graph_events(2)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=main, capture_error_mode="thread_local"):
                step(s, e)
            graphs.append(g)
            evs.append(e)
        launches = (tree.launches - l0) / len(plan)
        runs = [g.replay for g in graphs]
        for s in range(W):
            runs[s]()
    torch.cuda.synchronize()
    for s in range(W, W + K):
        flush.zero_()
        if eager:
            torch.cuda.synchronize()
            with torch.cuda.stream(main):
                runs[s]()
        else:
            runs[s]()
    torch.cuda.synchronize()
    assert tree.check() == zha.ZHA_OK, "device error word set during the buffered steps"
    t = np.array([evs[s][0].elapsed_time(evs[s][1]) for s in range(W, W + K)])
    commits = sum(1 for s in range(W, W + K) if plan[s][2] is not None)
    tree.close()
    return {"ms_per_step": float(t.mean()), "qps": B * Hq / (t.mean() * 1e-3),
            "commit_step_ms": float(np.mean([t[i] for i in range(K) if plan[W + i][2] is not None] or [0.0])),
            "plain_step_ms": float(np.mean([t[i] for i in range(K) if plan[W + i][2] is None] or [0.0])),
            "commits": commits, "buffer_leaves": buf_leaves, "launches_per_step": launches}


def run_1m(W, K, rank, dev, flush, eager=False, summary_dtype=None):
    """1M-token cache, 8 KV heads: route + attend with 64 queries per head (throughput)
    and with 1 query per head (single step).  summary_dtype: the tree's summary storage
    (fp32 by default; torch.bfloat16 halves the rows a route reads)."""
    import torch
    from tree_indexed_sparse_build_b200 import ranks, synth, workloads, zha

    w = workloads.get("deep_1m")
    w = w.with_(seed=ranks.rank_seed(w.seed, rank))
    nqt = workloads.THROUGHPUT_NQ
    Qn = synth.queries(w, nq=nqt)
    Kn = synth.keys(w, Q=Qn)
    Vn = synth.values(w)
    Kd, Vd, Qd = synth.to_torch(Kn, dev), synth.to_torch(Vn, dev), synth.to_torch(Qn, dev)
    K0, V0 = np.ascontiguousarray(Kn[:1, :1]), np.ascontiguousarray(Vn[:1, :1])  # unit 0, for parity
    del Kn, Vn
    d, beam, N = w.head_dim, w.beam, w.seq_len
    summary_dtype = summary_dtype or torch.float32
    sum_bytes = 2 if summary_dtype == torch.bfloat16 else 4
    tree = zha.Tree(w.batch, w.kv_heads, d, w.branching, w.leaf_block, N, torch.bfloat16,
                    summary_dtype=summary_dtype)
    tree.build(Kd, N)
    torch.cuda.synchronize()
    counts = level_counts(N, w.leaf_block, w.branching)
    out = {}
    for mode, nq in (("throughput", nqt), ("single", 1)):
        Q = Qd[:, :, :nq].contiguous()
        idx = torch.empty((w.batch, w.q_heads, nq, beam), dtype=torch.int32, device=dev)
        tr = torch.empty((w.batch, w.q_heads, nq, tree.levels, beam), dtype=torch.int32, device=dev)
        O = torch.empty((w.batch, w.q_heads, nq, d), dtype=torch.bfloat16, device=dev)
        scratch = tree.scratch_for(w.q_heads, nq, beam, dev)

        def one_step(e):
            """e = [start, end]: the fused call (zha_decode); e = [start, after route, end]:
            zha_route then zha_sparse_attn_decode, for the per-call breakdown."""
            e[0].record()
            if len(e) == 2:
                zha.zha_decode(tree.handle, Q, beam, Kd, Vd, w.scale, idx, O, None, tr)
            else:
                zha.zha_route(tree.handle, Q, beam, idx, None, tr)
                e[1].record()
                zha.zha_sparse_attn_decode(tree.handle, Q, Kd, Vd, idx, beam, w.scale, O, scratch)
            e[-1].record()

        runs = {}
        for nev in (2, 3):  # fused (the bench figure), then the two-call breakdown
            l0 = tree.launches
            if eager:
                e = [torch.cuda.Event(enable_timing=True) for _ in range(nev)]
                runs[nev] = (e, (lambda e=e: one_step(e)))
            else:
                e = _graph_events(nev)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=torch.cuda.Stream(), capture_error_mode="thread_local"):
                    one_step(e)
                runs[nev] = (e, g.replay, g)
            if nev == 2:
                launches = tree.launches - l0
        times = {}
        for nev in (3, 2):
            e, run = runs[nev][0], runs[nev][1]
            for _ in range(W):
                run()
            torch.cuda.synchronize()
            rows = []
            for _ in range(K):
                flush.zero_()
                run()
                torch.cuda.synchronize()
                rows.append([e[i].elapsed_time(e[i + 1]) for i in range(nev - 1)])
            times[nev] = np.array(rows)
        tr_ms, at_ms = times[3][:, 0], times[3][:, 1]
        step_ms = times[2][:, 0]
        pb = path_bytes(idx.cpu().numpy(), tr.cpu().numpy(), counts, N, w.leaf_block,
                        w.branching, d, 2, w.group, 2, sum_bytes=sum_bytes)
        if mode == "throughput":  # the needles were planted for these 64 queries per head
            out["needle_recall"] = needle_recall(w, Qn, idx.cpu().numpy())
        par = parity_sample(w, Qn[:, :, :nq], K0, V0, N, idx.cpu().numpy(), tr.cpu().numpy(),
                            O.float().cpu().numpy(), (0,), summary="bf16" if sum_bytes == 2 else "f64")
        out[mode] = {"route_ms": tr_ms, "attend_ms": at_ms, "step_ms": step_ms, "parity": par,
                     "queries_per_step": w.batch * w.q_heads * nq, "launches_per_step": launches, **pb}
        del runs
    out["dense_bytes_per_step"] = int(2 * N * d * 2 * w.kv_heads * w.batch)
    out["levels"] = tree.levels
    tree.close()
    return out


def run_build_256k(W, K, dev, flush):
    """256K cache: build from scratch, append 4,096 tokens in one call, route + attend 64
    queries per head (one zha_decode call)."""
    import torch
    from tree_indexed_sparse_build_b200 import synth, workloads, zha

    w = workloads.get("build_256k")
    Qn = synth.queries(w)
    Kn = synth.keys(w)
    Vn = synth.values(w)
    Kd, Vd, Qd = synth.to_torch(Kn, dev), synth.to_torch(Vn, dev), synth.to_torch(Qn, dev)
    d, N, cap = w.head_dim, w.seq_len, w.capacity
    tree = zha.Tree(w.batch, w.kv_heads, d, w.branching, w.leaf_block, cap, torch.bfloat16)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    build_ms, append_ms, ra_ms = [], [], []
    for it in range(W + max(1, min(K, 10))):
        flush.zero_()
        ev[0].record()
        tree.build(Kd, N)
        ev[1].record()
        flush.zero_()
        ev[2].record()
        tree.append(Kd, cap)
        ev[3].record()
        flush.zero_()
        ev[4].record()
        last = tree.decode(Qd, Kd, Vd, w.beam, w.scale)
        ev[5].record()
        torch.cuda.synchronize()
        if it >= W:
            build_ms.append(ev[0].elapsed_time(ev[1]))
            append_ms.append(ev[2].elapsed_time(ev[3]))
            ra_ms.append(ev[4].elapsed_time(ev[5]))
    counts = level_counts(N, w.leaf_block, w.branching)
    rows = sum(counts)
    build_bytes = N * d * 2 * w.units + rows * d * 4 * w.units
    q = w.batch * w.q_heads * w.nq
    O, idx = last[0], last[1]
    par = parity_sample(w, Qn, Kn, Vn, cap, idx.cpu().numpy(), None, O.float().cpu().numpy(),
                        (0, w.units - 1),
                        gpu_levels=lambda u: [tree.level(l)[u].float().cpu().numpy() for l in range(tree.levels + 1)])
    del Kn, Vn
    res = {"parity": par, "build_ms": float(np.mean(build_ms)), "build_bytes": int(build_bytes),
           "build_gbs": build_bytes / (np.mean(build_ms) * 1e-3) / 1e9,
           "append_4096_ms": float(np.mean(append_ms)), "levels_after_append": tree.levels,
           "route_attend_ms": float(np.mean(ra_ms)), "queries": q,
           "qps": q / (np.mean(ra_ms) * 1e-3)}
    tree.close()
    return res


def needle_recall(w, Qn, idx) -> dict:
    """Planted needles whose leaf the assigned query's routed leaves include (a reported figure,
    not a pass mark: mean pooling over a leaf block dilutes a single key).  idx: the route's
    leaf indices [batch, q_heads, nq, beam] for the queries Qn the needles were planted with."""
    from tree_indexed_sparse_build_b200 import synth
    hits = total = 0
    for u, lst in enumerate(synth.needles(w, Qn)):
        b = u // w.kv_heads
        for p, hq, qi in lst:
            total += 1
            hits += int((idx[b, hq, qi] == p // w.leaf_block).any())
    return {"needles": total, "retrieved": hits, "recall": hits / total if total else None}


def run_needles(dev) -> dict:
    """Needle recall of zha_route on the workloads with planted needles (tiny_fp32: 4 needles
    = 3 q_hat + N(0, 0.1^2); gqa_32k: 16 per KV head = 4 q_hat + N(0, 0.2^2))."""
    import torch
    from tree_indexed_sparse_build_b200 import synth, workloads, zha
    out = {}
    for name in ("tiny_fp32", "gqa_32k"):
        w = workloads.get(name)
        Qn = synth.queries(w)
        Kn = synth.keys(w, Q=Qn)
        tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, w.seq_len,
                        torch.float32 if w.kv_dtype == "f32" else torch.bfloat16)
        tree.build(synth.to_torch(Kn, dev), w.seq_len)
        idx, _, _ = tree.route(synth.to_torch(Qn, dev), w.beam)
        out[name] = needle_recall(w, Qn, idx.cpu().numpy())
        tree.close()
    return out


def run_causal(W, K, dev, flush):
    """Causal (per-position) routing + attention, zha_decode_causal: (1) every position of a
    1,024-token cache (tiny_fp32's tree: binary, 16-token leaves, beam 2) with the keys read
    per query against dense causal attention; (2) 256 evenly spaced positions of every head of
    the gqa_32k cache (b 8, 64-token leaves, beam 8)."""
    import torch
    from tree_indexed_sparse_build_b200 import synth, workloads, zha

    out = {}
    cases = (("prefix_1024", workloads.get("tiny_fp32").with_(needles=0), 1024),
             ("gqa_32k", workloads.get("gqa_32k").with_(needles=0), 256))
    for name, w, npos in cases:
        Qn = synth.queries(w, nq=npos)
        Kn, Vn = synth.keys(w), synth.values(w)
        dt = torch.float32 if w.kv_dtype == "f32" else torch.bfloat16
        Kd, Vd, Qd = synth.to_torch(Kn, dev), synth.to_torch(Vn, dev), synth.to_torch(Qn, dev)
        del Kn, Vn
        tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, w.seq_len, dt)
        tree.build(Kd, w.seq_len)
        pos = np.linspace(0, w.seq_len - 1, npos).round().astype(np.int64)
        pos_d = torch.from_numpy(pos).to(dev)
        idx = torch.empty((w.batch, w.q_heads, npos, w.beam), dtype=torch.int32, device=dev)
        O = torch.empty((w.batch, w.q_heads, npos, w.head_dim), dtype=dt if name == "prefix_1024" else torch.bfloat16,
                        device=dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ms = []
        for it in range(W + K):
            flush.zero_()
            e0.record()
            zha.zha_decode_causal(tree.handle, Qd, pos_d, w.beam, Kd, Vd, w.scale, idx, O)
            e1.record()
            torch.cuda.synchronize()
            if it >= W:
                ms.append(e0.elapsed_time(e1))
        assert tree.check() == zha.ZHA_OK
        li = idx.cpu().numpy().astype(np.int64)
        tok = np.where(li >= 0, np.minimum((li + 1) * w.leaf_block, pos[None, None, :, None] + 1)
                       - li * w.leaf_block, 0).sum(axis=-1)
        q = w.batch * w.q_heads * npos
        out[name] = {"queries": q, "ms": float(np.mean(ms)), "qps": q / (np.mean(ms) * 1e-3),
                     "keys_per_query": float(tok.mean()), "dense_keys_per_query": float((pos + 1).mean())}
        tree.close()
    return out


def run_threshold(W, K, dev, flush):
    """Threshold (halfspace) descent, zha_threshold_route, on two 32K caches of the gqa_32k
    geometry (8 x 8 KV heads, 32 query heads, b 8, 64-token leaves): its own keys (N(0, 1)
    with planted needles) and clustered keys (each leaf block a random center plus 0.1 N(0, 1)
    noise).  Per query tau lies halfway between its 16th and 17th largest key scores (dense
    pass, untimed); every token at or above it is returned."""
    import torch
    from tree_indexed_sparse_build_b200 import synth, workloads, zha

    base = workloads.get("gqa_32k")
    out = {}
    for name in ("gqa_32k", "clustered_32k"):
        w = base if name == "gqa_32k" else base.with_(needles=0)
        Qn = synth.queries(w)
        Kn = synth.keys(w, Q=Qn) if name == "gqa_32k" else synth.clustered_keys(w, 0.1)
        Kd, Qd = synth.to_torch(Kn, dev), synth.to_torch(Qn, dev)
        del Kn
        tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, w.seq_len, torch.bfloat16)
        tree.build(Kd, w.seq_len)
        tree.attach_radii(Kd)
        kv = Kd.float().repeat_interleave(w.group, dim=1)  # [B, Hq, N, d]
        top = torch.topk(torch.einsum("bhqd,bhnd->bhqn", Qd.float(), kv), 17, dim=-1).values
        tau = ((top[..., 15] + top[..., 16]) / 2).contiguous()
        del kv, top
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ms = []
        for it in range(W + K):
            flush.zero_()
            e0.record()
            toks, cnt, st = tree.threshold(Kd, Qd, tau, 64, stats=True)
            e1.record()
            torch.cuda.synchronize()
            if it >= W:
                ms.append(e0.elapsed_time(e1))
        assert tree.check() == zha.ZHA_OK
        cnt, st = cnt.cpu().numpy(), st.cpu().numpy()
        q = w.batch * w.q_heads * w.nq
        nodes = sum(tree.level_nodes(lvl) for lvl in range(tree.levels))
        out[name] = {"queries": q, "ms": float(np.mean(ms)), "qps": q / (np.mean(ms) * 1e-3),
                     "found_per_query": float(cnt[cnt >= 0].mean()), "overflowed": int((cnt < 0).sum()),
                     "spheres_tested_per_query": float(st[..., 0].mean()), "scored_nodes_per_tree": int(nodes),
                     "tokens_checked_per_query": float(st[..., 1].mean()), "dense_keys_per_query": w.seq_len}
        tree.close()
    return out


def run_profile_case(case: str, W: int, K: int):
    """A small case of a bench workload for ncu captures (eager launches, no graphs):
    deep_1m_2kv = the 1M-token tree with 2 KV heads and 16 query heads (group 8, 64 queries
    per head) instead of 8 and 64, so a capture holds about 1.5 GB on the device;
    deep_1m_2kv_q256 = the same with 256 queries per head (4,096 queries, as many per SM as
    the full batch)."""
    import torch
    from tree_indexed_sparse_build_b200 import synth, workloads, zha

    dev = torch.device("cuda", 0)
    w = workloads.get("deep_1m").with_(kv_heads=2, q_heads=16)
    nq = workloads.THROUGHPUT_NQ * (4 if case.endswith("_q256") else 1)
    Qn = synth.queries(w, nq=nq)
    Kn = synth.keys(w, Q=Qn)
    Vn = synth.values(w)
    Kd, Vd, Q = synth.to_torch(Kn, dev), synth.to_torch(Vn, dev), synth.to_torch(Qn, dev)
    del Kn, Vn
    tree = zha.Tree(w.batch, w.kv_heads, w.head_dim, w.branching, w.leaf_block, w.seq_len, torch.bfloat16)
    tree.build(Kd, w.seq_len)
    idx = torch.empty((w.batch, w.q_heads, nq, w.beam), dtype=torch.int32, device=dev)
    O = torch.empty((w.batch, w.q_heads, nq, w.head_dim), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = []
    for it in range(W + K):
        flush.zero_()
        e0.record()
        zha.zha_decode(tree.handle, Q, w.beam, Kd, Vd, w.scale, idx, O)
        e1.record()
        torch.cuda.synchronize()
        if it >= W:
            ms.append(e0.elapsed_time(e1))
    assert tree.check() == zha.ZHA_OK
    tree.close()
    return {"case": case, "queries": w.batch * w.q_heads * nq, "zha_decode_ms": float(np.mean(ms))}


# ----------------------------------------------------------------------------- parity sample

def parity_sample(w, Q, K, V, N, idx, trace, O, units, summary="f64", gpu_levels=None):
    """A sampled check of one call's results against the fp64 oracle, reported (not raised).

    Per sampled (batch, KV head) unit: the oracle's tree over tokens [0, N) (fp64 summaries,
    or bf16-stored ones with summary="bf16"), its beam descent for every query of the unit,
    and exact attention over the leaves the GPU selected.  A query is well-conditioned when
    its fp64 margins between the beam-th and next score exceed 1e-3 |score| at every level;
    its leaves and per-level survivors must then equal the oracle's (counted in "exact").
    The other queries' leaf sets may differ and are counted as mismatches.  Q: stored queries
    [B, Hq, nq, d]; K, V: stored caches [B, H_kv, >= N, d]; idx, trace, O: the call's outputs
    as numpy arrays (trace may be None; O as floats).  gpu_levels(unit), when given, returns
    the GPU tree's levels of that unit (numpy, leaves first); each node must then be within
    1e-6 normwise relative error of the oracle's (bit-exact for bf16-stored summaries)."""
    import oracle
    from tree_indexed_sparse_build_b200 import synth

    t0 = time.perf_counter()
    Q64 = synth.to_f64(Q)
    O64 = np.asarray(O, dtype=np.float64)
    g = w.group
    wc = exact = ill = ill_mis = n = 0
    max_abs = max_rel = 0.0
    sum_err, sum_ok = 0.0, True
    for u in units:
        b, h = divmod(u, w.kv_heads)
        ot = oracle.OracleTree(w.head_dim, w.leaf_block, w.branching, summary=summary).build(K[b, h], N)
        if gpu_levels is not None:
            got_levels = gpu_levels(u)
            sum_ok &= len(got_levels) == len(ot.levels)
            for got, ref in zip(got_levels, ot.levels):
                got = np.asarray(got, dtype=np.float64)
                sum_ok &= got.shape == ref.shape
                if got.shape != ref.shape:
                    continue
                if summary == "bf16":
                    sum_ok &= bool(np.array_equal(got, ref))
                den = np.linalg.norm(ref, axis=-1)
                rel = np.linalg.norm(got - ref, axis=-1) / np.where(den > 0, den, 1.0)
                sum_err = max(sum_err, float(rel.max()) if rel.size else 0.0)
        flat = ot.flat()
        for hq in range(h * g, (h + 1) * g):
            res = ot.route(Q64[b, hq], w.beam, flat=flat)
            ok = oracle.well_conditioned(res["bounds"])
            got = idx[b, hq]
            same = (got == res["leaves"]).all(axis=-1)
            if trace is not None:
                same &= (trace[b, hq] == res["survivors"]).all(axis=(-2, -1))
            n += got.shape[0]
            wc += int(ok.sum())
            exact += int((same & ok).sum())
            ill += int((~ok).sum())
            ill_mis += int((~same & ~ok).sum())
            for i in range(got.shape[0]):
                ref, _ = oracle.attend(Q64[b, hq, i], K[b, h], V[b, h], N, w.leaf_block,
                                       got[i].astype(np.int64), w.scale)
                err = O64[b, hq, i] - ref
                max_abs = max(max_abs, float(np.abs(err).max()))
                max_rel = max(max_rel, float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)))
    fp32 = w.kv_dtype == "f32" and w.out_dtype == "f32"
    attn_ok = max_abs <= 1e-5 if fp32 else max_rel <= 2e-2
    extra = {}
    if gpu_levels is not None:
        sum_ok &= sum_err <= 1e-6
        extra = {"summary_max_rel_err": sum_err, "summaries_ok": bool(sum_ok)}
        attn_ok &= bool(sum_ok)
    return {**extra, "units": list(units), "summaries": "bf16" if summary == "bf16" else "fp32", "queries": n,
            "well_conditioned": wc, "exact": exact, "ill_conditioned": ill, "ill_mismatch": ill_mis,
            "ill_mismatch_rate": ill_mis / max(n, 1), "attn_max_abs": max_abs, "attn_max_rel_l2": max_rel,
            "attn_bar": "max-abs 1e-5" if fp32 else "rel L2 2e-2",
            "pass": bool(exact == wc and attn_ok), "oracle_s": time.perf_counter() - t0}


def parity_brief(p) -> str:
    """One short line of a parity_sample result."""
    if not p:
        return "not checked"
    err = f"abs {p['attn_max_abs']:.1e}" if p["attn_bar"].startswith("max") else f"rl2 {p['attn_max_rel_l2']:.1e}"
    return (f"{'ok' if p['pass'] else 'FAIL'} {p['exact']}/{p['well_conditioned']} exact, "
            f"ill {p['ill_mismatch']}/{p['ill_conditioned']} differ, {err}")


# ----------------------------------------------------------------------------- small workloads

def run_small(name, W, K, dev, flush):
    """One zha_decode call (route + attention, one launch) over a tree built on the workload's
    cache, replayed from a CUDA graph with start and end events, L2 flushed between calls:
    tiny_fp32 (1,024 fp32 tokens, 16 queries, fp32 output) and gqa_32k (one decode step: 8 x
    32 query heads, one query each, over 32,768 bf16 tokens)."""
    import torch
    from tree_indexed_sparse_build_b200 import synth, workloads, zha

    w = workloads.get(name)
    Qn = synth.queries(w)
    Kn = synth.keys(w, Q=Qn if w.needles else None)
    Vn = synth.values(w)
    Kd, Vd, Qd = synth.to_torch(Kn, dev), synth.to_torch(Vn, dev), synth.to_torch(Qn, dev)
    tdt = torch.float32 if w.kv_dtype == "f32" else torch.bfloat16
    odt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    d, N, beam = w.head_dim, w.seq_len, w.beam
    tree = zha.Tree(w.batch, w.kv_heads, d, w.branching, w.leaf_block, N, tdt)
    tree.build(Kd, N)
    idx = torch.empty((w.batch, w.q_heads, w.nq, beam), dtype=torch.int32, device=dev)
    tr = torch.empty((w.batch, w.q_heads, w.nq, tree.levels, beam), dtype=torch.int32, device=dev)
    O = torch.empty((w.batch, w.q_heads, w.nq, d), dtype=odt, device=dev)
    e = _graph_events(2)
    g = torch.cuda.CUDAGraph()
    l0 = tree.launches
    with torch.cuda.graph(g, stream=torch.cuda.Stream(), capture_error_mode="thread_local"):
        e[0].record()
        zha.zha_decode(tree.handle, Qd, beam, Kd, Vd, w.scale, idx, O, None, tr)
        e[1].record()
    launches = tree.launches - l0
    for _ in range(W):
        g.replay()
    torch.cuda.synchronize()
    ms = []
    for _ in range(K):
        flush.zero_()
        g.replay()
        torch.cuda.synchronize()
        ms.append(e[0].elapsed_time(e[1]))
    assert tree.check() == zha.ZHA_OK, f"device error word set during {name}"
    kvb = 4 if w.kv_dtype == "f32" else 2
    ob = 4 if w.out_dtype == "f32" else 2
    idx_n, tr_n = idx.cpu().numpy(), tr.cpu().numpy()
    pb = path_bytes(idx_n, tr_n, level_counts(N, w.leaf_block, w.branching), N, w.leaf_block,
                    w.branching, d, kvb, w.group, ob)
    t = float(np.mean(ms))
    q = w.batch * w.q_heads * w.nq
    peak, _ = hbm_peak()
    byts = pb["route_bytes"] + pb["attend_bytes"]
    units = range(w.units) if w.units <= 8 else range(0, w.units, w.units // 8)
    par = parity_sample(w, Qn, Kn, Vn, N, idx_n, tr_n, O.float().cpu().numpy(), units)
    del g
    tree.close()
    return {"call": "zha_decode (route + attention, one launch)", "queries": q, "ms": t,
            "qps": q / (t * 1e-3), "bytes": int(byts), "gbs": byts / (t * 1e-3) / 1e9,
            "frac_of_peak": byts / (t * 1e-3) / 1e9 / peak, "keys_per_query": pb["keys_per_query"],
            "summaries_per_query": pb["summaries_per_query"], "launches": launches, "parity": par}


# ----------------------------------------------------------------------------- oracle arm

def oracle_decode_sample(w, seconds: float, max_steps: int, units=(0, 1, 2, 3), warmup: int = 0,
                         start=None):
    """Time the fp64 oracle on decode steps of `w` for a few units (single thread).

    Setup (not timed): each sampled unit's tree over the first N tokens and every step's
    queries.  Timed: per step and unit, append one token, route the unit's query heads,
    attend each.
    """
    import oracle
    from tree_indexed_sparse_build_b200 import synth

    N = w.seq_len
    cap = N + warmup + max_steps
    units = list(units)
    Kn = synth.keys(w, capacity=cap, units=units)
    Vn = synth.values(w, capacity=cap, units=units)
    trees = {u: oracle.OracleTree(w.head_dim, w.leaf_block, w.branching).build(
        Kn[u // w.kv_heads, u % w.kv_heads], N) for u in units}

    # every step's queries are drawn before the clock starts (drawing them is not oracle work)
    Qsteps = [synth.queries(w, step=s) for s in range(warmup + max_steps)]

    def step(s):
        q = Qsteps[s]
        n = 0
        for u in units:
            b, h = divmod(u, w.kv_heads)
            t = trees[u]
            t.append(Kn[b, h], N + s + 1)
            qs = synth.to_f64(q[b, h * w.group:(h + 1) * w.group, 0])
            res = t.route(qs, w.beam)
            for i in range(qs.shape[0]):
                oracle.attend(qs[i], Kn[b, h], Vn[b, h], N + s + 1, w.leaf_block,
                              res["leaves"][i], w.scale)
                n += 1
        return n

    for s in range(warmup):
        step(s)
    if start is not None:  # threads of a host-parallel run begin their timed steps together
        start.wait()
    t0 = time.perf_counter()
    nq = steps = 0
    per_step = []
    while steps < max_steps and (time.perf_counter() - t0) < seconds:
        ts = time.perf_counter()
        nq += step(warmup + steps)
        per_step.append(time.perf_counter() - ts)
        steps += 1
    el = time.perf_counter() - t0
    return {"value": nq / el, "queries": nq, "seconds": el, "steps": steps, "units": len(units),
            "per_step_s": per_step}


def oracle_route_attend_sample(w, seconds: float, nq: int, units=(0,), N=None, start=None):
    """Time the fp64 oracle's route + attention over prebuilt trees (single thread).

    Setup (not timed): the sampled units' caches, their trees over tokens [0, N) (N defaults to
    the workload's), the stacked levels the descent reads, and nq queries per query head.
    Timed: every query of the units' heads routed and attended, unit after unit, repeated
    until `seconds` have passed (at least one pass)."""
    import oracle
    from tree_indexed_sparse_build_b200 import synth

    N = N or w.seq_len
    units = list(units)
    Qn = synth.queries(w, nq=nq)
    Kn = synth.keys(w, capacity=N, Q=Qn if w.needles else None, units=units)
    Vn = synth.values(w, capacity=N, units=units)
    Q64 = synth.to_f64(Qn)
    trees, flats = {}, {}
    for u in units:
        b, h = divmod(u, w.kv_heads)
        trees[u] = oracle.OracleTree(w.head_dim, w.leaf_block, w.branching).build(Kn[b, h], N)
        flats[u] = trees[u].flat()
    g = w.group
    if start is not None:  # processes of a host-parallel run begin their timed work together
        start.wait()
    t0 = time.perf_counter()
    n = 0
    while True:
        for u in units:
            b, h = divmod(u, w.kv_heads)
            for hq in range(h * g, (h + 1) * g):
                res = trees[u].route(Q64[b, hq], w.beam, flat=flats[u])
                for i in range(nq):
                    oracle.attend(Q64[b, hq, i], Kn[b, h], Vn[b, h], N, w.leaf_block, res["leaves"][i], w.scale)
                n += nq
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": n / el, "queries": n, "seconds": el, "units": len(units)}


def oracle_build_sample(w, N_build: int, N_final: int):
    """The fp64 oracle's build of one unit over N_build tokens and its append up to N_final
    (single thread): seconds of each."""
    import oracle
    from tree_indexed_sparse_build_b200 import synth

    wi = w.with_(batch=1, kv_heads=1, q_heads=w.group)
    Kn = synth.keys(wi, capacity=N_final)
    t0 = time.perf_counter()
    ot = oracle.OracleTree(w.head_dim, w.leaf_block, w.branching).build(Kn[0, 0], N_build)
    t1 = time.perf_counter()
    ot.append(Kn[0, 0], N_final)
    t2 = time.perf_counter()
    return {"build_s": t1 - t0, "append_s": t2 - t1}


def _replica(w, i):
    """A single-unit copy of workload w's shape with its own seed (host-parallel process i)."""
    return w.with_(batch=1, kv_heads=1, q_heads=w.group, seed=w.seed + 104729 * (i + 1))


def _host_parallel_worker(i, jobs, start, out):
    """One process of oracle_host_parallel: every job in turn on its own single-unit replica,
    each started together with the other processes."""
    for j, (kind, w, nq, N, seconds, max_steps) in enumerate(jobs):
        wi = _replica(w, i)
        try:
            if kind == "decode":
                r = oracle_decode_sample(wi, seconds=seconds, max_steps=max_steps, units=(0,), start=start)
            else:
                r = oracle_route_attend_sample(wi, seconds, nq, units=(0,), N=N, start=start)
            out.put((j, i, r["queries"], r["seconds"]))
        except Exception as e:  # report and keep the barrier count right for the others
            out.put((j, i, None, repr(e)))
            try:
                start.wait()
            except Exception:
                pass


def oracle_host_parallel(jobs, timeout_s: float = 300.0):
    """The fp64 oracle on every host core: one process per core (spawned, so safe after CUDA
    initialisation), each a single-threaded oracle working on its own single-unit replica of
    each job's workload.  jobs: (kind, workload, nq, N, seconds, max_steps) with kind "decode"
    (append + route + attend steps) or "route_attend" (prebuilt tree).  Setup is untimed; the
    processes start each job's timed work together.  Per job: rate = all processes' queries /
    the slowest process's time."""
    import multiprocessing as mp
    import queue as _queue

    cores = os.cpu_count() or 1
    n = min(cores, 64)
    ctx = mp.get_context("spawn")
    start = ctx.Barrier(n, timeout=timeout_s)
    out = ctx.Queue()
    procs = [ctx.Process(target=_host_parallel_worker, args=(i, jobs, start, out)) for i in range(n)]
    for p in procs:
        p.start()
    res = []
    deadline = time.time() + timeout_s + sum(j[4] for j in jobs) * 2
    while len(res) < n * len(jobs):
        try:
            res.append(out.get(timeout=5))
        except _queue.Empty:
            if time.time() > deadline or any(p.exitcode not in (None, 0) for p in procs):
                for p in procs:
                    if p.is_alive():
                        p.terminate()
                raise RuntimeError("host-parallel oracle processes failed or timed out")
    for p in procs:
        p.join(timeout=60)
    per_job = []
    for j in range(len(jobs)):
        rows = [r for r in res if r[0] == j]
        bad = [r for r in rows if r[2] is None]
        if bad:
            per_job.append({"value": None, "error": bad[0][3]})
            continue
        q = sum(r[2] for r in rows)
        t = max(r[3] for r in rows)
        per_job.append({"value": q / t, "queries": q, "seconds": t, "processes": n, "cores": cores})
    return per_job


# ----------------------------------------------------------------------------- main

def workload_config(w):
    return {"workload": f"{w.name}: decode steps (append 1 token, route, attend) over a "
                        f"{w.seq_len}-token bf16 cache",
            "batch": w.batch, "kv_heads": w.kv_heads, "q_heads": w.q_heads,
            "head_dim": w.head_dim, "seq_len": w.seq_len, "branching": w.branching,
            "leaf_block": w.leaf_block, "beam": w.beam, "nq": 1, "kv_dtype": "bf16",
            "out_dtype": "bf16",
            "l2": f"flushed between steps ({FLUSH_BYTES >> 20} MiB memset outside the timed events)",
            "inputs": "seeded synthetic: K ~ N(0,1) + rank-8 positional drift, V, Q ~ N(0,1)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=61)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-1m", action="store_true")
    ap.add_argument("--no-build", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the 128K variants (bf16 summaries, append buffer) and the 1M bf16-summary run")
    ap.add_argument("--profile-case", choices=["deep_1m_2kv", "deep_1m_2kv_q256"], default=None,
                    help="run only a small case for ncu captures: the 1M-token tree at 2 of its "
                         "8 KV heads, zha_decode, eager launches; 64 queries per head (1,024), or "
                         "256 per head (4,096: the full batch's queries per SM)")
    ap.add_argument("--mode", choices=["step", "decode", "two_call"], default="step",
                    help="decode step calls: zha_decode_step (one launch); zha_tree_append + "
                         "zha_decode; zha_tree_append + zha_route + zha_sparse_attn_decode")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--shard", choices=["replicas", "units"], default="replicas",
                    help="N GPUs: independent replicas of the 128K workload (weak scaling), or one "
                         "128K workload split over the ranks by (batch, KV head) unit with the "
                         "outputs all-gathered every step (strong scaling)")
    ap.add_argument("--eager", action="store_true",
                    help="launch the same kernels without CUDA graphs (for profilers)")
    args = ap.parse_args()
    K, W = args.steps, args.warmup

    from tree_indexed_sparse_build_b200 import ranks, workloads
    w = workloads.get("decode_128k")
    ri = ranks.rank_info()
    rank, world, local = ri.rank, ri.world, ri.local

    if args.impl == "reference":
        if rank != 0:
            return
        r = oracle_decode_sample(w, seconds=1e9, max_steps=K, warmup=W, units=(0,))
        t = float(np.sum(r["per_step_s"]))
        qps = r["queries"] / t
        line = {"impl": "reference", "metric": METRIC, "value": qps, "unit": UNIT, "n_gpus": args.gpus,
                "steps": K, "warmup": W, "ms_per_step": 1e3 * t / max(r["steps"], 1),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": workload_config(w),
                "cpu_baseline": {"value": qps, "unit": UNIT, "cores": 1, "kind": "oracle",
                                 "sample": f"1 (batch, KV head) unit, {r['steps']} decode steps x "
                                           f"{w.group} query heads, single-threaded fp64 C oracle"},
                "e2e": {"value": qps, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if args.profile_case:
        print(json.dumps(run_profile_case(args.profile_case, W, K)))
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def barrier():
        ranks.barrier(world)

    def max_over_ranks(x: float) -> float:
        return ranks.max_over_ranks(x, world, dev)

    sampler = lambda: ClockSampler(local)  # noqa: E731

    if args.shard == "units":
        barrier()
        with sampler() as smp:
            rs = run_decode_split(w, W, K, rank, world, dev, flush)
        step_ms = max_over_ranks(float(rs["step_ms"].mean()))
        q = w.batch * w.q_heads
        if rank == 0:
            cfg = dict(workload_config(w), parallelism=f"units{world}",
                       split="each rank decodes a contiguous range of the 32 (batch, KV head) units; "
                             "outputs all-gathered into unit order every step")
            print(json.dumps({"metric": METRIC, "value": q / (step_ms * 1e-3), "unit": UNIT, "n_gpus": world,
                              "steps": K, "warmup": W, "ms_per_step": step_ms, "higher_is_better": True,
                              "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                              "config": cfg, "units_rank0": rs["units"], "parity_rank0": rs["parity"],
                              "clocks": smp.summary(), "launch": "one CUDA graph per step (zha_decode_step) "
                              "+ an eager all-gather of O, events on the same stream"}))
        if world > 1:
            dist.destroy_process_group()
        return

    barrier()
    torch.cuda.synchronize()
    r = run_decode(w, W, K, rank, dev, flush, sampler, eager=args.eager, mode=args.mode)
    torch.cuda.synchronize()
    barrier()

    peak, peak_kind = hbm_peak()
    step_ms = max_over_ranks(float(r["step_ms"].mean()))
    qps = ranks.weak_scaling_rate(r["queries_per_step"], world, step_ms)
    e2e_ms = max_over_ranks(r["e2e_ms_per_step"])
    # the dominant launch: append + route + attention in one kernel (mode "step"), route +
    # attention in one kernel (mode "decode"), or the route and attention calls together
    dec_ms = float(r["decode_ms"].mean())
    fused_append = args.mode == "step"
    dec_bytes = r["route_bytes"] + r["attend_bytes"] + (r["append_bytes"] if fused_append else 0)
    dom_kernel = {"step": "route_group_kernel (fused append + route + attention)",
                  "decode": "route_group_kernel (fused route + attention)",
                  "two_call": "route_group_kernel (route) + attend_kernel"}[args.mode]
    kern = {"decode": {"ms": dec_ms, "bytes": int(dec_bytes), "gbs": dec_bytes / (dec_ms * 1e-3) / 1e9,
                       "route_bytes": int(r["route_bytes"]), "attend_bytes": int(r["attend_bytes"]),
                       "append_bytes": int(r["append_bytes"]), "includes_append": fused_append},
            "append": {"ms": float(r["append_ms"].mean()), "separate_launch": not fused_append}}
    dom = "decode"
    ra_bytes = r["route_bytes"] + r["attend_bytes"]
    ra_ms = dec_ms
    line = {
        "metric": METRIC, "value": qps, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w),
        "roofline": {"bound": "hbm", "kernel": dom_kernel, "achieved": kern[dom]["gbs"],
                     "peak": peak, "unit": "GB/s", "frac": kern[dom]["gbs"] / peak,
                     "traffic": kernel_traffic({"step": "decode_step_fused", "decode": "decode_fused"}.get(args.mode, "")),
                     "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": kern[dom]["bytes"]},
        "route_attend": {"gbs": ra_bytes / (ra_ms * 1e-3) / 1e9, "frac": ra_bytes / (ra_ms * 1e-3) / 1e9 / peak,
                         "ms": ra_ms, "bytes": int(ra_bytes)},
        "kernels": kern,
        "keys_per_query": r["keys_per_query"], "summaries_per_query": r["summaries_per_query"],
        "e2e": {"value": r["queries_per_step"] * world / (e2e_ms * 1e-3), "unit": UNIT,
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": r["h2d_bytes_per_step"],
                "d2h_bytes_per_step": r["d2h_bytes_per_step"],
                "launch": "one CUDA graph per step: H2D of the step's K/V rows (one 2-D copy per cache "
                          "into its strided rows) and query from pinned memory, zha_decode_step, D2H of "
                          "O; host synchronizes every step"},
        "e2e_eager": {"value": r["queries_per_step"] * world / (max_over_ranks(r["e2e_eager_ms_per_step"]) * 1e-3),
                      "unit": UNIT, "ms_per_step": max_over_ranks(r["e2e_eager_ms_per_step"]),
                      "launch": "the same calls issued eagerly each step"},
        "gpu_launches": int(round(r["launches_per_step"] * K)),
        "launch_mode": "eager" if args.eager else "cuda_graph_per_step",
        "decode_call": {"step": "zha_decode_step (append + route + attention, one launch)",
                        "decode": "zha_tree_append + zha_decode",
                        "two_call": "zha_tree_append + zha_route + zha_sparse_attn_decode"}[args.mode],
        "clocks": r["clocks"],
    }

    line["parity"] = r["parity"]

    def ctx_1m(m):
        one = {}
        for mode in ("throughput", "single"):
            x = m[mode]
            ms = max_over_ranks(float(x["step_ms"].mean()))
            byts = x["route_bytes"] + x["attend_bytes"]
            one[mode] = {"qps": x["queries_per_step"] * world / (ms * 1e-3), "ms_per_step": ms,
                         "route_ms": float(x["route_ms"].mean()), "attend_ms": float(x["attend_ms"].mean()),
                         "route_attend_gbs": byts / (ms * 1e-3) / 1e9,
                         "frac_of_peak": byts / (ms * 1e-3) / 1e9 / peak,
                         "route_gbs": x["route_bytes"] / (x["route_ms"].mean() * 1e-3) / 1e9,
                         "attend_gbs": x["attend_bytes"] / (x["attend_ms"].mean() * 1e-3) / 1e9,
                         "bytes_per_step": int(byts), "keys_per_query": x["keys_per_query"],
                         "summaries_per_query": x["summaries_per_query"],
                         "queries_per_step": x["queries_per_step"], "parity": x["parity"]}
        one["dense_bytes_per_step"] = m["dense_bytes_per_step"]
        one["workload"] = ("deep_1m: 1 x 8 KV heads x 64 query heads, d 128, 1,048,576 bf16 tokens, "
                           "b 8, leaf block 4, beam 8; throughput = 64 queries per head per step")
        one["launches_per_step"] = {k: m[k]["launches_per_step"] for k in ("throughput", "single")}
        one["needle_recall"] = m["needle_recall"]
        return one

    if not args.no_extras:
        # the same 128K decode steps over bf16-stored summaries (device-timed pass only)
        rb = run_decode(w, W, K, rank, dev, flush, sampler, eager=args.eager, mode=args.mode,
                        summary_dtype=torch.bfloat16, e2e=False)
        ms_b = max_over_ranks(float(rb["step_ms"].mean()))
        dec_b = rb["route_bytes"] + rb["attend_bytes"] + (rb["append_bytes"] if fused_append else 0)
        line["decode_128k_bf16_summaries"] = {
            "qps": ranks.weak_scaling_rate(rb["queries_per_step"], world, ms_b), "ms_per_step": ms_b,
            "decode_kernel_ms": float(rb["decode_ms"].mean()),
            "decode_kernel_gbs": dec_b / (float(rb["decode_ms"].mean()) * 1e-3) / 1e9,
            "decode_kernel_bytes": int(dec_b), "route_bytes": int(rb["route_bytes"]),
            "summaries_per_query": rb["summaries_per_query"], "clocks": rb["clocks"], "parity": rb["parity"]}

        # the same 128K steps with an append buffer (decode reads the buffer; commits overlap)
        bu = run_buffered(w, W, K, rank, dev, flush, eager=args.eager)
        line["decode_128k_buffered"] = {
            "qps": ranks.weak_scaling_rate(w.batch * w.q_heads, world, max_over_ranks(bu["ms_per_step"])), **bu,
            "call": "zha_decode_buffered per step; zha_tree_append of 2 leaves on a second stream when full"}

    if not args.no_build and rank == 0:
        line["tiny_fp32"] = run_small("tiny_fp32", W, K, dev, flush)
        line["gqa_32k"] = run_small("gqa_32k", W, K, dev, flush)
        line["build_256k"] = run_build_256k(W, K, dev, flush)
        line["causal"] = run_causal(W, min(K, 10), dev, flush)
        line["needle_recall"] = run_needles(dev)
        line["threshold"] = run_threshold(W, min(K, 10), dev, flush)

    if not args.no_1m:
        line["ctx_1m"] = ctx_1m(run_1m(W, K, rank, dev, flush, eager=args.eager))
        if not args.no_extras:
            # the same step over bf16-stored summaries (half the route's bytes; routing then
            # follows the bf16 tree, so the leaf sets may differ from the fp32 tree's)
            line["ctx_1m_bf16_summaries"] = ctx_1m(run_1m(W, K, rank, dev, flush, eager=args.eager,
                                                          summary_dtype=torch.bfloat16))

    oracle_1c, oracle_hp = {}, {}
    if rank == 0 and world == 1:
        try:
            cb = oracle_decode_sample(w, seconds=args.cpu_seconds, max_steps=64,
                                      units=tuple(range(8)))
            line["cpu_baseline"] = {"value": cb["value"], "unit": UNIT, "cores": 1, "kind": "oracle",
                                    "sample": f"{cb['units']} (batch, KV head) unit(s) x {cb['steps']} "
                                              f"decode steps x {w.group} query heads of decode_128k, "
                                              "single-threaded fp64 C oracle"}
            oracle_1c["decode_128k"] = cb["value"]
        except Exception as e:  # the baseline must never sink the GPU number
            line["cpu_baseline"] = {"value": None, "unit": UNIT, "cores": 1, "kind": "oracle",
                                    "sample": f"failed: {e}"}
        if args.cpu_seconds > 0:
            sec = max(1.0, args.cpu_seconds / 5)
            from tree_indexed_sparse_build_b200 import workloads as _wl
            ra_jobs = {"tiny_fp32": (_wl.get("tiny_fp32"), 16, None),
                       "gqa_32k": (_wl.get("gqa_32k"), 1, None),
                       "deep_1m": (_wl.get("deep_1m"), _wl.THROUGHPUT_NQ, None),
                       "build_256k": (_wl.get("build_256k"), 64, _wl.get("build_256k").capacity)}
            detail = {}
            for name, (wj, nqj, Nj) in ra_jobs.items():
                try:
                    r1 = oracle_route_attend_sample(wj, sec, nqj, units=(0,), N=Nj)
                    oracle_1c[name] = r1["value"]
                    detail[name] = {"qps": r1["value"], "queries": r1["queries"], "seconds": r1["seconds"]}
                except Exception as e:
                    detail[name] = {"qps": None, "error": repr(e)}
            try:
                wb = _wl.get("build_256k")
                bs = oracle_build_sample(wb, wb.seq_len, wb.capacity)
                rows = sum(level_counts(wb.seq_len, wb.leaf_block, wb.branching))
                detail["build_256k"].update({"build_s_per_unit": bs["build_s"], "append_4096_s_per_unit": bs["append_s"],
                                             "build_gbs": (wb.seq_len * wb.head_dim * 2 + rows * wb.head_dim * 4)
                                             / bs["build_s"] / 1e9})
            except Exception as e:
                detail["build_256k"]["build_error"] = repr(e)
            line["oracle_1core"] = {"kind": "oracle", "cores": 1, "seconds_per_config": sec,
                                    "what": "route + attention of every query of one (batch, KV head) unit over "
                                            "its prebuilt tree (decode_128k: cpu_baseline's decode steps)",
                                    **detail}
            try:
                jobs = [("route_attend", _wl.get("tiny_fp32"), 16, None, sec, 0),
                        ("route_attend", _wl.get("gqa_32k"), 1, None, sec, 0),
                        ("decode", w, 1, None, sec, 64),
                        ("route_attend", _wl.get("deep_1m"), _wl.THROUGHPUT_NQ, None, sec, 0),
                        ("route_attend", _wl.get("build_256k"), 64, _wl.get("build_256k").capacity, sec, 0)]
                names = ["tiny_fp32", "gqa_32k", "decode_128k", "deep_1m", "build_256k"]
                hp = oracle_host_parallel(jobs)
                oracle_hp = {n: h.get("value") for n, h in zip(names, hp)}
                line["cpu_baseline_host_parallel"] = {
                    "value": hp[2].get("value"), "unit": UNIT, "cores": hp[2].get("processes"),
                    "host_cores": hp[2].get("cores"), "kind": "oracle",
                    "sample": "one spawned process per host core, each a single-threaded fp64 C oracle on its "
                              "own single-unit replica (own seed) of each workload; value = decode_128k",
                    "per_config": dict(zip(names, hp))}
            except Exception as e:
                line["cpu_baseline_host_parallel"] = {"value": None, "sample": f"failed: {e}"}

    if rank == 0:
        line["configs"] = config_summary(line, oracle_1c, oracle_hp)
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


def config_summary(line, oracle_1c, oracle_hp):
    """The five workloads in one short object (it ends the JSON line): GPU queries/s, time per
    call, fraction of the measured HBM peak on algorithmic bytes, keys read per query, the
    parity sample in one phrase, and the oracle's queries/s on 1 core and on every host core."""
    def r(x, n=3):
        return None if x is None else float(f"{x:.{n}g}")

    out = {}
    o1, oh = oracle_1c or {}, oracle_hp or {}
    for name in ("tiny_fp32", "gqa_32k"):
        x = line.get(name)
        if x:
            out[name] = {"qps": r(x["qps"]), "us": r(x["ms"] * 1e3), "frac": r(x["frac_of_peak"], 2),
                         "keys_q": r(x["keys_per_query"]), "parity": parity_brief(x["parity"]),
                         "oracle_qps": [r(o1.get(name)), r(oh.get(name))]}
    ro = line.get("roofline", {})
    out["decode_128k"] = {"qps": r(line.get("value")), "us": r(line.get("ms_per_step", 0) * 1e3),
                          "frac": r(ro.get("frac"), 2), "keys_q": r(line.get("keys_per_query")),
                          "parity": parity_brief(line.get("parity")),
                          "oracle_qps": [r(o1.get("decode_128k")), r(oh.get("decode_128k"))]}
    for key, tag in (("ctx_1m", "deep_1m"), ("ctx_1m_bf16_summaries", "deep_1m_bf16sum")):
        x = line.get(key)
        if x:
            t, s1 = x["throughput"], x["single"]
            out[tag] = {"qps": r(t["qps"]), "us": r(t["ms_per_step"] * 1e3), "frac": r(t["frac_of_peak"], 2),
                        "single_us": r(s1["ms_per_step"] * 1e3), "keys_q": r(t["keys_per_query"]),
                        "parity": parity_brief(t["parity"])}
            if tag == "deep_1m":
                out[tag]["oracle_qps"] = [r(o1.get("deep_1m")), r(oh.get("deep_1m"))]
    x = line.get("build_256k")
    if x:
        out["build_256k"] = {"build_gbs": r(x["build_gbs"]), "append_us": r(x["append_4096_ms"] * 1e3),
                             "qps": r(x["qps"]), "parity": parity_brief(x.get("parity")),
                             "oracle_qps": [r(o1.get("build_256k")), r(oh.get("build_256k"))]}
    return out


if __name__ == "__main__":
    main()
