"""Seeded synthetic KV caches and decode queries.

Draws only (see ``synth.c`` for the generator): no means, scores or softmax.
Both the CUDA path's tests/benchmark and the fp64 oracle take their inputs
from here.

Recipe (per workload, seed = ``Workload.seed``; one independent stream per
tensor; a value depends only on (seed, stream, counter), never on how large
the tensor is allocated):

* K, V: N(0, 1) per element, counter ``(unit << 40) + t*d + k`` where
  ``unit = b*H_kv + h``; streams 1 (K) and 2 (V).
* Q: N(0, 1), counter ``((b*H_q + h) << 24) + i*d + k``; stream 3.  Decode
  step s of a multi-step run uses stream 8, counter
  ``(s << 32) + ((b*H_q + h) << 16) + i*d + k``.
* Needles (planted keys): per unit, ``needles`` distinct positions drawn
  uniformly in [0, N) (stream 4, rejection of repeats); needle i is tied to
  query head ``h*g + (i mod g)``, query index ``(i // g) mod nq`` and set to
  ``amp * q_hat + sigma * z`` with q_hat = q / |q| of the stored query and
  z ~ N(0, I) (stream 5).
* Drift (decode_128k): ``K[t] += 0.5 * A_u f(t)``, ``A_u`` in R^{d x 8} with
  N(0, 1/8) entries (stream 6), ``f_j(t) = sin(2 pi t / P_j + phi_{u,j})``,
  ``P_j = 64 (N/64)^{j/7}``, ``phi`` uniform in [0, 2 pi) (stream 7).
* Everything is formed in fp64 and rounded once, round-to-nearest-even, to
  the storage type (fp32, or bf16 stored as uint16 bit patterns).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from ..workloads import Workload

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None

STREAM_K, STREAM_V, STREAM_Q, STREAM_NPOS, STREAM_NNOISE = 1, 2, 3, 4, 5
STREAM_DRIFT_A, STREAM_DRIFT_PHI, STREAM_STEP_Q = 6, 7, 8
STREAM_CLUSTER = 9  # cluster centers of clustered_keys

_U64, _I64, _P, _D = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_double


def build_library(force: bool = False) -> str:
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-shared", "-fPIC", "-pthread",
                               _SRC, "-o", _LIB_PATH, "-lm"])
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build_library()
        lib = ctypes.CDLL(_LIB_PATH)
        for nm in ("synth_normal_f64", "synth_normal_f32", "synth_normal_bf16"):
            f = getattr(lib, nm)
            f.restype = ctypes.c_int
            f.argtypes = [_U64, _U64, _U64, _I64, _D, _D, _P, ctypes.c_int]
        lib.synth_uniform_f64.restype = ctypes.c_int
        lib.synth_uniform_f64.argtypes = [_U64, _U64, _U64, _I64, _P, ctypes.c_int]
        lib.synth_round_bf16.restype = None
        lib.synth_round_bf16.argtypes = [_P, _I64, _P]
        lib.synth_round_f32.restype = None
        lib.synth_round_f32.argtypes = [_P, _I64, _P]
        lib.synth_drift_keys.restype = ctypes.c_int
        lib.synth_drift_keys.argtypes = [_U64, _U64, _U64, _I64, _I64, _I64, _D, _P, _P, _P, _P, _P,
                                         ctypes.c_int]
        _lib = lib
    return _lib


def _threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def normal(seed: int, stream: int, offset: int, n: int, dtype: str = "f64", std: float = 1.0,
           mean: float = 0.0) -> np.ndarray:
    """n normals at counters offset .. offset+n-1; dtype "f64", "f32" or "bf16" (uint16 bits)."""
    lib = _load()
    if dtype == "f64":
        out = np.empty(n, np.float64)
        lib.synth_normal_f64(seed, stream, offset, n, mean, std, _p(out), _threads())
    elif dtype == "f32":
        out = np.empty(n, np.float32)
        lib.synth_normal_f32(seed, stream, offset, n, mean, std, _p(out), _threads())
    elif dtype == "bf16":
        out = np.empty(n, np.uint16)
        lib.synth_normal_bf16(seed, stream, offset, n, mean, std, _p(out), _threads())
    else:
        raise ValueError(dtype)
    return out


def uniform(seed: int, stream: int, offset: int, n: int) -> np.ndarray:
    out = np.empty(n, np.float64)
    _load().synth_uniform_f64(seed, stream, offset, n, _p(out), _threads())
    return out


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64 values RNE to "f32" or "bf16" (uint16 bit patterns)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    if dtype == "f32":
        out = np.empty(x.shape, np.float32)
        _load().synth_round_f32(_p(x), x.size, _p(out))
    elif dtype == "bf16":
        out = np.empty(x.shape, np.uint16)
        _load().synth_round_bf16(_p(x), x.size, _p(out))
    else:
        raise ValueError(dtype)
    return out


def to_f64(x: np.ndarray) -> np.ndarray:
    """Exact widening of stored values (fp32, or bf16 bits in uint16) to fp64."""
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def queries(w: Workload, nq: int | None = None, step: int | None = None) -> np.ndarray:
    """Decode queries [B, H_q, nq, d] in the workload's storage type."""
    nq = w.nq if nq is None else nq
    d = w.head_dim
    out = np.empty((w.batch, w.q_heads, nq, d), np.uint16 if w.kv_dtype == "bf16" else np.float32)
    for b in range(w.batch):
        for h in range(w.q_heads):
            hq = b * w.q_heads + h
            if step is None:
                off, stream = (hq << 24), STREAM_Q
            else:
                off, stream = (step << 32) + (hq << 16), STREAM_STEP_Q
            out[b, h] = normal(w.seed, stream, off, nq * d, w.kv_dtype).reshape(nq, d)
    return out


def _needle_positions(w: Workload, unit: int, N: int) -> list[int]:
    pos: list[int] = []
    seen = set()
    ctr = unit << 20
    while len(pos) < min(w.needles, N):
        u = uniform(w.seed, STREAM_NPOS, ctr, 64)
        ctr += 64
        for x in u:
            p = int(x * N)
            if p not in seen:
                seen.add(p)
                pos.append(p)
                if len(pos) == min(w.needles, N):
                    break
    return pos


def needles(w: Workload, Q: np.ndarray) -> list[list[tuple[int, int, int]]]:
    """Per unit: list of (position, query head, query index) of its needles."""
    g, nq = w.group, Q.shape[2]
    res = []
    for b in range(w.batch):
        for h in range(w.kv_heads):
            u = b * w.kv_heads + h
            pos = _needle_positions(w, u, w.seq_len) if w.needles else []
            res.append([(p, h * g + (i % g), (i // g) % nq) for i, p in enumerate(pos)])
    return res


def _drift_params(w: Workload, unit: int):
    d, r = w.head_dim, 8
    A = normal(w.seed, STREAM_DRIFT_A, unit << 20, d * r, "f64", std=(1.0 / r) ** 0.5)
    phi = 2.0 * np.pi * uniform(w.seed, STREAM_DRIFT_PHI, unit << 20, r)
    P = 64.0 * (w.seq_len / 64.0) ** (np.arange(r) / (r - 1))
    return np.ascontiguousarray(A), np.ascontiguousarray(P), np.ascontiguousarray(phi)


def keys(w: Workload, capacity: int | None = None, Q: np.ndarray | None = None,
         units: list[int] | None = None) -> np.ndarray:
    """K cache [B, H_kv, capacity, d] (rows >= capacity not drawn).

    ``Q`` (from ``queries``) is needed when the workload plants needles.
    ``units`` restricts drawing to some flat (b*H_kv + h) units; the others are
    left zero.
    """
    cap = w.capacity if capacity is None else capacity
    d = w.head_dim
    dt = np.uint16 if w.kv_dtype == "bf16" else np.float32
    out = np.zeros((w.batch, w.kv_heads, cap, d), dt)
    flat = out.reshape(w.units, cap * d)
    todo = range(w.units) if units is None else units
    nd = needles(w, Q) if (w.needles and Q is not None) else None
    if w.needles and Q is None:
        raise ValueError("this workload plants needles: pass its queries")
    for u in todo:
        if w.drift:
            A, P, phi = _drift_params(w, u)
            row = flat[u]
            _load().synth_drift_keys(w.seed, STREAM_K, u << 40, cap, d, 8, 0.5, _p(A), _p(P),
                                     _p(phi), _p(row) if w.kv_dtype == "bf16" else None,
                                     _p(row) if w.kv_dtype == "f32" else None, _threads())
        else:
            flat[u] = normal(w.seed, STREAM_K, u << 40, cap * d, w.kv_dtype)
        if nd is not None:
            b = u // w.kv_heads
            for i, (p, hq, qi) in enumerate(nd[u]):
                q = to_f64(Q[b, hq, qi])
                qhat = q / np.linalg.norm(q)
                z = normal(w.seed, STREAM_NNOISE, (u << 20) + i * d, d, "f64")
                flat[u, p * d:(p + 1) * d] = round_to(w.needle_amp * qhat + w.needle_sigma * z,
                                                      w.kv_dtype)
    return out


def clustered_keys(w: Workload, spread: float, capacity: int | None = None) -> np.ndarray:
    """K cache [B, H_kv, capacity, d] whose tokens cluster in blocks of w.leaf_block
    consecutive tokens: K[t] = C[t // leaf_block] + spread * e_t, C and e ~ N(0, I) (streams
    STREAM_CLUSTER and STREAM_K), rounded once to the storage type."""
    cap = w.capacity if capacity is None else capacity
    d, lb = w.head_dim, w.leaf_block
    dt = np.uint16 if w.kv_dtype == "bf16" else np.float32
    out = np.zeros((w.batch, w.kv_heads, cap, d), dt)
    flat = out.reshape(w.units, cap, d)
    nblk = -(-cap // lb)
    for u in range(w.units):
        C = normal(w.seed, STREAM_CLUSTER, u << 40, nblk * d).reshape(nblk, d)
        e = normal(w.seed, STREAM_K, u << 40, cap * d).reshape(cap, d)
        flat[u] = round_to(np.repeat(C, lb, axis=0)[:cap] + spread * e, w.kv_dtype)
    return out


def values(w: Workload, capacity: int | None = None, units: list[int] | None = None) -> np.ndarray:
    """V cache [B, H_kv, capacity, d], N(0, 1)."""
    cap = w.capacity if capacity is None else capacity
    d = w.head_dim
    dt = np.uint16 if w.kv_dtype == "bf16" else np.float32
    out = np.zeros((w.batch, w.kv_heads, cap, d), dt)
    flat = out.reshape(w.units, cap * d)
    for u in (range(w.units) if units is None else units):
        flat[u] = normal(w.seed, STREAM_V, u << 40, cap * d, w.kv_dtype)
    return out


def to_torch(x: np.ndarray, device):
    """Move a stored array to a torch device; uint16 bf16 bit patterns become torch.bfloat16."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x))
    if x.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.to(device)
