"""fp64 oracle for tree-indexed sparse decode attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, nothing else.  It shares no code
with the CUDA path (``tree_indexed_sparse_build_b200``) and never imports it.

The arithmetic lives in ``zha_oracle.c`` (plain single-threaded fp64 C); this
module only marshals numpy arrays and composes the per-level C routines into
the tree operations:

* ``OracleTree.build``   -- leaf means, then parent means level by level up to
  a single root (ZHA abstract: "a tree of recursively compressed key
  summaries over the KV cache").
* ``OracleTree.append``  -- recompute the leaves that received tokens and every
  ancestor of them, growing the depth when the leaves outgrow b^L (ZHA
  abstract: "iteratively growing the tree's depth").
* ``OracleTree.route``   -- top-down beam descent, top-B per level by
  (score desc, index asc) (ZHA abstract: "future queries traverse from the top
  down to retrieve a sparse subset of keys").
* ``attend`` / ``dense`` -- exact softmax attention over the selected leaves'
  tokens / over all tokens (ZHA abstract: "final attention").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zha_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

F32, BF16 = 0, 1

_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def build_library(force: bool = False) -> str:
    """Compile zha_oracle.c into liboracle.so (gcc, IEEE fp64, no contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
             _SRC, "-o", _LIB_PATH, "-lm"])
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build_library()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.orc_num_leaves.restype = _I64
        lib.orc_num_leaves.argtypes = [_I64, _I64]
        lib.orc_num_levels.restype = ctypes.c_int
        lib.orc_num_levels.argtypes = [_I64, _I64]
        lib.orc_leaf_means.restype = None
        lib.orc_leaf_means.argtypes = [_P, ctypes.c_int, _I64, _I64, _I64, _I64, _I64, _P]
        lib.orc_parent_means.restype = None
        lib.orc_parent_means.argtypes = [_P, _I64, _I64, _I64, _I64, _I64, _P]
        lib.orc_route.restype = ctypes.c_int
        lib.orc_route.argtypes = [_P, _P, _P, ctypes.c_int, _I64, _I64, _P, _I64, _I64,
                                  _P, _P, _P, _P, _P]
        lib.orc_attend.restype = _I64
        lib.orc_attend.argtypes = [_P, _P, _P, ctypes.c_int, _I64, _I64, _I64, _P, _I64,
                                   ctypes.c_double, _P]
        lib.orc_dense.restype = None
        lib.orc_dense.argtypes = [_P, _P, _P, ctypes.c_int, _I64, _I64, ctypes.c_double, _P]
        lib.orc_leaf_radii.restype = None
        lib.orc_leaf_radii.argtypes = [_P, ctypes.c_int, _I64, _I64, _I64, _P, _I64, _P]
        lib.orc_parent_radii.restype = None
        lib.orc_parent_radii.argtypes = [_P, _P, _I64, _P, _I64, _I64, _I64, _P]
        lib.orc_threshold_brute.restype = _I64
        lib.orc_threshold_brute.argtypes = [_P, ctypes.c_int, _I64, _I64, _P, ctypes.c_double, _P, _I64]
        lib.orc_round_bf16.restype = None
        lib.orc_round_bf16.argtypes = [_P, _I64]
        lib.orc_threshold_descent.restype = _I64
        lib.orc_threshold_descent.argtypes = [_P, _P, _P, _P, ctypes.c_int, _I64, _I64, _I64, _I64, _P,
                                              ctypes.c_int, _P, ctypes.c_double, _P, _I64, _P]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _kv_view(K: np.ndarray):
    """(array, dtype code) for a [tokens, d] slice stored as fp32 or bf16 bits (uint16)."""
    K = np.ascontiguousarray(K)
    if K.dtype == np.float32:
        return K, F32
    if K.dtype == np.uint16:
        return K, BF16
    raise TypeError(f"keys/values must be float32 or bf16 bits (uint16), got {K.dtype}")


def num_leaves(N: int, lb: int) -> int:
    return int(_load().orc_num_leaves(N, lb))


def num_levels(n0: int, b: int) -> int:
    return int(_load().orc_num_levels(n0, b))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """The stored value of each element under bf16 summary storage: nearest fp32 (ties to
    even), then nearest bf16 (ties to even), as fp64 (orc_round_bf16)."""
    out = np.array(x, dtype=np.float64, copy=True, order="C")
    if out.size:
        _load().orc_round_bf16(_ptr(out), out.size)
    return out


class OracleTree:
    """Tree of mean key summaries over one (batch, KV-head) slice, in fp64.

    ``levels[l]`` is an ``[n_l, d]`` fp64 array; ``levels[0]`` are the leaves
    and ``levels[L]`` the single root.

    ``summary="f64"`` keeps every summary exact (the reference for fp32-stored trees);
    ``summary="bf16"`` mirrors bf16 storage: every node computed is replaced by its stored
    value (``round_bf16``) before its parent averages it.
    """

    def __init__(self, d: int, leaf_block: int, branching: int, summary: str = "f64"):
        if leaf_block < 1 or branching < 2:
            raise ValueError("leaf_block >= 1 and branching >= 2 required")
        if summary not in ("f64", "bf16"):
            raise ValueError("summary must be 'f64' or 'bf16'")
        self.d, self.lb, self.b = d, leaf_block, branching
        self.summary = summary
        self.N = 0
        self.levels: list[np.ndarray] = []

    def _store(self, x):
        return round_bf16(x) if self.summary == "bf16" else x

    @property
    def L(self) -> int:
        return len(self.levels) - 1 if self.levels else 0

    def _leaf_means(self, K, N, i0, i1):
        K, dt = _kv_view(K)
        out = np.empty((max(i1 - i0, 0), self.d), np.float64)
        if i1 > i0:
            _load().orc_leaf_means(_ptr(K), dt, self.d, N, self.lb, i0, i1, _ptr(out))
        return self._store(out)

    def _parent_means(self, child, i0, i1):
        child = np.ascontiguousarray(child, dtype=np.float64)
        out = np.empty((max(i1 - i0, 0), self.d), np.float64)
        if i1 > i0:
            _load().orc_parent_means(_ptr(child), child.shape[0], self.d, self.b, i0, i1, _ptr(out))
        return self._store(out)

    def build(self, K: np.ndarray, N: int) -> "OracleTree":
        """Summaries of tokens [0, N) of K ([>=N, d])."""
        self.N = N
        n0 = num_leaves(N, self.lb)
        self.levels = []
        if n0 == 0:
            return self
        self.levels.append(self._leaf_means(K, N, 0, n0))
        L = num_levels(n0, self.b)
        for _ in range(L):
            child = self.levels[-1]
            n = -(-child.shape[0] // self.b)
            self.levels.append(self._parent_means(child, 0, n))
        assert self.levels[-1].shape[0] == 1
        return self

    def append(self, K: np.ndarray, new_N: int) -> "OracleTree":
        """Extend to tokens [0, new_N): recompute touched leaves and their ancestors."""
        if new_N < self.N:
            raise ValueError("append cannot shrink the cache")
        if new_N == self.N:
            return self
        if self.N == 0:
            return self.build(K, new_N)
        lo = self.N // self.lb
        hi = (new_N - 1) // self.lb
        n0 = hi + 1
        leaves = np.empty((n0, self.d), np.float64)
        leaves[:lo] = self.levels[0][:lo]
        leaves[lo:] = self._leaf_means(K, new_N, lo, n0)
        new_levels = [leaves]
        L = num_levels(n0, self.b)
        for lvl in range(1, L + 1):
            child = new_levels[-1]
            n = -(-child.shape[0] // self.b)
            lo //= self.b
            hi //= self.b
            cur = np.empty((n, self.d), np.float64)
            if lvl < len(self.levels):
                keep = min(lo, self.levels[lvl].shape[0])
                cur[:keep] = self.levels[lvl][:keep]
            else:
                keep = 0
            assert keep == lo, "untouched prefix must already exist"
            cur[lo:hi + 1] = self._parent_means(child, lo, hi + 1)
            new_levels.append(cur)
        self.levels = new_levels
        self.N = new_N
        assert self.levels[-1].shape[0] == 1
        return self

    def flat(self):
        """(rows, offsets, counts): all levels stacked, level l at rows [off[l], off[l]+cnt[l])."""
        cnt = np.array([lv.shape[0] for lv in self.levels], np.int64)
        off = np.concatenate([[0], np.cumsum(cnt)[:-1]]).astype(np.int64)
        return np.ascontiguousarray(np.concatenate(self.levels, axis=0)), off, cnt

    def radii(self, K: np.ndarray) -> list[np.ndarray]:
        """Bounding-sphere radius of every node, per level (centers = the summaries): leaves
        cover their tokens, a parent covers its children's spheres (orc_leaf_radii,
        orc_parent_radii)."""
        Kv, dt = _kv_view(K)
        lib = _load()
        out = [np.empty(self.levels[0].shape[0], np.float64)]
        c0 = np.ascontiguousarray(self.levels[0])
        lib.orc_leaf_radii(_ptr(Kv), dt, self.d, self.N, self.lb, _ptr(c0), c0.shape[0], _ptr(out[0]))
        for lvl in range(1, self.L + 1):
            cc = np.ascontiguousarray(self.levels[lvl - 1])
            pc = np.ascontiguousarray(self.levels[lvl])
            r = np.empty(pc.shape[0], np.float64)
            lib.orc_parent_radii(_ptr(cc), _ptr(out[-1]), cc.shape[0], _ptr(pc), pc.shape[0], self.d, self.b,
                                 _ptr(r))
            out.append(r)
        return out

    def threshold(self, K: np.ndarray, q: np.ndarray, tau: float, radii=None, max_out: int | None = None):
        """Threshold descent: (tokens t < N with q . k_t >= tau, ascending; sphere tests)."""
        Kv, dt = _kv_view(K)
        q = np.ascontiguousarray(q, dtype=np.float64).reshape(-1)
        radii = radii if radii is not None else self.radii(K)
        rows, off, cnt = self.flat()
        rad = np.ascontiguousarray(np.concatenate(radii))
        cap = self.N if max_out is None else max_out
        out = np.empty(max(cap, 1), np.int64)
        tested = np.zeros(1, np.int64)
        n = _load().orc_threshold_descent(_ptr(rows), _ptr(rad), _ptr(off), _ptr(cnt), self.L, self.d, self.b,
                                          self.lb, self.N, _ptr(Kv), dt, _ptr(q), float(tau), _ptr(out), cap,
                                          _ptr(tested))
        return out[:min(n, cap)].copy(), int(tested[0])

    def route(self, Q: np.ndarray, beam: int, flat=None):
        """Beam descent for queries Q ([nq, d], any float dtype, converted to fp64).

        Returns a dict with ``leaves`` [nq, beam] (ascending, -1 padded),
        ``leaf_scores`` [nq, beam], ``bounds`` [nq, L, 2] (s_(B), s_(B+1) per
        level, levels L-1 .. 0, NaN where a level has <= B candidates),
        ``survivors`` [nq, L, beam] and ``ncand`` [nq, L].
        """
        Q = np.ascontiguousarray(np.atleast_2d(Q), dtype=np.float64)
        nq = Q.shape[0]
        L = self.L
        if L < 1:
            raise ValueError("route on an empty tree")
        rows, off, cnt = flat if flat is not None else self.flat()
        leaves = np.empty((nq, beam), np.int64)
        scores = np.empty((nq, beam), np.float64)
        bounds = np.empty((nq, L, 2), np.float64)
        surv = np.empty((nq, L, beam), np.int64)
        ncand = np.empty((nq, L), np.int64)
        rc = _load().orc_route(_ptr(rows), _ptr(off), _ptr(cnt), L, self.d, self.b, _ptr(Q), nq,
                               beam, _ptr(leaves), _ptr(scores), _ptr(bounds), _ptr(surv),
                               _ptr(ncand))
        if rc != 0:
            raise RuntimeError("orc_route failed")
        return {"leaves": leaves, "leaf_scores": scores, "bounds": bounds,
                "survivors": surv, "ncand": ncand}


def threshold_brute(q: np.ndarray, K: np.ndarray, N: int, tau: float) -> np.ndarray:
    """Every token t < N with q . k_t >= tau (fp64 scan of all keys), ascending."""
    Kv, dt = _kv_view(K)
    q = np.ascontiguousarray(q, dtype=np.float64).reshape(-1)
    out = np.empty(max(N, 1), np.int64)
    n = _load().orc_threshold_brute(_ptr(Kv), dt, q.shape[0], N, _ptr(q), float(tau), _ptr(out), N)
    return out[:n].copy()


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, N: int, leaf_block: int,
           leaves: np.ndarray, scale: float) -> tuple[np.ndarray, int]:
    """Exact softmax attention of one query over the selected leaves' tokens (t < N)."""
    q = np.ascontiguousarray(q, dtype=np.float64).ravel()
    K, dt = _kv_view(K)
    V, dt2 = _kv_view(V)
    assert dt == dt2
    leaves = np.ascontiguousarray(leaves, dtype=np.int64).ravel()
    out = np.empty(q.shape[0], np.float64)
    ntok = _load().orc_attend(_ptr(q), _ptr(K), _ptr(V), dt, q.shape[0], N, leaf_block,
                              _ptr(leaves), leaves.shape[0], scale, _ptr(out))
    return out, int(ntok)


def buffer_leaves(n_routed: int, n_tokens: int, lb: int) -> np.ndarray:
    """Leaves holding the buffered tokens n_routed .. n_tokens - 1 (n_routed a multiple of lb)."""
    return np.arange(n_routed // lb, -(-n_tokens // lb), dtype=np.int64)


def attend_buffered(q: np.ndarray, K: np.ndarray, V: np.ndarray, leaves: np.ndarray, n_routed: int,
                    n_tokens: int, lb: int, scale: float) -> tuple[np.ndarray, int]:
    """Decode with an append buffer ("Louver" explainer, dynamic updates: keys that arrive during
    decoding wait in a buffer the queries read directly): exact softmax attention over the
    tokens of the routed leaves (a route over the tree of the first n_routed tokens, so all of
    them lie before n_routed) together with every buffered token n_routed .. n_tokens - 1."""
    lv = np.asarray(leaves, dtype=np.int64).ravel()
    lv = lv[lv >= 0]
    return attend(q, K, V, n_tokens, lb, np.concatenate([lv, buffer_leaves(n_routed, n_tokens, lb)]), scale)


def dense(q: np.ndarray, K: np.ndarray, V: np.ndarray, N: int, scale: float) -> np.ndarray:
    """Exact softmax attention of one query over all tokens t < N."""
    q = np.ascontiguousarray(q, dtype=np.float64).ravel()
    K, dt = _kv_view(K)
    V, _ = _kv_view(V)
    out = np.empty(q.shape[0], np.float64)
    _load().orc_dense(_ptr(q), _ptr(K), _ptr(V), dt, q.shape[0], N, scale, _ptr(out))
    return out


def well_conditioned(bounds: np.ndarray, rel: float = 1e-3) -> np.ndarray:
    """Per query: True iff at every level with more than B candidates,
    s_(B) - s_(B+1) > rel * max(|s_(B)|, |s_(B+1)|) (the fp64 margin rule).

    ``bounds`` is the ``[nq, L, 2]`` array returned by ``OracleTree.route``.
    """
    sB, sB1 = bounds[..., 0], bounds[..., 1]
    ok = np.isnan(sB) | ((sB - sB1) > rel * np.maximum(np.abs(sB), np.abs(sB1)))
    return ok.all(axis=-1)
