"""Thin ctypes binding of libzha (include/zha.h).

The functions keep the C names and only marshal arguments: torch tensors become
device pointers, the current torch stream becomes the cudaStream_t.  Every step
of the computation runs in libzha's CUDA kernels; there is no other code path,
and importing this module fails loudly when libzha.so has not been built.

``Tree`` bundles a handle with a caller-owned workspace tensor for convenience.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzha.so")

ZHA_OK, ZHA_ERR_INVALID_ARG, ZHA_ERR_CAPACITY, ZHA_ERR_UNSUPPORTED = 0, 1, 2, 3
ZHA_ERR_CUDA, ZHA_ERR_TIMEOUT, ZHA_ERR_DEVICE = 4, 5, 6
ZHA_F32, ZHA_BF16 = 0, 1

EXPORTED = [
    "zha_tree_workspace_bytes", "zha_tree_init", "zha_tree_destroy", "zha_tree_build",
    "zha_tree_append", "zha_route", "zha_attn_scratch_bytes", "zha_sparse_attn_decode",
    "zha_tree_check", "zha_tree_seq_len", "zha_tree_levels", "zha_tree_level_nodes",
    "zha_tree_level_offset", "zha_tree_unit_rows", "zha_tree_summaries", "zha_tree_launch_count",
    "zha_status_string", "zha_sparse_attn_decode_noalloc", "zha_noalloc_scratch_capacity",
    "zha_decode", "zha_decode_step", "zha_route_causal", "zha_decode_causal",
    "zha_tree_radii_bytes", "zha_tree_attach_radii", "zha_threshold_route", "zha_decode_buffered",
    "zha_tree_get_desc", "zha_tree_device", "zha_tree_set_wait_limit",
]


class zha_tree_desc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("branching", ctypes.c_int), ("leaf_block", ctypes.c_int),
                ("capacity_tokens", ctypes.c_longlong), ("kv_dtype", ctypes.c_int),
                ("summary_dtype", ctypes.c_int)]


class ZhaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None
_P, _I, _LL, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """The loaded libzha.  Raises if the library is missing (build it first)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libzha.so not built at {LIB_PATH}; run "
                               "`python -m tree_indexed_sparse_build_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "zha_tree_workspace_bytes": (_SZ, [ctypes.POINTER(zha_tree_desc)]),
            "zha_tree_init": (_I, [ctypes.POINTER(zha_tree_desc), _P, _SZ, ctypes.POINTER(_P)]),
            "zha_tree_destroy": (_I, [_P]),
            "zha_tree_build": (_I, [_P, _P, _LL, _P]),
            "zha_tree_append": (_I, [_P, _P, _LL, _P]),
            "zha_route": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P]),
            "zha_attn_scratch_bytes": (_SZ, [_P, _I, _I, _I]),
            "zha_sparse_attn_decode": (_I, [_P, _P, _I, _I, _I, _P, _P, _P, _I, ctypes.c_float,
                                            _P, _I, _P, _SZ, _P]),
            "zha_sparse_attn_decode_noalloc": (_I, [_P, _P, _I, _I, _I, _P, _P, _P, _I,
                                                    ctypes.c_float, _P, _I, _P]),
            "zha_noalloc_scratch_capacity": (_SZ, []),
            "zha_decode": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, ctypes.c_float, _P, _P, _P, _P, _I,
                                _P]),
            "zha_decode_step": (_I, [_P, _P, _P, _LL, _P, _I, _I, _I, _I, ctypes.c_float, _P, _P, _P,
                                     _P, _I, _P]),
            "zha_route_causal": (_I, [_P, _P, _P, _I, _I, _I, _P, _I, _P, _P, _P, _P]),
            "zha_tree_radii_bytes": (_SZ, [_P]),
            "zha_tree_attach_radii": (_I, [_P, _P, _SZ, _P, _P]),
            "zha_threshold_route": (_I, [_P, _P, _P, _I, _I, _I, _P, _I, _P, _P, _P, _P]),
            "zha_decode_causal": (_I, [_P, _P, _I, _I, _I, _P, _I, _P, _P, ctypes.c_float, _P, _P, _P,
                                       _P, _I, _P]),
            "zha_decode_buffered": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _LL, _LL, ctypes.c_float, _P, _P,
                                         _P, _P, _I, _P]),
            "zha_tree_check": (_I, [_P, _P]),
            "zha_tree_seq_len": (_LL, [_P]),
            "zha_tree_levels": (_I, [_P]),
            "zha_tree_level_nodes": (_LL, [_P, _I]),
            "zha_tree_level_offset": (_LL, [_P, _I]),
            "zha_tree_unit_rows": (_LL, [_P]),
            "zha_tree_summaries": (_P, [_P]),
            "zha_tree_launch_count": (_LL, [_P]),
            "zha_tree_get_desc": (_I, [_P, ctypes.POINTER(zha_tree_desc)]),
            "zha_tree_device": (_I, [_P]),
            "zha_tree_set_wait_limit": (_I, [_P, _LL]),
            "zha_status_string": (ctypes.c_char_p, [_I]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().zha_status_string(status).decode()


def _check(status: int, where: str):
    if status != ZHA_OK:
        raise ZhaError(status, where)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libzha takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libzha takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _expect(t: torch.Tensor | None, what: str, numel: int, dtypes: tuple) -> None:
    """Refuse a buffer the library would read or write past, or read as another type: the C
    calls take plain pointers, so sizes are checked here (they follow from Q's shape)."""
    if t is None:
        return
    if t.dtype not in dtypes:
        raise ValueError(f"{what}: dtype {t.dtype}, expected {' or '.join(str(d) for d in dtypes)}")
    if t.numel() != numel:
        raise ValueError(f"{what}: {t.numel()} elements, expected {numel}")


_I32, _I64, _F32 = (torch.int32,), (torch.int64,), (torch.float32,)
_OUT = (torch.float32, torch.bfloat16)
_TORCH_DT = {ZHA_F32: torch.float32, ZHA_BF16: torch.bfloat16}


def zha_tree_get_desc(handle) -> zha_tree_desc:
    d = zha_tree_desc()
    _check(lib().zha_tree_get_desc(handle, ctypes.byref(d)), "zha_tree_get_desc")
    return d


def zha_tree_device(handle) -> int:
    return int(lib().zha_tree_device(handle))


def zha_tree_set_wait_limit(handle, cycles: int) -> None:
    """Test hook: bound the first wait for a kernel's copies to `cycles` SM clocks (0: default)."""
    _check(lib().zha_tree_set_wait_limit(handle, int(cycles)), "zha_tree_set_wait_limit")


def _check_q(handle, Q: torch.Tensor, what: str = "Q") -> None:
    """Refuse a query tensor that does not fit the tree: the kernels size their reads of Q,
    and their writes of every per-query output, from the tree's batch and head_dim and the
    call's q_heads and nq, so a Q of another batch or head_dim would be read past its end.
    (A null handle is left to the library, which refuses it.)"""
    if handle is None:
        return
    d = zha_tree_get_desc(handle)
    if Q.dim() != 4:
        raise ValueError(f"{what}: expected [batch, q_heads, nq, head_dim], got shape {tuple(Q.shape)}")
    if Q.dtype not in _OUT:
        raise ValueError(f"{what}: dtype {Q.dtype}, expected torch.float32 or torch.bfloat16")
    B, _, _, hd = Q.shape  # q_heads % kv_heads is checked by the library itself
    if B != d.batch or hd != d.head_dim:
        raise ValueError(f"{what}: shape {tuple(Q.shape)} does not fit the tree "
                         f"(batch {d.batch}, head_dim {d.head_dim})")


def _check_kv(handle, *caches) -> None:
    """Refuse a K or V cache of another type or size than the tree's
    [batch, kv_heads, capacity_tokens, head_dim] in kv_dtype (None entries are skipped): the
    kernels address rows by the tree's capacity, so any other size is read past or mis-strided."""
    if handle is None:
        return
    d = zha_tree_get_desc(handle)
    n = d.batch * d.kv_heads * d.capacity_tokens * d.head_dim
    for name, t in zip("KV", caches):
        if t is None:
            continue
        if t.dtype != _TORCH_DT[d.kv_dtype]:
            raise ValueError(f"{name}: dtype {t.dtype}, the tree's caches are {_TORCH_DT[d.kv_dtype]}")
        if t.numel() != n:
            raise ValueError(f"{name}: {t.numel()} elements, the tree's [batch, kv_heads, capacity, "
                             f"head_dim] cache has {n}")


def _route_buffers(handle, Q: torch.Tensor, beam: int, leaf_idx, leaf_score=None, trace=None,
                   O=None, appending: bool = False) -> None:
    """leaf_idx / leaf_score [batch, q_heads, nq, beam], trace [.., levels, beam], O like Q.
    appending: the call first appends, so the trace has the levels of the grown tree (at
    least the current ones)."""
    B, Hq, nq, _ = Q.shape
    n = B * Hq * nq * int(beam)
    _expect(leaf_idx, "leaf_idx", n, _I32)
    _expect(leaf_score, "leaf_score", n, _F32)
    _expect(O, "O", Q.numel(), _OUT)
    if trace is not None:
        L = max(zha_tree_levels(handle), 1)
        if not appending:
            _expect(trace, "trace", n * L, _I32)
        elif trace.dtype != torch.int32 or n == 0 or trace.numel() % n or trace.numel() // n < L:
            raise ValueError(f"trace: {trace.numel()} {trace.dtype} elements, expected int32 "
                             f"[batch, q_heads, nq, levels >= {L}, beam]")


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return ZHA_BF16
    if dt == torch.float32:
        return ZHA_F32
    raise ValueError(f"unsupported dtype {dt}")


# ---------------------------------------------------------------- C-named wrappers

def zha_tree_workspace_bytes(desc: zha_tree_desc) -> int:
    return int(lib().zha_tree_workspace_bytes(ctypes.byref(desc)))


def zha_tree_init(desc: zha_tree_desc, workspace: torch.Tensor) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(lib().zha_tree_init(ctypes.byref(desc), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), ctypes.byref(h)),
           "zha_tree_init")
    return h


def zha_tree_destroy(handle) -> None:
    _check(lib().zha_tree_destroy(handle), "zha_tree_destroy")


def zha_tree_build(handle, K: torch.Tensor, seq_len: int, stream=None) -> None:
    _check_kv(handle, K)
    _check(lib().zha_tree_build(handle, _ptr(K), seq_len, _stream(stream)), "zha_tree_build")


def zha_tree_append(handle, K: torch.Tensor, new_seq_len: int, stream=None) -> None:
    _check_kv(handle, K)
    _check(lib().zha_tree_append(handle, _ptr(K), new_seq_len, _stream(stream)), "zha_tree_append")


def zha_route(handle, Q: torch.Tensor, beam: int, leaf_idx: torch.Tensor,
              leaf_score: torch.Tensor | None = None, trace: torch.Tensor | None = None,
              stream=None) -> None:
    _check_q(handle, Q)
    B, Hq, nq, _ = Q.shape
    _route_buffers(handle, Q, beam, leaf_idx, leaf_score, trace)
    _check(lib().zha_route(handle, _ptr(Q), dtype_code(Q.dtype), Hq, nq, beam, _ptr(leaf_idx),
                           _ptr(leaf_score), _ptr(trace), _stream(stream)), "zha_route")


def zha_attn_scratch_bytes(handle, q_heads: int, nq: int, beam: int) -> int:
    return int(lib().zha_attn_scratch_bytes(handle, q_heads, nq, beam))


def zha_sparse_attn_decode(handle, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                           leaf_idx: torch.Tensor, beam: int, scale: float, O: torch.Tensor,
                           scratch: torch.Tensor | None = None, stream=None) -> None:
    _check_q(handle, Q)
    B, Hq, nq, _ = Q.shape
    _check_kv(handle, K, V)
    _route_buffers(handle, Q, beam, leaf_idx, O=O)
    nbytes = 0 if scratch is None else scratch.numel() * scratch.element_size()
    _check(lib().zha_sparse_attn_decode(handle, _ptr(Q), dtype_code(Q.dtype), Hq, nq, _ptr(K),
                                        _ptr(V), _ptr(leaf_idx), beam, scale, _ptr(O),
                                        dtype_code(O.dtype), _ptr(scratch), nbytes,
                                        _stream(stream)), "zha_sparse_attn_decode")


def zha_sparse_attn_decode_noalloc(handle, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                                   leaf_idx: torch.Tensor, beam: int, scale: float,
                                   O: torch.Tensor, stream=None) -> None:
    """zha_sparse_attn_decode with the library's own fixed scratch (no caller buffer)."""
    _check_q(handle, Q)
    B, Hq, nq, _ = Q.shape
    _check_kv(handle, K, V)
    _route_buffers(handle, Q, beam, leaf_idx, O=O)
    _check(lib().zha_sparse_attn_decode_noalloc(handle, _ptr(Q), dtype_code(Q.dtype), Hq, nq,
                                                _ptr(K), _ptr(V), _ptr(leaf_idx), beam, scale,
                                                _ptr(O), dtype_code(O.dtype), _stream(stream)),
           "zha_sparse_attn_decode_noalloc")


def zha_decode(handle, Q: torch.Tensor, beam: int, K: torch.Tensor, V: torch.Tensor, scale: float,
               leaf_idx: torch.Tensor, O: torch.Tensor, leaf_score: torch.Tensor | None = None,
               trace: torch.Tensor | None = None, stream=None) -> None:
    """Route + attention in one call (one launch when the levels fit shared memory)."""
    _check_q(handle, Q)
    B, Hq, nq, _ = Q.shape
    _check_kv(handle, K, V)
    _route_buffers(handle, Q, beam, leaf_idx, leaf_score, trace, O)
    _check(lib().zha_decode(handle, _ptr(Q), dtype_code(Q.dtype), Hq, nq, beam, _ptr(K), _ptr(V),
                            scale, _ptr(leaf_idx), _ptr(leaf_score), _ptr(trace), _ptr(O),
                            dtype_code(O.dtype), _stream(stream)), "zha_decode")


def zha_decode_step(handle, K: torch.Tensor, V: torch.Tensor, new_seq_len: int, Q: torch.Tensor,
                    beam: int, scale: float, leaf_idx: torch.Tensor, O: torch.Tensor,
                    leaf_score: torch.Tensor | None = None, trace: torch.Tensor | None = None,
                    stream=None) -> None:
    """Append up to new_seq_len, then route + attention (one launch for one-leaf appends)."""
    _check_q(handle, Q)
    B, Hq, nq, _ = Q.shape
    _check_kv(handle, K, V)
    _route_buffers(handle, Q, beam, leaf_idx, leaf_score, trace, O, appending=True)
    _check(lib().zha_decode_step(handle, _ptr(K), _ptr(V), new_seq_len, _ptr(Q), dtype_code(Q.dtype),
                                 Hq, nq, beam, scale, _ptr(leaf_idx), _ptr(leaf_score), _ptr(trace),
                                 _ptr(O), dtype_code(O.dtype), _stream(stream)), "zha_decode_step")


def zha_route_causal(handle, K: torch.Tensor, Q: torch.Tensor, positions: torch.Tensor, beam: int,
                     leaf_idx: torch.Tensor, leaf_score: torch.Tensor | None = None,
                     trace: torch.Tensor | None = None, stream=None) -> None:
    """Query i of every head routes over the tree of tokens 0 .. positions[i] (int64, device)."""
    _check_q(handle, Q)
    B, Hq, nq, _ = Q.shape
    _expect(positions, "positions", nq, _I64)
    _check_kv(handle, K)
    _route_buffers(handle, Q, beam, leaf_idx, leaf_score, trace)
    _check(lib().zha_route_causal(handle, _ptr(K), _ptr(Q), dtype_code(Q.dtype), Hq, nq, _ptr(positions),
                                  beam, _ptr(leaf_idx), _ptr(leaf_score), _ptr(trace), _stream(stream)),
           "zha_route_causal")


def zha_decode_causal(handle, Q: torch.Tensor, positions: torch.Tensor, beam: int, K: torch.Tensor,
                      V: torch.Tensor, scale: float, leaf_idx: torch.Tensor, O: torch.Tensor,
                      leaf_score: torch.Tensor | None = None, trace: torch.Tensor | None = None,
                      stream=None) -> None:
    """Causal routing + attention over each query's prefix, one launch."""
    _check_q(handle, Q)
    B, Hq, nq, _ = Q.shape
    _expect(positions, "positions", nq, _I64)
    _check_kv(handle, K, V)
    _route_buffers(handle, Q, beam, leaf_idx, leaf_score, trace, O)
    _check(lib().zha_decode_causal(handle, _ptr(Q), dtype_code(Q.dtype), Hq, nq, _ptr(positions), beam,
                                   _ptr(K), _ptr(V), scale, _ptr(leaf_idx), _ptr(leaf_score), _ptr(trace),
                                   _ptr(O), dtype_code(O.dtype), _stream(stream)), "zha_decode_causal")


def zha_decode_buffered(handle, Q: torch.Tensor, beam: int, K: torch.Tensor, V: torch.Tensor, n_routed: int,
                        n_tokens: int, scale: float, leaf_idx: torch.Tensor, O: torch.Tensor,
                        leaf_score: torch.Tensor | None = None, trace: torch.Tensor | None = None,
                        stream=None) -> None:
    """Route over the tree of the first n_routed tokens, attend over the routed leaves and the
    buffered tokens n_routed .. n_tokens - 1, one launch."""
    _check_q(handle, Q)
    B, Hq, nq, _ = Q.shape
    _check_kv(handle, K, V)
    _route_buffers(handle, Q, beam, leaf_idx, leaf_score, trace, O)
    _check(lib().zha_decode_buffered(handle, _ptr(Q), dtype_code(Q.dtype), Hq, nq, beam, _ptr(K), _ptr(V),
                                     n_routed, n_tokens, scale, _ptr(leaf_idx), _ptr(leaf_score), _ptr(trace),
                                     _ptr(O), dtype_code(O.dtype), _stream(stream)), "zha_decode_buffered")


def zha_tree_radii_bytes(handle) -> int:
    return int(lib().zha_tree_radii_bytes(handle))


def zha_tree_attach_radii(handle, radii: torch.Tensor | None, K: torch.Tensor | None, stream=None) -> None:
    _check_kv(handle, K)
    nbytes = 0 if radii is None else radii.numel() * radii.element_size()
    _check(lib().zha_tree_attach_radii(handle, _ptr(radii), nbytes, _ptr(K), _stream(stream)),
           "zha_tree_attach_radii")


def zha_threshold_route(handle, K: torch.Tensor, Q: torch.Tensor, tau: torch.Tensor, max_tokens: int,
                        tokens: torch.Tensor, count: torch.Tensor, stats: torch.Tensor | None = None,
                        stream=None) -> None:
    _check_q(handle, Q)
    B, Hq, nq, _ = Q.shape
    _check_kv(handle, K)
    _expect(tau, "tau", B * Hq * nq, _F32)
    _expect(tokens, "tokens", B * Hq * nq * int(max_tokens), _I32)
    _expect(count, "count", B * Hq * nq, _I32)
    _expect(stats, "stats", B * Hq * nq * 2, _I32)
    _check(lib().zha_threshold_route(handle, _ptr(K), _ptr(Q), dtype_code(Q.dtype), Hq, nq, _ptr(tau),
                                     max_tokens, _ptr(tokens), _ptr(count), _ptr(stats), _stream(stream)),
           "zha_threshold_route")


def zha_noalloc_scratch_capacity() -> int:
    return int(lib().zha_noalloc_scratch_capacity())


def zha_tree_check(handle, stream=None) -> int:
    return int(lib().zha_tree_check(handle, _stream(stream)))


def zha_tree_seq_len(handle) -> int:
    return int(lib().zha_tree_seq_len(handle))


def zha_tree_levels(handle) -> int:
    return int(lib().zha_tree_levels(handle))


def zha_tree_level_nodes(handle, level: int) -> int:
    return int(lib().zha_tree_level_nodes(handle, level))


def zha_tree_level_offset(handle, level: int) -> int:
    return int(lib().zha_tree_level_offset(handle, level))


def zha_tree_unit_rows(handle) -> int:
    return int(lib().zha_tree_unit_rows(handle))


def zha_tree_launch_count(handle) -> int:
    return int(lib().zha_tree_launch_count(handle))


# ---------------------------------------------------------------- convenience owner

class Tree:
    """A tree set over a [batch, kv_heads, capacity, head_dim] cache, with its workspace."""

    def __init__(self, batch: int, kv_heads: int, head_dim: int, branching: int,
                 leaf_block: int, capacity: int, kv_dtype: torch.dtype, device="cuda",
                 summary_dtype: torch.dtype = torch.float32):
        self.desc = zha_tree_desc(batch, kv_heads, head_dim, branching, leaf_block, capacity,
                                  dtype_code(kv_dtype), dtype_code(summary_dtype))
        self.summary_dtype = summary_dtype
        nbytes = zha_tree_workspace_bytes(self.desc)
        if nbytes == 0:
            raise ZhaError(ZHA_ERR_UNSUPPORTED, "zha_tree_workspace_bytes")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.handle = zha_tree_init(self.desc, self.workspace)
        self._scratch = None

    def close(self):
        if self.handle is not None:
            zha_tree_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def seq_len(self) -> int:
        return zha_tree_seq_len(self.handle)

    @property
    def levels(self) -> int:
        return zha_tree_levels(self.handle)

    @property
    def launches(self) -> int:
        return zha_tree_launch_count(self.handle)

    def level_nodes(self, level: int) -> int:
        return zha_tree_level_nodes(self.handle, level)

    def build(self, K: torch.Tensor, seq_len: int, stream=None):
        zha_tree_build(self.handle, K, seq_len, stream)

    def append(self, K: torch.Tensor, new_seq_len: int, stream=None):
        zha_tree_append(self.handle, K, new_seq_len, stream)

    def summaries(self) -> torch.Tensor:
        """[units, unit_rows, head_dim] view of the workspace's summaries (summary_dtype)."""
        rows = zha_tree_unit_rows(self.handle)
        units = self.desc.batch * self.desc.kv_heads
        d = self.desc.head_dim
        esz = 2 if self.summary_dtype == torch.bfloat16 else 4
        return self.workspace[256:256 + units * rows * d * esz].view(self.summary_dtype).view(units, rows, d)

    def level_offset(self, level: int) -> int:
        """Row offset of a level inside each unit's summaries (and radii)."""
        return zha_tree_level_offset(self.handle, level)

    def level(self, level: int) -> torch.Tensor:
        """[units, n_level, head_dim] view of one level's summaries."""
        off = zha_tree_level_offset(self.handle, level)
        return self.summaries()[:, off:off + self.level_nodes(level)]

    def route(self, Q: torch.Tensor, beam: int, scores: bool = False, trace: bool = False,
              stream=None):
        B, Hq, nq, _ = Q.shape
        idx = torch.empty((B, Hq, nq, beam), dtype=torch.int32, device=Q.device)
        sc = torch.empty((B, Hq, nq, beam), dtype=torch.float32, device=Q.device) if scores else None
        tr = (torch.empty((B, Hq, nq, max(self.levels, 1), beam), dtype=torch.int32, device=Q.device)
              if trace else None)
        zha_route(self.handle, Q, beam, idx, sc, tr, stream)
        return idx, sc, tr

    def scratch_for(self, q_heads: int, nq: int, beam: int, device) -> torch.Tensor | None:
        need = zha_attn_scratch_bytes(self.handle, q_heads, nq, beam)
        if need == 0:
            return None
        if self._scratch is None or self._scratch.numel() < need:
            self._scratch = torch.empty(need, dtype=torch.uint8, device=device)
        return self._scratch

    def attend(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, leaf_idx: torch.Tensor,
               beam: int, scale: float, out_dtype: torch.dtype = torch.bfloat16,
               O: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        B, Hq, nq, d = Q.shape
        if O is None:
            O = torch.empty((B, Hq, nq, d), dtype=out_dtype, device=Q.device)
        scratch = self.scratch_for(Hq, nq, beam, Q.device)
        zha_sparse_attn_decode(self.handle, Q, K, V, leaf_idx, beam, scale, O, scratch, stream)
        return O

    def decode(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, beam: int, scale: float,
               out_dtype: torch.dtype = torch.bfloat16, scores: bool = False, trace: bool = False,
               stream=None):
        """Route + attention in one call; returns (O, leaf_idx, leaf_score or None), plus the
        per-level trace when trace=True."""
        B, Hq, nq, d = Q.shape
        idx = torch.empty((B, Hq, nq, beam), dtype=torch.int32, device=Q.device)
        sc = torch.empty((B, Hq, nq, beam), dtype=torch.float32, device=Q.device) if scores else None
        tr = (torch.empty((B, Hq, nq, max(self.levels, 1), beam), dtype=torch.int32, device=Q.device)
              if trace else None)
        O = torch.empty((B, Hq, nq, d), dtype=out_dtype, device=Q.device)
        zha_decode(self.handle, Q, beam, K, V, scale, idx, O, sc, tr, stream)
        return (O, idx, sc, tr) if trace else (O, idx, sc)

    def levels_for(self, seq_len: int) -> int:
        """Levels below the root of a tree over seq_len tokens (shape only)."""
        n0 = -(-seq_len // self.desc.leaf_block)
        L, span = 1, self.desc.branching
        while span < n0:
            span *= self.desc.branching
            L += 1
        return L if n0 > 0 else 0

    def decode_step(self, K: torch.Tensor, V: torch.Tensor, new_seq_len: int, Q: torch.Tensor,
                    beam: int, scale: float, out_dtype: torch.dtype = torch.bfloat16,
                    trace: bool = False, stream=None):
        """Append to new_seq_len, then route + attention; returns (O, leaf_idx[, trace])."""
        B, Hq, nq, d = Q.shape
        idx = torch.empty((B, Hq, nq, beam), dtype=torch.int32, device=Q.device)
        O = torch.empty((B, Hq, nq, d), dtype=out_dtype, device=Q.device)
        tr = None
        if trace:
            L = self.levels_for(new_seq_len)
            tr = torch.empty((B, Hq, nq, L, beam), dtype=torch.int32, device=Q.device)
        zha_decode_step(self.handle, K, V, new_seq_len, Q, beam, scale, idx, O, None, tr, stream)
        return (O, idx, tr) if trace else (O, idx)

    def route_causal(self, K: torch.Tensor, Q: torch.Tensor, positions: torch.Tensor, beam: int,
                     trace: bool = False, stream=None):
        """Causal routing; returns (leaf_idx, trace or None)."""
        B, Hq, nq, _ = Q.shape
        idx = torch.empty((B, Hq, nq, beam), dtype=torch.int32, device=Q.device)
        tr = (torch.empty((B, Hq, nq, max(self.levels, 1), beam), dtype=torch.int32, device=Q.device)
              if trace else None)
        zha_route_causal(self.handle, K, Q, positions, beam, idx, None, tr, stream)
        return idx, tr

    def decode_causal(self, Q: torch.Tensor, positions: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                      beam: int, scale: float, out_dtype: torch.dtype = torch.bfloat16, stream=None):
        """Causal routing + attention; returns (O, leaf_idx)."""
        B, Hq, nq, d = Q.shape
        idx = torch.empty((B, Hq, nq, beam), dtype=torch.int32, device=Q.device)
        O = torch.empty((B, Hq, nq, d), dtype=out_dtype, device=Q.device)
        zha_decode_causal(self.handle, Q, positions, beam, K, V, scale, idx, O, None, None, stream)
        return O, idx

    def decode_buffered(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, n_routed: int, n_tokens: int,
                        beam: int, scale: float, out_dtype: torch.dtype = torch.bfloat16, trace: bool = False,
                        stream=None):
        """Decode with an append buffer; returns (O, leaf_idx) or (O, leaf_idx, trace)."""
        B, Hq, nq, d = Q.shape
        idx = torch.empty((B, Hq, nq, beam), dtype=torch.int32, device=Q.device)
        O = torch.empty((B, Hq, nq, d), dtype=out_dtype, device=Q.device)
        tr = (torch.empty((B, Hq, nq, self.levels, beam), dtype=torch.int32, device=Q.device)
              if trace else None)
        zha_decode_buffered(self.handle, Q, beam, K, V, n_routed, n_tokens, scale, idx, O, None, tr, stream)
        return (O, idx, tr) if trace else (O, idx)

    def attach_radii(self, K: torch.Tensor | None, stream=None) -> torch.Tensor:
        """Allocate and attach the bounding-sphere radii; returns them ([units, unit_rows])."""
        n = zha_tree_radii_bytes(self.handle) // 4
        self._radii = torch.zeros(n, dtype=torch.float32, device=self.workspace.device)
        zha_tree_attach_radii(self.handle, self._radii, K, stream)
        return self._radii.view(-1, zha_tree_unit_rows(self.handle))

    def threshold(self, K: torch.Tensor, Q: torch.Tensor, tau: torch.Tensor, max_tokens: int,
                  stats: bool = False, stream=None):
        """Threshold descent; returns (tokens, count, stats or None)."""
        B, Hq, nq, _ = Q.shape
        toks = torch.empty((B, Hq, nq, max_tokens), dtype=torch.int32, device=Q.device)
        cnt = torch.empty((B, Hq, nq), dtype=torch.int32, device=Q.device)
        st = torch.empty((B, Hq, nq, 2), dtype=torch.int32, device=Q.device) if stats else None
        zha_threshold_route(self.handle, K, Q, tau, max_tokens, toks, cnt, st, stream)
        return toks, cnt, st

    def check(self, stream=None) -> int:
        return zha_tree_check(self.handle, stream)
