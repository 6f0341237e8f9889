"""The C ABI without a GPU: the library loads, exports every function include/zha.h
declares, and rejects bad arguments on the host before touching the device."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from tree_indexed_sparse_build_b200 import zha

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zha.h")


def declared_functions() -> list[str]:
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(zha_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("zha_tree_build", "zha_tree_append", "zha_route", "zha_sparse_attn_decode"):
        assert must in names


def test_library_exports_every_declared_function():
    lib = zha.lib()
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"
    assert sorted(zha.EXPORTED) == declared_functions()


def test_status_strings():
    for s in range(7):
        assert zha.status_string(s) and zha.status_string(s) != "unknown status"
    assert zha.status_string(99) == "unknown status"


def _desc(**kw):
    d = dict(batch=1, kv_heads=8, head_dim=128, branching=8, leaf_block=4,
             capacity_tokens=1 << 20, kv_dtype=zha.ZHA_BF16)
    d.update(kw)
    return zha.zha_tree_desc(**d)


def test_workspace_bytes_matches_capacity_layout():
    # 1M tokens, leaf block 4, b = 8: levels of 262144, 32768, 4096, 512, 64, 8, 1 rows
    rows = 262144 + 32768 + 4096 + 512 + 64 + 8 + 1
    assert zha.zha_tree_workspace_bytes(_desc()) == 256 + 8 * rows * 128 * 4
    # tiny: 1024 tokens, leaf 16, b 2 -> 64+32+...+1 = 127 rows
    assert zha.zha_tree_workspace_bytes(
        _desc(batch=1, kv_heads=1, head_dim=64, branching=2, leaf_block=16,
              capacity_tokens=1024, kv_dtype=zha.ZHA_F32)) == 256 + 127 * 64 * 4
    # bf16-stored summaries: two bytes an element
    assert zha.zha_tree_workspace_bytes(_desc(summary_dtype=zha.ZHA_BF16)) == 256 + 8 * rows * 128 * 2


@pytest.mark.parametrize("bad", [dict(head_dim=96), dict(branching=1), dict(leaf_block=0),
                                 dict(capacity_tokens=0), dict(batch=0), dict(kv_heads=0),
                                 dict(batch=300, kv_heads=300), dict(kv_dtype=7),
                                 dict(summary_dtype=2)])
def test_workspace_bytes_rejects_bad_desc(bad):
    assert zha.zha_tree_workspace_bytes(_desc(**bad)) == 0


def test_calls_reject_null_tree_on_host():
    lib = zha.lib()
    assert lib.zha_tree_build(None, None, 0, None) == zha.ZHA_ERR_INVALID_ARG
    assert lib.zha_tree_append(None, None, 1, None) == zha.ZHA_ERR_INVALID_ARG
    assert lib.zha_route(None, None, 1, 8, 1, 4, None, None, None, None) == zha.ZHA_ERR_INVALID_ARG
    assert lib.zha_sparse_attn_decode(None, None, 1, 8, 1, None, None, None, 4,
                                      ctypes.c_float(0.1), None, 1, None, 0, None) == \
        zha.ZHA_ERR_INVALID_ARG
    assert lib.zha_sparse_attn_decode_noalloc(None, None, 1, 8, 1, None, None, None, 4,
                                              ctypes.c_float(0.1), None, 1, None) == \
        zha.ZHA_ERR_INVALID_ARG
    assert lib.zha_route_causal(None, None, None, 1, 8, 1, None, 4, None, None, None, None) == \
        zha.ZHA_ERR_INVALID_ARG
    assert lib.zha_decode_causal(None, None, 1, 8, 1, None, 4, None, None, ctypes.c_float(0.1), None,
                                 None, None, None, 1, None) == zha.ZHA_ERR_INVALID_ARG
    assert lib.zha_decode_buffered(None, None, 1, 8, 1, 4, None, None, 16, 16, ctypes.c_float(0.1), None,
                                   None, None, None, 1, None) == zha.ZHA_ERR_INVALID_ARG
    assert lib.zha_tree_attach_radii(None, None, 0, None, None) == zha.ZHA_ERR_INVALID_ARG
    assert lib.zha_tree_radii_bytes(None) == 0
    assert lib.zha_threshold_route(None, None, None, 1, 8, 1, None, 16, None, None, None, None) == \
        zha.ZHA_ERR_INVALID_ARG
    assert lib.zha_tree_destroy(None) == zha.ZHA_ERR_INVALID_ARG
    assert lib.zha_tree_check(None, None) == zha.ZHA_ERR_INVALID_ARG
    assert lib.zha_tree_levels(None) == -1
    assert lib.zha_attn_scratch_bytes(None, 8, 1, 4) == 0
    assert lib.zha_noalloc_scratch_capacity() == 128 * 1024


def test_init_rejects_bad_workspace_without_touching_the_device():
    lib = zha.lib()
    h = ctypes.c_void_p()
    d = _desc()
    # null workspace, misaligned workspace, too small: all host-side refusals
    assert lib.zha_tree_init(ctypes.byref(d), None, 1 << 30, ctypes.byref(h)) == zha.ZHA_ERR_INVALID_ARG
    assert lib.zha_tree_init(ctypes.byref(d), ctypes.c_void_p(0x1008), 1 << 40,
                             ctypes.byref(h)) == zha.ZHA_ERR_INVALID_ARG
    assert lib.zha_tree_init(ctypes.byref(d), ctypes.c_void_p(0x10000), 16,
                             ctypes.byref(h)) == zha.ZHA_ERR_INVALID_ARG
    bad = _desc(head_dim=96)
    assert lib.zha_tree_init(ctypes.byref(bad), ctypes.c_void_p(0x10000), 1 << 40,
                             ctypes.byref(h)) == zha.ZHA_ERR_UNSUPPORTED
    assert h.value is None
