"""The C ABI without a GPU: the library loads, exports every function that
include/crs.h declares, and rejects bad arguments on the host (no launch)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(crs_[a-z0-9_]+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(crs):
    names = _declared()
    assert len(names) >= 14
    missing = [n for n in sorted(names) if not hasattr(crs.lib(), n)]
    assert not missing, f"declared but not exported: {missing}"


def test_status_strings_and_version(crs):
    lib = crs.lib()
    assert lib.crs_status_string(0) == b"CRS_OK"
    assert lib.crs_status_string(6) == b"CRS_ERR_WORKSPACE"
    assert lib.crs_version() >= 100


def test_host_validation_without_gpu(crs):
    """Invalid parameters return an error code before any CUDA call."""
    lib = crs.lib()
    assert lib.crs_lsh_route(None, None, None, None, None, None, None, 0, None) == 1
    p = crs.LshParams(1, 1, 64, 7, 16, 1, 8, 0)          # d not a multiple of 8
    assert lib.crs_lsh_route(ctypes.byref(p), None, None, None, None, None, None, 0, None) == 1
    a = crs.LshAttnParams(crs.LshParams(1, 1, 64, 64, 16, 9, 8, 0), 1, 1, 1, 0.125)  # 9 rounds
    assert lib.crs_lsh_attn(ctypes.byref(a), *([None] * 9), 0, None) == 1
    ip = crs.IndexerParams(0, 10, 4, 32, 16, 0)         # d_idx != 64
    assert lib.crs_indexer_topk(ctypes.byref(ip), *([None] * 6), None, 0, None) == 2
    ap = crs.AttnParams(4, 48, 2, 128, 16, 1, 0, 0.1)    # G = 24 > 16
    assert lib.crs_sparse_attn(ctypes.byref(ap), *([None] * 8), 0, None) == 2
    bp = crs.BlockParams(1, 1, 64, 128, 31, 4, 0, 2)     # odd L
    assert lib.crs_block_describe(ctypes.byref(bp), None, None, None, None) == 2


def test_workspace_sizes_host_only(crs):
    lib = crs.lib()
    a = crs.LshAttnParams(crs.LshParams(2, 8, 16384, 64, 64, 4, 128, 1), 1, 0, 1, 0.125)
    assert lib.crs_lsh_attn_workspace_size(ctypes.byref(a)) >= 4 * 16 * 16384 * 64 * 4
    ip = crs.IndexerParams(1, 64, 4, 64, 2048, 131072)
    assert lib.crs_indexer_topk_workspace_size(ctypes.byref(ip)) > 0


def test_short_workspace_is_rejected_before_launch(crs):
    lib = crs.lib()
    a = crs.LshAttnParams(crs.LshParams(1, 1, 256, 64, 16, 2, 64, 0), 1, 1, 1, 0.125)
    dummy = ctypes.c_void_p(0x1000)
    st = lib.crs_lsh_attn(ctypes.byref(a), dummy, dummy, dummy, dummy, dummy, None, dummy, None,
                          dummy, 16, None)
    assert st == 6
