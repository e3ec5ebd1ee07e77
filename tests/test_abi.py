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
    ap = crs.AttnParams(4, 48, 2, 128, 16, 1, 100, 0.1)  # G = 24 > 16
    assert lib.crs_sparse_attn(ctypes.byref(ap), *([None] * 10), 0, None) == 2
    ap = crs.AttnParams(4, 16, 1, 128, 16, 1, 0, 0.1)    # no key count: no bound to check
    assert lib.crs_sparse_attn(ctypes.byref(ap), *([None] * 10), 0, None) == 1
    bp = crs.BlockParams(1, 1, 64, 128, 31, 4, 0, 2)     # odd L
    assert lib.crs_block_describe(ctypes.byref(bp), None, None, None, None) == 2
    # Q, K or V off a 16-byte boundary: rejected before any launch
    ap = crs.AttnParams(4, 16, 1, 128, 16, 1, 100, 0.1)
    f16, f2 = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10002)
    assert lib.crs_sparse_attn(ctypes.byref(ap), f16, f2, f16, None, f16, None, None, f16, None, None, 0,
                               None) == 1
    # the L2 probe: null pointers or empty sizes are rejected before any CUDA call
    f16 = ctypes.c_void_p(0x10000)
    assert lib.crs_probe_l2_gather(None, 1, f16, 1, f16, None) == 1
    assert lib.crs_probe_l2_gather(f16, 0, f16, 1, f16, None) == 1
    assert lib.crs_probe_l2_gather(f16, 1, f16, 0, f16, None) == 1
    # O not on a 16-byte boundary: rejected before the workspace is looked at (no launch)
    a = crs.LshAttnParams(crs.LshParams(1, 1, 256, 64, 16, 2, 128, 1), 1, 0, 1, 0.125)
    fake = ctypes.c_void_p(0x10000)
    assert lib.crs_lsh_attn(ctypes.byref(a), fake, fake, fake, fake, fake, None, ctypes.c_void_p(0x10004),
                            None, None, 0, None) == 1


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


def test_host_validation_of_the_later_entry_points(crs):
    """HISA, LSH decode, routing, the compressed / subspace / Quest block selectors:
    out-of-range parameters give CRS_ERR_INVALID_ARG (1), shapes the kernels do not
    implement CRS_ERR_UNSUPPORTED (2), missing buffers CRS_ERR_INVALID_ARG, all
    before any device work (these calls run on a machine without a GPU)."""
    lib = crs.lib()
    by = ctypes.byref
    # HISA: no rows; index head dim other than 64; then NULL buffers
    assert lib.crs_hisa_topk(by(crs.HisaParams(0, 4, 64, 2048, 64, 128, 131072)), *([None] * 10), 0, None) == 1
    assert lib.crs_hisa_describe(by(crs.HisaParams(4, 4, 32, 2048, 64, 128, 131072)), *([None] * 5)) == 2
    assert lib.crs_hisa_describe(by(crs.HisaParams(4, 4, 64, 2048, 64, 128, 131072)), *([None] * 5)) == 1
    assert lib.crs_hisa_topk(by(crs.HisaParams(4, 4, 64, 2048, 64, 128, 131072)), *([None] * 10), 0, None) == 1
    assert lib.crs_hisa_topk_workspace_size(by(crs.HisaParams(0, 4, 64, 2048, 64, 128, 131072))) == 0
    # LSH decode: odd bucket count; d other than 64; valid parameters with an empty state
    ld = dict(n_seq=2, n_heads=2, d=64, n_buckets=16, n_rounds=2, page_size=16, max_pages=8, list_page=8,
              list_pages=8, n_list_pages=64, max_len=128, no_self=1, key_norm=1, scale=0.125)
    st = crs.LshDecodeState()
    assert lib.crs_lsh_decode_step(by(crs.LshDecodeParams(**{**ld, "n_buckets": 15})), by(st), *([None] * 7)) == 1
    assert lib.crs_lsh_decode_step(by(crs.LshDecodeParams(**{**ld, "d": 32})), by(st), *([None] * 7)) == 2
    assert lib.crs_lsh_decode_step(by(crs.LshDecodeParams(**ld)), by(st), *([None] * 7)) == 1
    assert lib.crs_lsh_decode_prefill(by(crs.LshDecodeParams(**ld)), by(st), None, None, None, 4, None) == 1
    # routing: no centres; head dim other than 64; then NULL inputs
    assert lib.crs_route_attn(by(crs.RouteParams(1, 1, 256, 64, 0, 8, 1, 0, 0.125)), *([None] * 10), 0, None) == 1
    assert lib.crs_route_attn(by(crs.RouteParams(1, 1, 256, 32, 4, 8, 1, 0, 0.125)), *([None] * 10), 0, None) == 2
    assert lib.crs_route_attn(by(crs.RouteParams(1, 1, 256, 64, 4, 8, 1, 0, 0.125)), *([None] * 10), 0, None) == 1
    # block selectors on FP4 codes, the query subspace and Quest boxes: NULL inputs
    bp = crs.BlockParams(2, 2, 4096, 128, 32, 4, 0, 4096 // 32)
    sp = crs.BlockSelParams(bp, 16, 16, 256, 0.0884)
    assert lib.crs_block_select_fp4(by(sp), *([None] * 7), 0, None) == 1
    assert lib.crs_block_select_ss(by(sp), None, None, 16, *([None] * 5), 0, None) == 1
    assert lib.crs_block_select_quest(by(sp), *([None] * 6), 0, None) == 1
    assert lib.crs_block_quest_describe(by(bp), None, None, None, None) == 1
    assert lib.crs_block_quantize(by(bp), *([None] * 6)) == 1


def test_host_validation_of_the_csr_export(crs):
    """crs_lsh_candidates_csr: too many rounds, a chunk past 128, NULL routing arrays and
    an input beyond the export's size limit are rejected before any launch."""
    lib = crs.lib()
    by = ctypes.byref
    dummy = ctypes.c_void_p(0x1000)
    bad_rounds = crs.LshAttnParams(crs.LshParams(1, 1, 64, 64, 16, 9, 8, 1), 1, 0, 1, 0.125)
    assert lib.crs_lsh_candidates_csr(by(bad_rounds), dummy, dummy, dummy, None, dummy, None, None) == 1
    bad_chunk = crs.LshAttnParams(crs.LshParams(1, 1, 64, 64, 16, 2, 256, 1), 1, 0, 1, 0.125)
    assert lib.crs_lsh_candidates_csr(by(bad_chunk), dummy, dummy, dummy, None, dummy, None, None) == 1
    ok = crs.LshAttnParams(crs.LshParams(1, 1, 64, 64, 16, 2, 32, 1), 1, 0, 1, 0.125)
    assert lib.crs_lsh_candidates_csr(by(ok), None, dummy, dummy, None, dummy, None, None) == 1
    big = crs.LshAttnParams(crs.LshParams(1, 1, 70000, 64, 16, 2, 32, 1), 1, 0, 1, 0.125)
    assert lib.crs_lsh_candidates_csr(by(big), dummy, dummy, dummy, None, dummy, None, None) == 2
