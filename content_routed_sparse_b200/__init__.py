"""content_routed_sparse_b200 -- Python binding of libcrs (content-routed sparse
attention on NVIDIA B200, sm_100a).

Argument marshalling only: every step runs in the CUDA kernels of libcrs.so,
reached through the C ABI declared in include/crs.h.  PyTorch provides device
memory and streams.  Importing this module loads libcrs.so and raises if it
is missing; there is no fallback.

Functions (same names as the C entry points, without the ``crs_`` prefix):
  lsh_route, lsh_attn, indexer_topk, block_describe, block_select,
  block_quantize, block_select_fp4, sparse_attn, get_device_error.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcrs.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libcrs.so not found at {LIB_PATH}; build it with "
        "`python content_routed_sparse_b200/build.py` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

CRS_F32, CRS_BF16 = 0, 1
CRS_IDX_PREFILL, CRS_IDX_DECODE = 0, 1
STATUS = {0: "CRS_OK", 1: "CRS_ERR_INVALID_ARG", 2: "CRS_ERR_UNSUPPORTED", 3: "CRS_ERR_CUDA",
          4: "CRS_ERR_NONFINITE", 5: "CRS_ERR_TIMEOUT", 6: "CRS_ERR_WORKSPACE",
          7: "CRS_ERR_INDEX"}
DEVERR_NONFINITE, DEVERR_TIMEOUT, DEVERR_INDEX = 0x1, 0x2, 0x4


class CrsError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")
        self.status = status


class LshParams(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("n", ctypes.c_int),
                ("d", ctypes.c_int), ("n_buckets", ctypes.c_int), ("n_rounds", ctypes.c_int),
                ("chunk", ctypes.c_int), ("dtype", ctypes.c_int)]


class LshAttnParams(ctypes.Structure):
    _fields_ = [("p", LshParams), ("causal", ctypes.c_int), ("no_self", ctypes.c_int),
                ("key_norm", ctypes.c_int), ("scale", ctypes.c_float)]


class IndexerParams(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("n_rows", ctypes.c_int), ("n_idx_heads", ctypes.c_int),
                ("d_idx", ctypes.c_int), ("topk", ctypes.c_int), ("max_keys", ctypes.c_int)]


class HisaParams(ctypes.Structure):
    _fields_ = [("n_rows", ctypes.c_int), ("n_idx_heads", ctypes.c_int), ("d_idx", ctypes.c_int),
                ("topk", ctypes.c_int), ("blk", ctypes.c_int), ("top_blocks", ctypes.c_int),
                ("max_keys", ctypes.c_int)]


class LshDecodeParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("n_seq", "n_heads", "d", "n_buckets", "n_rounds", "page_size",
                                              "max_pages", "list_page", "list_pages", "n_list_pages",
                                              "max_len", "no_self", "key_norm")] + [("scale", ctypes.c_float)]


class LshDecodeState(ctypes.Structure):
    _fields_ = [("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("bucket_store", ctypes.c_void_p), ("list_table", ctypes.c_void_p), ("list_len", ctypes.c_void_p),
                ("list_pool", ctypes.c_void_p), ("alloc", ctypes.c_void_p), ("seq_len", ctypes.c_void_p)]


class RouteParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "H", "n", "d", "C", "m", "causal", "no_self")] + \
               [("scale", ctypes.c_float)]


class BlockParams(ctypes.Structure):
    _fields_ = [("n_seq", ctypes.c_int), ("n_kv", ctypes.c_int), ("T", ctypes.c_int),
                ("D", ctypes.c_int), ("L", ctypes.c_int), ("rank", ctypes.c_int),
                ("blk_begin", ctypes.c_int), ("blk_end", ctypes.c_int)]


class BlockSelParams(ctypes.Structure):
    _fields_ = [("b", BlockParams), ("n_q", ctypes.c_int), ("top_blocks", ctypes.c_int),
                ("window", ctypes.c_int), ("scale", ctypes.c_float)]


class AttnParams(ctypes.Structure):
    _fields_ = [("n_rows", ctypes.c_int), ("n_q", ctypes.c_int), ("n_kv", ctypes.c_int),
                ("D", ctypes.c_int), ("max_idx", ctypes.c_int), ("n_lists", ctypes.c_int),
                ("n_keys", ctypes.c_int), ("scale", ctypes.c_float)]


class KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int64),
                ("timed_launches", ctypes.c_int64), ("total_ms", ctypes.c_double)]


_VP = ctypes.c_void_p
_SZ = ctypes.c_size_t


def _sig(name, restype, argtypes):
    f = getattr(_lib, name, None)
    if f is None:
        return None
    f.restype = restype
    f.argtypes = argtypes
    return f


_lib.crs_status_string.restype = ctypes.c_char_p
_lib.crs_status_string.argtypes = [ctypes.c_int]
_lib.crs_version.restype = ctypes.c_int
_lib.crs_get_device_error.restype = ctypes.c_int
_lib.crs_get_device_error.argtypes = [_VP, ctypes.POINTER(ctypes.c_uint32)]
_sig("crs_lsh_route_workspace_size", _SZ, [ctypes.POINTER(LshParams)])
_sig("crs_lsh_route", ctypes.c_int, [ctypes.POINTER(LshParams), _VP, _VP, _VP, _VP, _VP, _VP,
                                      _SZ, _VP])
_sig("crs_lsh_attn_workspace_size", _SZ, [ctypes.POINTER(LshAttnParams)])
_sig("crs_lsh_attn", ctypes.c_int, [ctypes.POINTER(LshAttnParams), _VP, _VP, _VP, _VP, _VP, _VP,
                                     _VP, _VP, _VP, _SZ, _VP])
_sig("crs_lsh_candidates_csr", ctypes.c_int, [ctypes.POINTER(LshAttnParams), _VP, _VP, _VP, _VP, _VP, _VP,
                                               _VP])
_sig("crs_indexer_topk_workspace_size", _SZ, [ctypes.POINTER(IndexerParams)])
_sig("crs_indexer_topk", ctypes.c_int, [ctypes.POINTER(IndexerParams), _VP, _VP, _VP, _VP, _VP,
                                         _VP, _VP, _SZ, _VP])
_sig("crs_block_describe", ctypes.c_int, [ctypes.POINTER(BlockParams), _VP, _VP, _VP, _VP])
_sig("crs_block_select_workspace_size", _SZ, [ctypes.POINTER(BlockSelParams)])
_sig("crs_block_select", ctypes.c_int, [ctypes.POINTER(BlockSelParams), _VP, _VP, _VP, _VP, _VP,
                                         _VP, _SZ, _VP])
_sig("crs_block_quantize", ctypes.c_int, [ctypes.POINTER(BlockParams), _VP, _VP, _VP, _VP, _VP, _VP])
_sig("crs_block_select_fp4", ctypes.c_int, [ctypes.POINTER(BlockSelParams), _VP, _VP, _VP, _VP, _VP,
                                             _VP, _VP, _SZ, _VP])
_sig("crs_route_attn_workspace_size", _SZ, [ctypes.POINTER(RouteParams)])
_sig("crs_route_attn", ctypes.c_int, [ctypes.POINTER(RouteParams), _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                       _VP, _SZ, _VP])
_sig("crs_lsh_decode_prefill", ctypes.c_int, [ctypes.POINTER(LshDecodeParams), ctypes.POINTER(LshDecodeState),
                                                _VP, _VP, _VP, ctypes.c_int, _VP])
_sig("crs_lsh_decode_step", ctypes.c_int, [ctypes.POINTER(LshDecodeParams), ctypes.POINTER(LshDecodeState),
                                             _VP, _VP, _VP, _VP, _VP, _VP, _VP])
_sig("crs_hisa_describe", ctypes.c_int, [ctypes.POINTER(HisaParams), _VP, _VP, _VP, _VP, _VP])
_sig("crs_hisa_topk_workspace_size", _SZ, [ctypes.POINTER(HisaParams)])
_sig("crs_hisa_topk", ctypes.c_int, [ctypes.POINTER(HisaParams), _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                      _VP, _SZ, _VP])
_sig("crs_hisa_topk_prefill_workspace_size", _SZ, [ctypes.POINTER(HisaParams)])
_sig("crs_hisa_topk_prefill", ctypes.c_int, [ctypes.POINTER(HisaParams), _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                              _SZ, _VP])
_sig("crs_block_quantize_ss", ctypes.c_int, [ctypes.POINTER(BlockParams), _VP, _VP, ctypes.c_int, _VP, _VP, _VP,
                                              _VP])
_sig("crs_block_select_fp4_ss_workspace_size", _SZ, [ctypes.POINTER(BlockSelParams), ctypes.c_int])
_sig("crs_block_select_fp4_ss", ctypes.c_int, [ctypes.POINTER(BlockSelParams), _VP, _VP, ctypes.c_int, _VP, _VP,
                                                _VP, _VP, _VP, _VP, _SZ, _VP])
_sig("crs_block_describe_ss", ctypes.c_int, [ctypes.POINTER(BlockParams), _VP, _VP, ctypes.c_int, _VP, _VP,
                                              _VP])
_sig("crs_block_select_ss_workspace_size", _SZ, [ctypes.POINTER(BlockSelParams), ctypes.c_int])
_sig("crs_block_select_ss", ctypes.c_int, [ctypes.POINTER(BlockSelParams), _VP, _VP, ctypes.c_int, _VP, _VP,
                                            _VP, _VP, _VP, _SZ, _VP])
_sig("crs_block_quest_describe", ctypes.c_int, [ctypes.POINTER(BlockParams), _VP, _VP, _VP, _VP])
_sig("crs_block_select_quest", ctypes.c_int, [ctypes.POINTER(BlockSelParams), _VP, _VP, _VP, _VP, _VP,
                                               _VP, _SZ, _VP])
_sig("crs_block_select_noalloc", ctypes.c_int, [ctypes.POINTER(BlockSelParams), _VP, _VP, _VP,
                                                 _VP, _VP, _VP])
_sig("crs_sparse_attn_workspace_size", _SZ, [ctypes.POINTER(AttnParams)])
_sig("crs_sparse_attn", ctypes.c_int, [ctypes.POINTER(AttnParams), _VP, _VP, _VP, _VP, _VP, _VP,
                                        _VP, _VP, _VP, _VP, _SZ, _VP])


_sig("crs_profile_set", ctypes.c_int, [ctypes.c_int])
_sig("crs_profile_collect", ctypes.c_int, [ctypes.POINTER(KernelStat), ctypes.c_int,
                                            ctypes.POINTER(ctypes.c_int)])


def lib():
    """The loaded ctypes handle of libcrs.so."""
    return _lib


# ------------------------------------------------------------------ utils --
def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, st):
    if st != 0:
        raise CrsError(fn, st)


def _need(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]):
    if nbytes == 0:
        return None, 0
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace too small: need {nbytes} bytes")
        return workspace, workspace.numel() * workspace.element_size()
    return torch.empty(nbytes, dtype=torch.uint8, device=device), nbytes


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return CRS_F32
    if t.dtype == torch.bfloat16:
        return CRS_BF16
    raise ValueError(f"unsupported dtype {t.dtype}")


def get_device_error(stream=None) -> int:
    """Synchronize, read and clear the device error word (CRS_DEVERR_* bits)."""
    v = ctypes.c_uint32(0)
    _check("crs_get_device_error", _lib.crs_get_device_error(_stream(stream), ctypes.byref(v)))
    return int(v.value)


_sig("crs_get_device_diag", ctypes.c_int, [_VP, ctypes.POINTER(ctypes.c_uint32), ctypes.c_int])


def get_device_diag(stream=None) -> list:
    """Synchronize, read and clear the kernels' diagnostic record (16 words, [0] == 0: none)."""
    buf = (ctypes.c_uint32 * 16)()
    _check("crs_get_device_diag", _lib.crs_get_device_diag(_stream(stream), buf, 16))
    return [int(x) for x in buf]


_sig("crs_debug_force_wait_timeout", ctypes.c_int, [ctypes.c_int])


def debug_force_wait_timeout(on: bool) -> None:
    """Make the first bounded wait of the tensor-core LSH kernels give up at once
    (failure-path test switch; see include/crs.h)."""
    _check("crs_debug_force_wait_timeout", _lib.crs_debug_force_wait_timeout(1 if on else 0))


_sig("crs_probe_l2_gather", ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                                             ctypes.c_void_p, ctypes.c_void_p])


def probe_l2_gather(table: torch.Tensor, idx: torch.Tensor, sink: torch.Tensor) -> None:
    """Gather the 512-byte rows idx of table (rows x 512 bytes) once, on the current
    stream; a measurement aid for the L2 gather ceiling (see include/crs.h)."""
    if not (table.is_cuda and idx.is_cuda and sink.is_cuda) or idx.dtype != torch.int32:
        raise ValueError("probe_l2_gather: CUDA table, int32 idx and sink expected")
    if table.numel() * table.element_size() % 512 or not table.is_contiguous() or not idx.is_contiguous():
        raise ValueError("probe_l2_gather: contiguous table of 512-byte rows expected")
    if sink.numel() * sink.element_size() < 16:
        raise ValueError("probe_l2_gather: sink of at least 16 bytes expected")
    rows = table.numel() * table.element_size() // 512
    _check("crs_probe_l2_gather", _lib.crs_probe_l2_gather(table.data_ptr(), rows, idx.data_ptr(), idx.numel(),
                                                           sink.data_ptr(), _stream(None)))


def profile_set(enabled: bool) -> None:
    """Turn per-launch CUDA-event timing on or off (launch counting is always on)."""
    _check("crs_profile_set", _lib.crs_profile_set(1 if enabled else 0))


def profile_collect() -> dict:
    """{kernel: {"launches", "timed_launches", "total_ms"}} since the last collect (then reset)."""
    buf = (KernelStat * 64)()
    n = ctypes.c_int(0)
    _check("crs_profile_collect", _lib.crs_profile_collect(buf, 64, ctypes.byref(n)))
    out = {}
    for i in range(min(n.value, 64)):
        out[buf[i].name.decode()] = {"launches": int(buf[i].launches),
                                     "timed_launches": int(buf[i].timed_launches),
                                     "total_ms": float(buf[i].total_ms)}
    return out


# -------------------------------------------------------------------- LSH --
def lsh_params(QK: torch.Tensor, n_buckets: int, n_rounds: int, chunk: int) -> LshParams:
    B, H, n, d = QK.shape
    return LshParams(B, H, n, d, int(n_buckets), int(n_rounds), int(chunk), _dtype_code(QK))


def lsh_route(X: torch.Tensor, R: torch.Tensor, n_buckets: int, chunk: int = 1,
              out=None, stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Bucket ids, perm (slot -> position) and inv_perm, each [B,H,rounds,n] int32."""
    _need(X, "X")
    B, H, n, d = X.shape
    n_rounds = R.shape[1]
    _need(R, "R", torch.float32, (H, n_rounds, d, n_buckets // 2))
    p = lsh_params(X, n_buckets, n_rounds, chunk)
    shape = (B, H, n_rounds, n)
    if out is None:
        out = tuple(torch.empty(shape, dtype=torch.int32, device=X.device) for _ in range(3))
    bucket, perm, inv = out
    for t, nm in ((bucket, "bucket"), (perm, "perm"), (inv, "inv_perm")):
        _need(t, nm, torch.int32, shape)
    st = _lib.crs_lsh_route(ctypes.byref(p), _ptr(X), _ptr(R), _ptr(bucket), _ptr(perm),
                            _ptr(inv), None, 0, _stream(stream))
    _check("crs_lsh_route", st)
    return bucket, perm, inv


def lsh_attn(QK, V, bucket, perm, inv_perm, valid_len=None, *, n_buckets, chunk, causal=1,
             no_self=0, key_norm=1, scale=None, out=None, lse=None, workspace=None,
             stream=None):
    """Chunked multi-round LSH attention; returns (O [B,H,n,d] fp32, lse [B,H,n] or None)."""
    _need(QK, "QK")
    B, H, n, d = QK.shape
    _need(V, "V", QK.dtype, QK.shape)
    n_rounds = bucket.shape[2]
    for t, nm in ((bucket, "bucket"), (perm, "perm"), (inv_perm, "inv_perm")):
        _need(t, nm, torch.int32, (B, H, n_rounds, n))
    if valid_len is not None:
        _need(valid_len, "valid_len", torch.int32, (B,))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    a = LshAttnParams(lsh_params(QK, n_buckets, n_rounds, chunk), int(causal), int(no_self),
                      int(key_norm), float(scale))
    if out is None:
        out = torch.empty(QK.shape, dtype=torch.float32, device=QK.device)
    _need(out, "out", torch.float32, QK.shape)
    if lse is not None:
        _need(lse, "lse", torch.float32, (B, H, n))
    ws, wsb = _workspace(int(_lib.crs_lsh_attn_workspace_size(ctypes.byref(a))), QK.device,
                         workspace)
    st = _lib.crs_lsh_attn(ctypes.byref(a), _ptr(QK), _ptr(V), _ptr(bucket), _ptr(perm),
                           _ptr(inv_perm), _ptr(valid_len), _ptr(out), _ptr(lse), _ptr(ws), wsb,
                           _stream(stream))
    _check("crs_lsh_attn", st)
    return out, lse


# ---------------------------------------------------------------- indexer --
def lsh_candidates_csr(bucket, perm, inv_perm, valid_len=None, *, chunk, causal=1, no_self=0,
                       stream=None):
    """The candidate sets U(i) of lsh_attn as CSR: (row_ptr [B*H*n + 1] int64,
    col_idx int32), rows ordered (b, h, i), each row ascending.  Two library calls
    (counts, then the rows) with one host read of the total in between."""
    _need(bucket, "bucket", torch.int32)
    B, H, R, n = bucket.shape
    _need(perm, "perm", torch.int32, bucket.shape)
    _need(inv_perm, "inv_perm", torch.int32, bucket.shape)
    if valid_len is not None:
        _need(valid_len, "valid_len", torch.int32, (B,))
    a = LshAttnParams(LshParams(B, H, n, 8, 2, R, int(chunk), CRS_BF16), int(causal), int(no_self), 1, 1.0)
    row_ptr = torch.empty(B * H * n + 1, dtype=torch.int64, device=bucket.device)
    args = (ctypes.byref(a), _ptr(bucket), _ptr(perm), _ptr(inv_perm), _ptr(valid_len), _ptr(row_ptr))
    _check("crs_lsh_candidates_csr", _lib.crs_lsh_candidates_csr(*args, None, _stream(stream)))
    nnz = int(row_ptr[-1].item())
    col = torch.empty(max(nnz, 1), dtype=torch.int32, device=bucket.device)
    _check("crs_lsh_candidates_csr", _lib.crs_lsh_candidates_csr(*args, _ptr(col), _stream(stream)))
    return row_ptr, col[:nnz]


def indexer_topk(q_idx, w, k_idx, topk: int, mode: int = CRS_IDX_PREFILL, k_offsets=None,
                 max_keys: int = 0, out=None, count=None, workspace=None, stream=None):
    """Lightning-indexer top-k; returns (idx [rows, topk] int32 ascending, -1 pad; count [rows])."""
    _need(q_idx, "q_idx", torch.bfloat16)
    rows, heads, d = q_idx.shape
    _need(w, "w", torch.float32, (rows, heads))
    _need(k_idx, "k_idx", torch.bfloat16)
    if mode == CRS_IDX_DECODE:
        _need(k_offsets, "k_offsets", torch.int64, (rows + 1,))
    p = IndexerParams(int(mode), rows, heads, d, int(topk), int(max_keys))
    if out is None:
        out = torch.empty((rows, topk), dtype=torch.int32, device=q_idx.device)
    if count is None:
        count = torch.empty((rows,), dtype=torch.int32, device=q_idx.device)
    _need(out, "out", torch.int32, (rows, topk))
    _need(count, "count", torch.int32, (rows,))
    ws, wsb = _workspace(int(_lib.crs_indexer_topk_workspace_size(ctypes.byref(p))),
                         q_idx.device, workspace)
    st = _lib.crs_indexer_topk(ctypes.byref(p), _ptr(q_idx), _ptr(w), _ptr(k_idx),
                               _ptr(k_offsets), _ptr(out), _ptr(count), _ptr(ws), wsb,
                               _stream(stream))
    _check("crs_indexer_topk", st)
    return out, count


# ---------------------------------------------------------------- routing --
def route_attn(Q, K, V, M, m: int, causal=True, no_self=False, scale=None, out=None, lse=None, count=None,
               JQ=None, JK=None, workspace=None, stream=None):
    """Routing attention with quota execution: Q, K, V [B, H, n, d] bf16, M [H, C, d] f32
    (frozen centres), quota m -> (JQ, JK [B, H, C, m], O [B, H, n, d] f32, lse, count)."""
    _need(Q, "Q", torch.bfloat16)
    B, H, n, d = Q.shape
    _need(K, "K", torch.bfloat16, (B, H, n, d))
    _need(V, "V", torch.bfloat16, (B, H, n, d))
    _need(M, "M", torch.float32)
    C = M.shape[1]
    _need(M, "M", torch.float32, (H, C, d))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    p = RouteParams(B, H, n, d, C, int(m), int(causal), int(no_self), float(scale))
    dev = Q.device
    JQ = torch.empty((B, H, C, m), dtype=torch.int32, device=dev) if JQ is None else JQ
    JK = torch.empty((B, H, C, m), dtype=torch.int32, device=dev) if JK is None else JK
    out = torch.empty((B, H, n, d), dtype=torch.float32, device=dev) if out is None else out
    lse = torch.empty((B, H, n), dtype=torch.float32, device=dev) if lse is None else lse
    count = torch.empty((B, H, n), dtype=torch.int32, device=dev) if count is None else count
    ws, wsb = _workspace(int(_lib.crs_route_attn_workspace_size(ctypes.byref(p))), dev, workspace)
    st = _lib.crs_route_attn(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(M), _ptr(JQ), _ptr(JK), _ptr(out),
                             _ptr(lse), _ptr(count), _ptr(ws), wsb, _stream(stream))
    _check("crs_route_attn", st)
    return JQ, JK, out, lse, count


# ------------------------------------------------------------- LSH decode --
class LshDecodeCache:
    """Device state of LSH attention in decode (paged K/V behind a block table, bucket
    lists of logical positions): see crs_lsh_decode_* in include/crs.h.  block_table maps
    each row's logical pages to physical pages of one pool (a permutation when given as
    "shuffled", so that rows' pages interleave as in a shared page pool)."""

    def __init__(self, n_seq, n_heads, n_buckets, n_rounds, max_len, d=64, page_size=64, list_page=64,
                 list_cap=None, n_list_pages=None, no_self=True, key_norm=True, scale=None, device="cuda",
                 shuffled=True, seed=0):
        max_pages = -(-max_len // page_size)
        if list_cap is None:
            list_cap = max(list_page, 4 * max_len // n_buckets)
        list_pages = -(-list_cap // list_page)
        if n_list_pages is None:
            n_list_pages = n_seq * n_heads * n_rounds * (n_buckets + -(-max_len // list_page))
        self.p = LshDecodeParams(n_seq, n_heads, d, n_buckets, n_rounds, page_size, max_pages, list_page,
                                 list_pages, n_list_pages, max_len, int(no_self), int(key_norm),
                                 float(scale if scale is not None else 1.0 / math.sqrt(d)))
        n_pages = n_seq * max_pages
        g = torch.Generator(device="cpu").manual_seed(seed)
        order = torch.randperm(n_pages, generator=g) if shuffled else torch.arange(n_pages)
        self.block_table = order.to(torch.int32).view(n_seq, max_pages).to(device)
        self.k_pool = torch.zeros((n_pages, page_size, n_heads, d), dtype=torch.bfloat16, device=device)
        self.v_pool = torch.zeros_like(self.k_pool)
        self.bucket_store = torch.zeros((n_seq, n_heads, n_rounds, max_len), dtype=torch.uint8, device=device)
        self.list_table = torch.full((n_seq, n_heads, n_rounds, n_buckets, list_pages), -1, dtype=torch.int32,
                                     device=device)
        self.list_len = torch.zeros((n_seq, n_heads, n_rounds, n_buckets), dtype=torch.int32, device=device)
        self.list_pool = torch.zeros((n_list_pages, list_page), dtype=torch.int32, device=device)
        self.alloc = torch.zeros((1,), dtype=torch.int32, device=device)
        self.seq_len = torch.zeros((n_seq,), dtype=torch.int32, device=device)
        self.st = LshDecodeState(*(t.data_ptr() for t in (self.k_pool, self.v_pool, self.block_table,
                                                         self.bucket_store, self.list_table, self.list_len,
                                                         self.list_pool, self.alloc, self.seq_len)))

    def prefill(self, x, v, rot, stream=None):
        """Append x, v [n_seq, n_tokens, n_heads, d] bf16 (rot [H, rounds, d, b/2] f32)."""
        _need(x, "x", torch.bfloat16)
        _need(v, "v", torch.bfloat16, tuple(x.shape))
        _need(rot, "rot", torch.float32)
        _check("crs_lsh_decode_prefill", _lib.crs_lsh_decode_prefill(ctypes.byref(self.p), ctypes.byref(self.st),
                                                                     _ptr(x), _ptr(v), _ptr(rot), x.shape[1],
                                                                     _stream(stream)))

    def step(self, x, v, rot, out=None, lse=None, count=None, stream=None):
        """Append one token per row (x, v [n_seq, 1, n_heads, d]) and attend with it ->
        (O [n_seq, n_heads, d] f32, lse [n_seq, n_heads], count [n_seq, n_heads])."""
        _need(x, "x", torch.bfloat16)
        _need(v, "v", torch.bfloat16, tuple(x.shape))
        S, H, d = self.p.n_seq, self.p.n_heads, self.p.d
        if out is None:
            out = torch.empty((S, H, d), dtype=torch.float32, device=x.device)
        if lse is None:
            lse = torch.empty((S, H), dtype=torch.float32, device=x.device)
        if count is None:
            count = torch.empty((S, H), dtype=torch.int32, device=x.device)
        _check("crs_lsh_decode_step", _lib.crs_lsh_decode_step(ctypes.byref(self.p), ctypes.byref(self.st), _ptr(x),
                                                               _ptr(v), _ptr(rot), _ptr(out), _ptr(lse), _ptr(count),
                                                               _stream(stream)))
        return out, lse, count


# ------------------------------------------------------------------- HISA --
def hisa_block_offsets(k_offsets, blk: int):
    """[rows + 1] int64 on k_offsets' device: first representative of each row (complete
    blocks of `blk` keys only).  Cache-layout bookkeeping, done when blocks fill."""
    ko = k_offsets.to("cpu", torch.int64)
    nb = (ko[1:] - ko[:-1]) // int(blk)
    bo = torch.zeros(ko.numel(), dtype=torch.int64)
    bo[1:] = torch.cumsum(nb, 0)
    return bo.to(k_offsets.device)


def hisa_describe(k_idx, k_offsets, blk: int, max_keys: int, blk_offsets=None, rep=None, stream=None):
    """Block representatives (mean index key per complete block) -> (rep [blocks, 64] f32,
    blk_offsets [rows + 1] int64)."""
    _need(k_idx, "k_idx", torch.bfloat16)
    rows = k_offsets.numel() - 1
    _need(k_offsets, "k_offsets", torch.int64, (rows + 1,))
    if blk_offsets is None:
        blk_offsets = hisa_block_offsets(k_offsets, blk)
    n_blocks = int(blk_offsets[-1].item())
    if rep is None:
        rep = torch.empty((max(1, n_blocks), k_idx.shape[1]), dtype=torch.float32, device=k_idx.device)
    p = HisaParams(rows, 1, k_idx.shape[1], 1, int(blk), 1, int(max_keys))
    _check("crs_hisa_describe", _lib.crs_hisa_describe(ctypes.byref(p), _ptr(k_idx), _ptr(k_offsets),
                                                       _ptr(blk_offsets), _ptr(rep), _stream(stream)))
    return rep, blk_offsets


def hisa_topk(q_idx, w, k_idx, k_offsets, rep, blk_offsets, topk: int, blk: int, top_blocks: int,
              max_keys: int, out_blocks=None, out=None, count=None, workspace=None, stream=None):
    """Hierarchical top-k for decode rows -> (blocks [rows, top_blocks], idx [rows, topk], count)."""
    _need(q_idx, "q_idx", torch.bfloat16)
    rows, heads, d = q_idx.shape
    _need(w, "w", torch.float32, (rows, heads))
    _need(k_idx, "k_idx", torch.bfloat16)
    _need(k_offsets, "k_offsets", torch.int64, (rows + 1,))
    _need(blk_offsets, "blk_offsets", torch.int64, (rows + 1,))
    _need(rep, "rep", torch.float32)
    p = HisaParams(rows, heads, d, int(topk), int(blk), int(top_blocks), int(max_keys))
    if out_blocks is None:
        out_blocks = torch.empty((rows, top_blocks), dtype=torch.int32, device=q_idx.device)
    if out is None:
        out = torch.empty((rows, topk), dtype=torch.int32, device=q_idx.device)
    if count is None:
        count = torch.empty((rows,), dtype=torch.int32, device=q_idx.device)
    _need(out_blocks, "out_blocks", torch.int32, (rows, top_blocks))
    _need(out, "out", torch.int32, (rows, topk))
    _need(count, "count", torch.int32, (rows,))
    ws, wsb = _workspace(int(_lib.crs_hisa_topk_workspace_size(ctypes.byref(p))), q_idx.device, workspace)
    st = _lib.crs_hisa_topk(ctypes.byref(p), _ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(k_offsets), _ptr(rep),
                            _ptr(blk_offsets), _ptr(out_blocks), _ptr(out), _ptr(count), _ptr(ws), wsb,
                            _stream(stream))
    _check("crs_hisa_topk", st)
    return out_blocks, out, count


# ----------------------------------------------------------------- blocks --
def hisa_topk_prefill(q_idx, w, k_idx, rep, topk: int, blk: int, top_blocks: int, out_blocks=None, out=None,
                      count=None, workspace=None, stream=None):
    """Hierarchical top-k for the n causal queries of one sequence -> (blocks [n,
    top_blocks], idx [n, topk], count [n]).  rep [n // blk, 64] from hisa_describe(k_idx,
    [0, n], blk, n)."""
    _need(q_idx, "q_idx", torch.bfloat16)
    n, H, d = q_idx.shape
    _need(w, "w", torch.float32, (n, H))
    _need(k_idx, "k_idx", torch.bfloat16, (n, d))
    _need(rep, "rep", torch.float32)
    p = HisaParams(n, H, d, int(topk), int(blk), int(top_blocks), n)
    if out_blocks is None:
        out_blocks = torch.empty((n, top_blocks), dtype=torch.int32, device=q_idx.device)
    if out is None:
        out = torch.empty((n, topk), dtype=torch.int32, device=q_idx.device)
    if count is None:
        count = torch.empty((n,), dtype=torch.int32, device=q_idx.device)
    _need(out_blocks, "out_blocks", torch.int32, (n, top_blocks))
    _need(out, "out", torch.int32, (n, topk))
    _need(count, "count", torch.int32, (n,))
    ws, wsb = _workspace(int(_lib.crs_hisa_topk_prefill_workspace_size(ctypes.byref(p))), q_idx.device, workspace)
    if wsb == 0:
        raise CrsError("crs_hisa_topk_prefill", 2)
    st = _lib.crs_hisa_topk_prefill(ctypes.byref(p), _ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(rep), _ptr(out_blocks),
                                    _ptr(out), _ptr(count), _ptr(ws), wsb, _stream(stream))
    _check("crs_hisa_topk_prefill", st)
    return out_blocks, out, count


def block_describe(K, L: int, rank: int, blk_range=None, mu=None, xi=None, stream=None):
    """Block descriptors of K [n_seq, T, n_kv, D] bf16 -> (mu, xi) fp32."""
    _need(K, "K", torch.bfloat16)
    n_seq, T, n_kv, D = K.shape
    nfull = T // L
    b0, b1 = (0, nfull) if blk_range is None else blk_range
    p = BlockParams(n_seq, n_kv, T, D, int(L), int(rank), int(b0), int(b1))
    if mu is None:
        mu = torch.empty((n_seq, n_kv, nfull, D), dtype=torch.float32, device=K.device)
    if xi is None:
        xi = torch.empty((n_seq, n_kv, nfull, rank, D), dtype=torch.float32, device=K.device)
    _need(mu, "mu", torch.float32, (n_seq, n_kv, nfull, D))
    _need(xi, "xi", torch.float32, (n_seq, n_kv, nfull, rank, D))
    st = _lib.crs_block_describe(ctypes.byref(p), _ptr(K), _ptr(mu), _ptr(xi), _stream(stream))
    _check("crs_block_describe", st)
    return mu, xi


def block_select(Q, mu, xi, T: int, L: int, top_blocks: int, window: int, scale=None,
                 tok=None, count=None, workspace=None, stream=None):
    """Block-mass selection -> (tok [n_seq, n_kv, top_blocks*L + window], count [n_seq, n_kv]).
    xi=None selects on the block means alone (the mean-pool selector, rank 0)."""
    _need(Q, "Q", torch.bfloat16)
    n_seq, n_q, D = Q.shape
    n_kv, nfull = mu.shape[1], mu.shape[2]
    rank = 0 if xi is None else xi.shape[3]
    _need(mu, "mu", torch.float32, (n_seq, n_kv, nfull, D))
    if xi is not None:
        _need(xi, "xi", torch.float32, (n_seq, n_kv, nfull, rank, D))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    p = BlockSelParams(BlockParams(n_seq, n_kv, int(T), D, int(L), rank, 0, nfull), n_q,
                       int(top_blocks), int(window), float(scale))
    cap = top_blocks * L + window
    if tok is None:
        tok = torch.empty((n_seq, n_kv, cap), dtype=torch.int32, device=Q.device)
    if count is None:
        count = torch.empty((n_seq, n_kv), dtype=torch.int32, device=Q.device)
    _need(tok, "tok", torch.int32, (n_seq, n_kv, cap))
    _need(count, "count", torch.int32, (n_seq, n_kv))
    ws, wsb = _workspace(int(_lib.crs_block_select_workspace_size(ctypes.byref(p))), Q.device,
                         workspace)
    st = _lib.crs_block_select(ctypes.byref(p), _ptr(Q), _ptr(mu), _ptr(xi), _ptr(tok),
                               _ptr(count), _ptr(ws), wsb, _stream(stream))
    _check("crs_block_select", st)
    return tok, count


def block_describe_ss(K, L: int, rank: int, U, out=None, stream=None):
    """Query-subspace descriptors: K [n_seq, T, n_kv, D] bf16, U [D, s] f32 ->
    (mu [n_seq, n_kv, T//L, D], xi_ss [n_seq, n_kv, T//L, rank, s]) f32."""
    _need(K, "K", torch.bfloat16)
    n_seq, T, n_kv, D = K.shape
    _need(U, "U", torch.float32)
    sd = U.shape[1]
    _need(U, "U", torch.float32, (D, sd))
    nfull = T // L
    if out is None:
        out = (torch.empty((n_seq, n_kv, nfull, D), dtype=torch.float32, device=K.device),
               torch.empty((n_seq, n_kv, nfull, rank, sd), dtype=torch.float32, device=K.device))
    mu, xi = out
    _need(mu, "mu", torch.float32, (n_seq, n_kv, nfull, D))
    _need(xi, "xi_ss", torch.float32, (n_seq, n_kv, nfull, rank, sd))
    p = BlockParams(n_seq, n_kv, int(T), D, int(L), int(rank), 0, nfull)
    _check("crs_block_describe_ss", _lib.crs_block_describe_ss(ctypes.byref(p), _ptr(K), _ptr(U), sd, _ptr(mu),
                                                               _ptr(xi), _stream(stream)))
    return mu, xi


def block_select_ss(Q, U, mu, xi_ss, T: int, L: int, top_blocks: int, window: int, scale=None,
                    tok=None, count=None, workspace=None, stream=None):
    """block_select on query-subspace descriptors (from block_describe_ss)."""
    _need(Q, "Q", torch.bfloat16)
    n_seq, n_q, D = Q.shape
    n_kv, nfull, rank, sd = xi_ss.shape[1], xi_ss.shape[2], xi_ss.shape[3], xi_ss.shape[4]
    _need(U, "U", torch.float32, (D, sd))
    _need(mu, "mu", torch.float32, (n_seq, n_kv, nfull, D))
    _need(xi_ss, "xi_ss", torch.float32, (n_seq, n_kv, nfull, rank, sd))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    p = BlockSelParams(BlockParams(n_seq, n_kv, int(T), D, int(L), rank, 0, nfull), n_q,
                       int(top_blocks), int(window), float(scale))
    cap = top_blocks * L + window
    if tok is None:
        tok = torch.empty((n_seq, n_kv, cap), dtype=torch.int32, device=Q.device)
    if count is None:
        count = torch.empty((n_seq, n_kv), dtype=torch.int32, device=Q.device)
    _need(tok, "tok", torch.int32, (n_seq, n_kv, cap))
    _need(count, "count", torch.int32, (n_seq, n_kv))
    ws, wsb = _workspace(int(_lib.crs_block_select_ss_workspace_size(ctypes.byref(p), sd)), Q.device,
                         workspace)
    st = _lib.crs_block_select_ss(ctypes.byref(p), _ptr(Q), _ptr(U), sd, _ptr(mu), _ptr(xi_ss), _ptr(tok),
                                  _ptr(count), _ptr(ws), wsb, _stream(stream))
    _check("crs_block_select_ss", st)
    return tok, count


def quest_describe(K, L: int, out=None, stream=None):
    """Quest summaries: K [n_seq, T, n_kv, D] bf16 -> (kmin, kmax) [n_seq, n_kv, T // L, D] bf16."""
    _need(K, "K", torch.bfloat16)
    n_seq, T, n_kv, D = K.shape
    nfull = T // L
    if out is None:
        out = (torch.empty((n_seq, n_kv, nfull, D), dtype=torch.bfloat16, device=K.device),
               torch.empty((n_seq, n_kv, nfull, D), dtype=torch.bfloat16, device=K.device))
    kmin, kmax = out
    _need(kmin, "kmin", torch.bfloat16, (n_seq, n_kv, nfull, D))
    _need(kmax, "kmax", torch.bfloat16, (n_seq, n_kv, nfull, D))
    p = BlockParams(n_seq, n_kv, int(T), D, int(L), 0, 0, nfull)
    _check("crs_block_quest_describe", _lib.crs_block_quest_describe(ctypes.byref(p), _ptr(K), _ptr(kmin),
                                                                     _ptr(kmax), _stream(stream)))
    return kmin, kmax


def block_select_quest(Q, kmin, kmax, T: int, L: int, top_blocks: int, window: int, scale=None,
                       tok=None, count=None, workspace=None, stream=None):
    """block_select with the Quest box score (summaries from quest_describe)."""
    _need(Q, "Q", torch.bfloat16)
    n_seq, n_q, D = Q.shape
    n_kv, nfull = kmin.shape[1], kmin.shape[2]
    _need(kmin, "kmin", torch.bfloat16, (n_seq, n_kv, nfull, D))
    _need(kmax, "kmax", torch.bfloat16, (n_seq, n_kv, nfull, D))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    p = BlockSelParams(BlockParams(n_seq, n_kv, int(T), D, int(L), 0, 0, nfull), n_q,
                       int(top_blocks), int(window), float(scale))
    cap = top_blocks * L + window
    if tok is None:
        tok = torch.empty((n_seq, n_kv, cap), dtype=torch.int32, device=Q.device)
    if count is None:
        count = torch.empty((n_seq, n_kv), dtype=torch.int32, device=Q.device)
    _need(tok, "tok", torch.int32, (n_seq, n_kv, cap))
    _need(count, "count", torch.int32, (n_seq, n_kv))
    ws, wsb = _workspace(int(_lib.crs_block_select_workspace_size(ctypes.byref(p))), Q.device,
                         workspace)
    st = _lib.crs_block_select_quest(ctypes.byref(p), _ptr(Q), _ptr(kmin), _ptr(kmax), _ptr(tok),
                                     _ptr(count), _ptr(ws), wsb, _stream(stream))
    _check("crs_block_select_quest", st)
    return tok, count


def block_quantize(mu, xi, T: int, L: int, out=None, stream=None):
    """Deployed descriptor compression: mu -> bf16, xi -> FP4 codes + fp32 scales.
    Returns (mu16 [.., D] bf16, xi4 [.., rank, D/2] uint8, xi_scale [.., rank] fp32)."""
    _need(mu, "mu", torch.float32)
    n_seq, n_kv, nfull, D = mu.shape
    rank = xi.shape[3]
    _need(xi, "xi", torch.float32, (n_seq, n_kv, nfull, rank, D))
    if out is None:
        out = (torch.empty((n_seq, n_kv, nfull, D), dtype=torch.bfloat16, device=mu.device),
               torch.empty((n_seq, n_kv, nfull, rank, D // 2), dtype=torch.uint8, device=mu.device),
               torch.empty((n_seq, n_kv, nfull, rank), dtype=torch.float32, device=mu.device))
    mu16, xi4, xs = out
    _need(mu16, "mu16", torch.bfloat16, (n_seq, n_kv, nfull, D))
    _need(xi4, "xi4", torch.uint8, (n_seq, n_kv, nfull, rank, D // 2))
    _need(xs, "xi_scale", torch.float32, (n_seq, n_kv, nfull, rank))
    p = BlockParams(n_seq, n_kv, int(T), D, int(L), rank, 0, nfull)
    _check("crs_block_quantize", _lib.crs_block_quantize(ctypes.byref(p), _ptr(mu), _ptr(xi), _ptr(mu16),
                                                         _ptr(xi4), _ptr(xs), _stream(stream)))
    return mu16, xi4, xs


def block_select_fp4(Q, mu16, xi4, xi_scale, T: int, L: int, top_blocks: int, window: int,
                     scale=None, tok=None, count=None, workspace=None, stream=None):
    """block_select on compressed descriptors (from block_quantize)."""
    _need(Q, "Q", torch.bfloat16)
    n_seq, n_q, D = Q.shape
    n_kv, nfull, rank = mu16.shape[1], mu16.shape[2], xi4.shape[3]
    _need(mu16, "mu16", torch.bfloat16, (n_seq, n_kv, nfull, D))
    _need(xi4, "xi4", torch.uint8, (n_seq, n_kv, nfull, rank, D // 2))
    _need(xi_scale, "xi_scale", torch.float32, (n_seq, n_kv, nfull, rank))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    p = BlockSelParams(BlockParams(n_seq, n_kv, int(T), D, int(L), rank, 0, nfull), n_q,
                       int(top_blocks), int(window), float(scale))
    cap = top_blocks * L + window
    if tok is None:
        tok = torch.empty((n_seq, n_kv, cap), dtype=torch.int32, device=Q.device)
    if count is None:
        count = torch.empty((n_seq, n_kv), dtype=torch.int32, device=Q.device)
    _need(tok, "tok", torch.int32, (n_seq, n_kv, cap))
    _need(count, "count", torch.int32, (n_seq, n_kv))
    ws, wsb = _workspace(int(_lib.crs_block_select_workspace_size(ctypes.byref(p))), Q.device,
                         workspace)
    st = _lib.crs_block_select_fp4(ctypes.byref(p), _ptr(Q), _ptr(mu16), _ptr(xi4), _ptr(xi_scale),
                                   _ptr(tok), _ptr(count), _ptr(ws), wsb, _stream(stream))
    _check("crs_block_select_fp4", st)
    return tok, count


SS_CODE_BYTES = 48        # stored codes per subspace eigenvector (96 dims, those past sd zero)


def block_quantize_ss(mu, xi_ss, T: int, L: int, out=None, stream=None):
    """The deployed descriptor: mu -> bf16 (full space), the query-subspace eigenvectors
    xi_ss [.., rank, sd] (sd <= 96) -> FP4 codes [.., rank, 48] + fp32 scales."""
    _need(mu, "mu", torch.float32)
    n_seq, n_kv, nfull, D = mu.shape
    rank, sd = xi_ss.shape[3], xi_ss.shape[4]
    _need(xi_ss, "xi_ss", torch.float32, (n_seq, n_kv, nfull, rank, sd))
    if out is None:
        out = (torch.empty((n_seq, n_kv, nfull, D), dtype=torch.bfloat16, device=mu.device),
               torch.empty((n_seq, n_kv, nfull, rank, SS_CODE_BYTES), dtype=torch.uint8, device=mu.device),
               torch.empty((n_seq, n_kv, nfull, rank), dtype=torch.float32, device=mu.device))
    mu16, xi4, xs = out
    _need(mu16, "mu16", torch.bfloat16, (n_seq, n_kv, nfull, D))
    _need(xi4, "xi4", torch.uint8, (n_seq, n_kv, nfull, rank, SS_CODE_BYTES))
    _need(xs, "xi_scale", torch.float32, (n_seq, n_kv, nfull, rank))
    p = BlockParams(n_seq, n_kv, int(T), D, int(L), rank, 0, nfull)
    _check("crs_block_quantize_ss", _lib.crs_block_quantize_ss(ctypes.byref(p), _ptr(mu), _ptr(xi_ss), int(sd),
                                                               _ptr(mu16), _ptr(xi4), _ptr(xs), _stream(stream)))
    return mu16, xi4, xs


def block_select_fp4_ss(Q, U, mu16, xi4, xi_scale, T: int, L: int, top_blocks: int, window: int, scale=None,
                        tok=None, count=None, workspace=None, stream=None):
    """block_select on the deployed descriptor (bf16 means, FP4 query-subspace
    eigenvectors from block_quantize_ss); U [D, sd] the subspace basis."""
    _need(Q, "Q", torch.bfloat16)
    n_seq, n_q, D = Q.shape
    _need(U, "U", torch.float32)
    sd = U.shape[1]
    n_kv, nfull, rank = mu16.shape[1], mu16.shape[2], xi4.shape[3]
    _need(mu16, "mu16", torch.bfloat16, (n_seq, n_kv, nfull, D))
    _need(xi4, "xi4", torch.uint8, (n_seq, n_kv, nfull, rank, SS_CODE_BYTES))
    _need(xi_scale, "xi_scale", torch.float32, (n_seq, n_kv, nfull, rank))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    p = BlockSelParams(BlockParams(n_seq, n_kv, int(T), D, int(L), rank, 0, nfull), n_q,
                       int(top_blocks), int(window), float(scale))
    cap = top_blocks * L + window
    if tok is None:
        tok = torch.empty((n_seq, n_kv, cap), dtype=torch.int32, device=Q.device)
    if count is None:
        count = torch.empty((n_seq, n_kv), dtype=torch.int32, device=Q.device)
    _need(tok, "tok", torch.int32, (n_seq, n_kv, cap))
    _need(count, "count", torch.int32, (n_seq, n_kv))
    ws, wsb = _workspace(int(_lib.crs_block_select_fp4_ss_workspace_size(ctypes.byref(p), int(sd))), Q.device,
                         workspace)
    st = _lib.crs_block_select_fp4_ss(ctypes.byref(p), _ptr(Q), _ptr(U), int(sd), _ptr(mu16), _ptr(xi4),
                                      _ptr(xi_scale), _ptr(tok), _ptr(count), _ptr(ws), wsb, _stream(stream))
    _check("crs_block_select_fp4_ss", st)
    return tok, count


NOALLOC_SCRATCH_BYTES = 16 << 20


def block_select_noalloc(Q, mu, xi, T: int, L: int, top_blocks: int, window: int, scale=None,
                         tok=None, count=None, stream=None):
    """block_select for callers that cannot allocate device memory at call time.

    Same inputs and outputs as block_select, but the scratch is a static 16 MiB
    device array inside libcrs (no workspace is allocated): problems with
    n_seq * n_q * (T // L) > 4,194,304 scores are rejected.  The first call on a
    device looks up that array's address; calls that overlap on the GPU share
    the array and race.  Pass preallocated ``tok``/``count`` to allocate nothing
    on the Python side either."""
    _need(Q, "Q", torch.bfloat16)
    n_seq, n_q, D = Q.shape
    n_kv, nfull, rank = mu.shape[1], mu.shape[2], xi.shape[3]
    _need(mu, "mu", torch.float32, (n_seq, n_kv, nfull, D))
    _need(xi, "xi", torch.float32, (n_seq, n_kv, nfull, rank, D))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    p = BlockSelParams(BlockParams(n_seq, n_kv, int(T), D, int(L), rank, 0, nfull), n_q,
                       int(top_blocks), int(window), float(scale))
    cap = top_blocks * L + window
    if tok is None:
        tok = torch.empty((n_seq, n_kv, cap), dtype=torch.int32, device=Q.device)
    if count is None:
        count = torch.empty((n_seq, n_kv), dtype=torch.int32, device=Q.device)
    _need(tok, "tok", torch.int32, (n_seq, n_kv, cap))
    _need(count, "count", torch.int32, (n_seq, n_kv))
    st = _lib.crs_block_select_noalloc(ctypes.byref(p), _ptr(Q), _ptr(mu), _ptr(xi), _ptr(tok),
                                       _ptr(count), _stream(stream))
    _check("crs_block_select_noalloc", st)
    return tok, count


# -------------------------------------------------------------- attention --
def sparse_attn(Q, K, V, I, kv_base=None, scale=None, key_valid=None, q_pos=None, out=None,
                lse=None, workspace=None, stream=None):
    """Attention over index lists -> (O [rows, n_q, D] fp32, lse).  Q [rows, n_q, D];
    K, V [tokens, n_kv, D] (token j of row t at kv_base[t] + j); I [rows, n_lists,
    max_idx] (n_lists 1 or n_kv).  key_valid [tokens] uint8/bool (0 = padding key)
    and q_pos [rows] int32 (entries j > q_pos[t] skipped) are optional masks.  Every
    entry is bounds-checked against K's token count on the device."""
    _need(Q, "Q", torch.bfloat16)
    rows, n_q, D = Q.shape
    _need(K, "K", torch.bfloat16)
    _need(V, "V", torch.bfloat16, K.shape)
    n_kv = K.shape[-2]
    if I.dim() == 2:
        I = I.view(rows, 1, I.shape[1])
    _need(I, "I", torch.int32)
    n_lists, max_idx = I.shape[1], I.shape[2]
    if kv_base is not None:
        _need(kv_base, "kv_base", torch.int64, (rows,))
    n_keys = K.numel() // (n_kv * D)
    if key_valid is not None:
        if key_valid.dtype == torch.bool:
            key_valid = key_valid.view(torch.uint8)
        _need(key_valid, "key_valid", torch.uint8, (n_keys,))
    if q_pos is not None:
        _need(q_pos, "q_pos", torch.int32, (rows,))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    p = AttnParams(rows, n_q, n_kv, D, max_idx, n_lists, int(n_keys), float(scale))
    if out is None:
        out = torch.empty((rows, n_q, D), dtype=torch.float32, device=Q.device)
    _need(out, "out", torch.float32, (rows, n_q, D))
    if lse is not None:
        _need(lse, "lse", torch.float32, (rows, n_q))
    ws, wsb = _workspace(int(_lib.crs_sparse_attn_workspace_size(ctypes.byref(p))), Q.device,
                         workspace)
    st = _lib.crs_sparse_attn(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(kv_base),
                              _ptr(I), _ptr(key_valid), _ptr(q_pos), _ptr(out), _ptr(lse),
                              _ptr(ws), wsb, _stream(stream))
    _check("crs_sparse_attn", st)
    return out, lse
