"""CPU oracle for content-routed sparse attention (ctypes wrapper).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  It shares no code with the CUDA path; the arithmetic lives in
``crs_oracle.c`` (plain C, fp64) and this module only marshals numpy arrays.

Parity status per function (pins in ``tests/test_oracle_*.py``):
  lsh_hash / lsh_sort / lsh_candidates / lsh_attn  -- pinned
  indexer_topk / indexer_score                     -- pinned
  block_describe / block_log_mass / block_select   -- pinned (rank 0 = mean-pool selector)
  quest_describe / quest_select                    -- pinned
  block_describe_ss / block_select_ss              -- pinned
  hisa_describe / hisa_topk / hisa_topk_prefill    -- pinned
  lsh_decode                                       -- pinned
  kmeans_route                                     -- pinned
  fp4_quantize / fp4_dequantize                    -- pinned
  sparse_attn                                      -- pinned
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import numpy as np

from . import build as _build

_LIB = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        I, L, D = ctypes.c_int, ctypes.c_long, ctypes.c_double
        lib.oracle_set_num_threads.argtypes = [I]
        lib.oracle_max_threads.restype = I
        lib.oracle_lsh_hash.argtypes = [I, I, I, I, I, I, _f32p, _f32p, _i32p]
        lib.oracle_lsh_margin.argtypes = [I, I, I, I, I, I, _f32p, _f32p, _f64p]
        lib.oracle_lsh_sort.argtypes = [I, I, _i32p, _i32p, _i32p]
        lib.oracle_lsh_candidates.argtypes = [I, I, I, I, I, I, _i32p, _i32p, _i32p, I, _i32p, _u8p]
        lib.oracle_lsh_candidates.restype = I
        lib.oracle_lsh_attn.argtypes = [I, I, I, I, I, I, I, I, I, D, _f64p, _f64p, _i32p, _i32p,
                                        _i32p, _i32p, _i32p, I, _f64p, _f64p, _i32p]
        lib.oracle_indexer_score.argtypes = [I, I, _f64p, _f64p, _f64p, L, _f64p]
        lib.oracle_indexer_topk.argtypes = [I, I, I, I, _f64p, _f64p, _f64p, _i64p, _i32p, _i32p,
                                            _i32p, _f64p, _f64p]
        lib.oracle_block_describe.argtypes = [I, I, I, I, _f64p, _i32p, _f64p, _f64p, _f64p]
        lib.oracle_block_log_mass.argtypes = [I, I, _f64p, _f64p]
        lib.oracle_block_log_mass.restype = D
        lib.oracle_fp4_quantize.argtypes = [I, I, _f32p, _u8p, _f32p]
        lib.oracle_fp4_dequantize.argtypes = [I, I, _u8p, _f32p, _f64p]
        lib.oracle_block_select.argtypes = [I, I, I, I, I, I, I, I, I, I, D, _f64p, _f64p, _f64p,
                                            I, _i32p, _i32p, _i32p, _f64p]
        lib.oracle_block_describe_ss.argtypes = [I, I, I, I, I, _f64p, _f64p, _f64p, _f64p, _f64p]
        lib.oracle_block_select_ss.argtypes = [I, I, I, I, I, I, I, I, I, I, I, D, _f64p, _f64p, _f64p,
                                               _f64p, I, _i32p, _i32p, _i32p, _f64p]
        lib.oracle_kmeans_route.argtypes = [I, I, I, I, I, I, I, I, D, _f32p, _f32p, _f32p, _f64p, _f64p, _f64p,
                                            _i32p, _i32p, _f64p, _f64p, _i32p]
        lib.oracle_lsh_decode.argtypes = [I, I, I, I, I, I, I, D, _f64p, _f64p, _i32p, _i32p, _f64p, _f64p,
                                          _i32p]
        lib.oracle_hisa_describe.argtypes = [I, I, I, _f64p, _i64p, _i64p, _f64p]
        lib.oracle_hisa_topk.argtypes = [I, I, I, I, I, I, _f64p, _f64p, _f64p, _i64p, _f64p, _i64p, _i32p,
                                         _i32p, _i32p, _i32p, _f64p]
        lib.oracle_quest_describe.argtypes = [I, I, I, I, I, _f64p, _f64p, _f64p]
        lib.oracle_hisa_topk_prefill.argtypes = [I, I, I, I, I, I, _f64p, _f64p, _f64p, _f64p, _i32p, _i32p, _i32p]
        lib.oracle_quest_select.argtypes = [I, I, I, I, I, I, I, I, I, D, _f64p, _f64p, _f64p, I,
                                            _i32p, _i32p, _i32p, _f64p]
        lib.oracle_sparse_attn.argtypes = [I, I, I, I, D, _f64p, _f64p, _f64p, _i64p, _i32p, I, I,
                                           _u8p, _i32p, _f64p, _f64p]
        _LIB = lib
    return _LIB


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a, ctype):
    return a.ctypes.data_as(ctype)


def set_threads(n: Optional[int]) -> None:
    """Number of OpenMP threads used by later calls (None: every core)."""
    _lib().oracle_set_num_threads(int(n) if n is not None else (os.cpu_count() or 1))


def threads() -> int:
    """Number of OpenMP threads later calls use."""
    return int(_lib().oracle_max_threads())


# ---------------------------------------------------------------- LSH --
def lsh_hash(X, R, n_buckets):
    """Bucket ids [B,H,rounds,n] from X [B,H,n,d] (fp32 values) and R [H,rounds,d,b/2]."""
    X = _c(X, np.float32)
    R = _c(R, np.float32)
    B, H, n, d = X.shape
    rounds = R.shape[1]
    out = np.empty((B, H, rounds, n), dtype=np.int32)
    _lib().oracle_lsh_hash(B, H, n, d, n_buckets, rounds, _p(X, _f32p), _p(R, _f32p),
                           _p(out, _i32p))
    return out


def lsh_margin(X, R, n_buckets):
    """fp64 gap between the two largest entries of [u; -u] per decision."""
    X = _c(X, np.float32)
    R = _c(R, np.float32)
    B, H, n, d = X.shape
    rounds = R.shape[1]
    out = np.empty((B, H, rounds, n), dtype=np.float64)
    _lib().oracle_lsh_margin(B, H, n, d, n_buckets, rounds, _p(X, _f32p), _p(R, _f32p),
                             _p(out, _f64p))
    return out


def lsh_sort(bucket):
    """(perm, inv_perm) with the shape of ``bucket`` (last axis = positions)."""
    bucket = _c(bucket, np.int32)
    n = bucket.shape[-1]
    segs = bucket.size // n
    perm = np.empty_like(bucket)
    inv = np.empty_like(bucket)
    _lib().oracle_lsh_sort(segs, n, _p(bucket, _i32p), _p(perm, _i32p), _p(inv, _i32p))
    return perm, inv


def lsh_candidates(bucket_bh, perm_bh, inv_bh, i, chunk, causal, no_self, valid_len):
    """U(i) for one (batch, head): arrays [rounds, n]; returns ascending int32 array."""
    bucket_bh = _c(bucket_bh, np.int32)
    perm_bh = _c(perm_bh, np.int32)
    inv_bh = _c(inv_bh, np.int32)
    rounds, n = bucket_bh.shape
    cand = np.empty(n, dtype=np.int32)
    mark = np.zeros(n, dtype=np.uint8)
    cnt = _lib().oracle_lsh_candidates(n, rounds, chunk, int(causal), int(no_self),
                                       int(valid_len), _p(bucket_bh, _i32p), _p(perm_bh, _i32p),
                                       _p(inv_bh, _i32p), int(i), _p(cand, _i32p),
                                       _p(mark, _u8p))
    return cand[:cnt].copy()


def lsh_attn(QK, V, bucket, perm, inv_perm, valid_len, chunk, causal=1, no_self=0,
             key_norm=1, scale=None, rows=None):
    """LSH attention over the union candidate sets (fp64).

    QK, V [B,H,n,d]; bucket/perm/inv_perm [B,H,rounds,n]; valid_len [B].
    Returns (O [B,H,nr,d], lse [B,H,nr], count [B,H,nr]) for the query
    positions ``rows`` (all when None).
    """
    QK = _c(QK, np.float64)
    V = _c(V, np.float64)
    B, H, n, d = QK.shape
    bucket = _c(bucket, np.int32)
    perm = _c(perm, np.int32)
    inv_perm = _c(inv_perm, np.int32)
    rounds = bucket.shape[2]
    vl = _c(valid_len, np.int32)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if rows is None:
        nr, rp = n, None
    else:
        rows = _c(rows, np.int32)
        nr, rp = rows.size, _p(rows, _i32p)
    O = np.empty((B, H, nr, d), dtype=np.float64)
    lse = np.empty((B, H, nr), dtype=np.float64)
    cnt = np.empty((B, H, nr), dtype=np.int32)
    _lib().oracle_lsh_attn(B, H, n, d, rounds, chunk, int(causal), int(no_self), int(key_norm),
                           float(scale), _p(QK, _f64p), _p(V, _f64p), _p(bucket, _i32p),
                           _p(perm, _i32p), _p(inv_perm, _i32p), _p(vl, _i32p), rp, nr,
                           _p(O, _f64p), _p(lse, _f64p), _p(cnt, _i32p))
    return O, lse, cnt


# ------------------------------------------------------------ indexer --
def indexer_score(q, w, K):
    """Scores r_s for one query: q [heads, d], w [heads], K [n_keys, d]."""
    q = _c(q, np.float64)
    w = _c(w, np.float64)
    K = _c(K, np.float64)
    out = np.empty(K.shape[0], dtype=np.float64)
    _lib().oracle_indexer_score(q.shape[0], q.shape[1], _p(q, _f64p), _p(w, _f64p),
                                _p(K, _f64p), K.shape[0], _p(out, _f64p))
    return out


def indexer_topk(q, w, K, key_base, n_visible, topk):
    """Top-k per row.  q [rows, heads, d]; w [rows, heads]; K [keys, d];
    key_base [rows] (first key of the row's sequence); n_visible [rows].
    Returns (idx [rows, topk] ascending, -1 padded; count; cutoff; next)."""
    q = _c(q, np.float64)
    w = _c(w, np.float64)
    K = _c(K, np.float64)
    kb = _c(key_base, np.int64)
    nv = _c(n_visible, np.int32)
    rows, heads, d = q.shape
    idx = np.empty((rows, topk), dtype=np.int32)
    cnt = np.empty(rows, dtype=np.int32)
    cut = np.empty(rows, dtype=np.float64)
    nxt = np.empty(rows, dtype=np.float64)
    _lib().oracle_indexer_topk(rows, heads, d, topk, _p(q, _f64p), _p(w, _f64p), _p(K, _f64p),
                               _p(kb, _i64p), _p(nv, _i32p), _p(idx, _i32p), _p(cnt, _i32p),
                               _p(cut, _f64p), _p(nxt, _f64p))
    return idx, cnt, cut, nxt


def kmeans_route(Q, K, V, M, m, causal=True, no_self=False, scale=None):
    """Routing attention with quota execution.  Q, K, V [B, H, n, d] (Q, K also scored in
    fp32), M [H, C, d] frozen centres, quota m.  Returns (JQ, JK [B, H, C, m] ascending,
    -1 padded; O [B, H, n, d]; lse [B, H, n]; count [B, H, n])."""
    Qf = _c(Q, np.float32)
    Kf = _c(K, np.float32)
    Mf = _c(M, np.float32)
    B, H, n, d = Qf.shape
    C = Mf.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    JQ = np.empty((B, H, C, m), dtype=np.int32)
    JK = np.empty((B, H, C, m), dtype=np.int32)
    O = np.empty((B, H, n, d), dtype=np.float64)
    lse = np.empty((B, H, n), dtype=np.float64)
    cnt = np.empty((B, H, n), dtype=np.int32)
    _lib().oracle_kmeans_route(B, H, n, d, C, m, int(causal), int(no_self), float(scale), _p(Qf, _f32p),
                               _p(Kf, _f32p), _p(Mf, _f32p), _p(_c(Q, np.float64), _f64p),
                               _p(_c(K, np.float64), _f64p), _p(_c(V, np.float64), _f64p), _p(JQ, _i32p),
                               _p(JK, _i32p), _p(O, _f64p), _p(lse, _f64p), _p(cnt, _i32p))
    return JQ, JK, O, lse, cnt


def lsh_decode(X, V, R, n_buckets, lengths, no_self=True, key_norm=True, scale=None):
    """LSH decode step for the newest token of each row.  X, V [S, H, n_max, d] (X also
    hashed in fp32 by lsh_hash), R [H, rounds, d, b/2]; lengths [S] (tokens including the
    new one).  Returns (O [S, H, d], lse [S, H], count [S, H])."""
    Xf = np.ascontiguousarray(X, dtype=np.float32)
    S, H, n_max, d = Xf.shape
    rounds = np.asarray(R).shape[1]
    bucket = lsh_hash(Xf, R, n_buckets)
    Xd = _c(X, np.float64)
    Vd = _c(V, np.float64)
    ln = _c(lengths, np.int32)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.zeros((S, H, d), dtype=np.float64)
    lse = np.empty((S, H), dtype=np.float64)
    cnt = np.empty((S, H), dtype=np.int32)
    _lib().oracle_lsh_decode(S, H, n_max, d, rounds, int(no_self), int(key_norm), float(scale), _p(Xd, _f64p),
                             _p(Vd, _f64p), _p(_c(bucket, np.int32), _i32p), _p(ln, _i32p), _p(O, _f64p),
                             _p(lse, _f64p), _p(cnt, _i32p))
    return O, lse, cnt


def hisa_block_offsets(k_offsets, blk):
    """[n_rows + 1] int64: first representative of each row (complete blocks only)."""
    ko = np.asarray(k_offsets, dtype=np.int64)
    nb = (ko[1:] - ko[:-1]) // blk
    return np.concatenate([[0], np.cumsum(nb)]).astype(np.int64)


def hisa_describe(K, k_offsets, blk):
    """Block representatives (mean index key per complete block).  K [keys, d]."""
    K = _c(K, np.float64)
    ko = _c(k_offsets, np.int64)
    bo = hisa_block_offsets(ko, blk)
    n_rows, d = len(ko) - 1, K.shape[1]
    rep = np.zeros((int(bo[-1]), d), dtype=np.float64)
    _lib().oracle_hisa_describe(n_rows, d, blk, _p(K, _f64p), _p(ko, _i64p), _p(bo, _i64p), _p(rep, _f64p))
    return rep, bo


def hisa_topk(q, w, K, k_offsets, rep, blk_offsets, topk, blk, top_blocks, given_blocks=None):
    """Hierarchical top-k for decode rows.  Returns (blocks [rows, top_blocks] ascending,
    idx [rows, topk] ascending, count [rows], coarse scores [n_blocks])."""
    q = _c(q, np.float64)
    w = _c(w, np.float64)
    K = _c(K, np.float64)
    ko = _c(k_offsets, np.int64)
    rep = _c(rep, np.float64)
    bo = _c(blk_offsets, np.int64)
    rows, heads, d = q.shape
    blocks = np.empty((rows, top_blocks), dtype=np.int32)
    idx = np.empty((rows, topk), dtype=np.int32)
    cnt = np.empty(rows, dtype=np.int32)
    coarse = np.zeros(max(1, rep.shape[0]), dtype=np.float64)
    gb = None if given_blocks is None else _c(given_blocks, np.int32)
    _lib().oracle_hisa_topk(rows, heads, d, topk, blk, top_blocks, _p(q, _f64p), _p(w, _f64p), _p(K, _f64p),
                            _p(ko, _i64p), _p(rep, _f64p), _p(bo, _i64p), None if gb is None else _p(gb, _i32p),
                            _p(blocks, _i32p), _p(idx, _i32p), _p(cnt, _i32p), _p(coarse, _f64p))
    return blocks, idx, cnt, coarse[: rep.shape[0]]


def hisa_topk_prefill(q, w, K, rep, topk, blk, top_blocks):
    """Hierarchical top-k for the n causal queries of one sequence: query i sees keys
    0..i, its complete blocks are j < (i + 1) // blk (rep [n // blk, d] from
    hisa_describe(K, [0, n], blk)).  Returns (blocks [n, top_blocks], idx [n, topk],
    count [n]), ascending and -1 padded."""
    q = _c(q, np.float64)
    w = _c(w, np.float64)
    K = _c(K, np.float64)
    rep = _c(rep, np.float64)
    n, heads, d = q.shape
    if rep.shape[0] == 0:
        rep = np.zeros((1, d), dtype=np.float64)
    blocks = np.empty((n, top_blocks), dtype=np.int32)
    idx = np.empty((n, topk), dtype=np.int32)
    cnt = np.empty(n, dtype=np.int32)
    _lib().oracle_hisa_topk_prefill(n, heads, d, topk, blk, top_blocks, _p(q, _f64p), _p(w, _f64p), _p(K, _f64p),
                                    _p(rep, _f64p), _p(blocks, _i32p), _p(idx, _i32p), _p(cnt, _i32p))
    return blocks, idx, cnt


# -------------------------------------------------------------- blocks --
def block_describe(Kblocks, rank, L_eff=None):
    """Kblocks [n_blocks, L, D] -> (mu [nb, D], xi [nb, rank, D], lam [nb, rank])."""
    Kb = _c(Kblocks, np.float64)
    nb, L, D = Kb.shape
    mu = np.empty((nb, D), dtype=np.float64)
    xi = np.empty((nb, rank, D), dtype=np.float64)
    lam = np.empty((nb, rank), dtype=np.float64)
    if L_eff is None:
        lp = None
    else:
        L_eff = _c(L_eff, np.int32)
        lp = _p(L_eff, _i32p)
    _lib().oracle_block_describe(nb, L, D, rank, _p(Kb, _f64p), lp, _p(mu, _f64p),
                                 _p(xi, _f64p), _p(lam, _f64p))
    return mu, xi, lam


def block_log_mass(q, Kb):
    """Exact ln sum_r exp(q . k_r) for one block Kb [L, D]."""
    q = _c(q, np.float64)
    Kb = _c(Kb, np.float64)
    return float(_lib().oracle_block_log_mass(Kb.shape[0], Kb.shape[1], _p(q, _f64p),
                                              _p(Kb, _f64p)))


def block_select(Q, mu, xi, T, L, top_blocks, window, scale=None):
    """Q [n_seq, n_q, D]; mu [n_seq, n_kv, n_full, D]; xi [n_seq, n_kv, n_full, rank, D].
    Returns (tok [n_seq, n_kv, cap], tok_count, blk [n_seq, n_kv, top], blk_score)."""
    Q = _c(Q, np.float64)
    mu = _c(mu, np.float64)
    xi = _c(xi, np.float64)
    n_seq, n_q, D = Q.shape
    n_kv, n_full = mu.shape[1], mu.shape[2]
    rank = xi.shape[3]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    cap = top_blocks * L + window
    tok = np.empty((n_seq, n_kv, cap), dtype=np.int32)
    cnt = np.empty((n_seq, n_kv), dtype=np.int32)
    blk = np.empty((n_seq, n_kv, top_blocks), dtype=np.int32)
    bs = np.empty((n_seq, n_kv, n_full), dtype=np.float64)
    _lib().oracle_block_select(n_seq, n_kv, n_q, D, rank, n_full, L, T, top_blocks, window,
                               float(scale), _p(Q, _f64p), _p(mu, _f64p), _p(xi, _f64p), cap,
                               _p(tok, _i32p), _p(cnt, _i32p), _p(blk, _i32p), _p(bs, _f64p))
    return tok, cnt, blk, bs


def block_describe_ss(Kblocks, U, rank):
    """Subspace descriptors: Kblocks [nb, L, D], U [D, s] -> (mu [nb, D], xi [nb, rank, s],
    lam [nb, rank]) with xi the scaled eigenvectors of U^T Sigma_b U ([P5] Eq.(17))."""
    Kb = _c(Kblocks, np.float64)
    U = _c(U, np.float64)
    nb, L, D = Kb.shape
    sd = U.shape[1]
    mu = np.empty((nb, D), dtype=np.float64)
    xi = np.empty((nb, rank, sd), dtype=np.float64)
    lam = np.empty((nb, rank), dtype=np.float64)
    _lib().oracle_block_describe_ss(nb, L, D, sd, rank, _p(Kb, _f64p), _p(U, _f64p), _p(mu, _f64p),
                                    _p(xi, _f64p), _p(lam, _f64p))
    return mu, xi, lam


def block_select_ss(Q, U, mu, xi, T, L, top_blocks, window, scale=None):
    """block_select with the subspace quadratic term ([P5] Eq.(18)): Q [n_seq, n_q, D],
    U [D, s], mu [n_seq, n_kv, n_full, D], xi [n_seq, n_kv, n_full, rank, s]."""
    Q = _c(Q, np.float64)
    U = _c(U, np.float64)
    mu = _c(mu, np.float64)
    xi = _c(xi, np.float64)
    n_seq, n_q, D = Q.shape
    n_kv, n_full, rank, sd = mu.shape[1], mu.shape[2], xi.shape[3], xi.shape[4]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    cap = top_blocks * L + window
    tok = np.empty((n_seq, n_kv, cap), dtype=np.int32)
    cnt = np.empty((n_seq, n_kv), dtype=np.int32)
    blk = np.empty((n_seq, n_kv, top_blocks), dtype=np.int32)
    bs = np.empty((n_seq, n_kv, n_full), dtype=np.float64)
    _lib().oracle_block_select_ss(n_seq, n_kv, n_q, D, sd, rank, n_full, L, T, top_blocks, window,
                                  float(scale), _p(Q, _f64p), _p(U, _f64p), _p(mu, _f64p), _p(xi, _f64p),
                                  cap, _p(tok, _i32p), _p(cnt, _i32p), _p(blk, _i32p), _p(bs, _f64p))
    return tok, cnt, blk, bs


def quest_describe(K, L):
    """K [n_seq, T, n_kv, D] -> (kmin, kmax) [n_seq, n_kv, T // L, D] ([P5] Eq.(23))."""
    K = _c(K, np.float64)
    n_seq, T, n_kv, D = K.shape
    n_full = T // L
    kmin = np.empty((n_seq, n_kv, n_full, D), dtype=np.float64)
    kmax = np.empty((n_seq, n_kv, n_full, D), dtype=np.float64)
    _lib().oracle_quest_describe(n_seq, T, n_kv, D, L, _p(K, _f64p), _p(kmin, _f64p), _p(kmax, _f64p))
    return kmin, kmax


def quest_select(Q, kmin, kmax, T, L, top_blocks, window, scale=None):
    """Quest box score ([P5] Eq.(24)) under the block_select rule.  Q [n_seq, n_q, D];
    kmin, kmax [n_seq, n_kv, n_full, D].  Returns (tok, tok_count, blk, blk_score)."""
    Q = _c(Q, np.float64)
    kmin = _c(kmin, np.float64)
    kmax = _c(kmax, np.float64)
    n_seq, n_q, D = Q.shape
    n_kv, n_full = kmin.shape[1], kmin.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    cap = top_blocks * L + window
    tok = np.empty((n_seq, n_kv, cap), dtype=np.int32)
    cnt = np.empty((n_seq, n_kv), dtype=np.int32)
    blk = np.empty((n_seq, n_kv, top_blocks), dtype=np.int32)
    bs = np.empty((n_seq, n_kv, n_full), dtype=np.float64)
    _lib().oracle_quest_select(n_seq, n_kv, n_q, D, n_full, L, T, top_blocks, window, float(scale),
                               _p(Q, _f64p), _p(kmin, _f64p), _p(kmax, _f64p), cap, _p(tok, _i32p),
                               _p(cnt, _i32p), _p(blk, _i32p), _p(bs, _f64p))
    return tok, cnt, blk, bs


def fp4_quantize(xi):
    """xi [..., D] float32 -> (codes [..., D/2] uint8, scale [...] float32): E2M1 with one
    fp32 absmax/6 scale per vector ([P5] §5.5; rounding reading in crs_oracle.c)."""
    x = _c(xi, np.float32)
    D = x.shape[-1]
    n = x.size // D
    codes = np.empty(x.shape[:-1] + (D // 2,), dtype=np.uint8)
    scale = np.empty(x.shape[:-1], dtype=np.float32)
    _lib().oracle_fp4_quantize(n, D, _p(x, _f32p), _p(codes, _u8p), _p(scale, _f32p))
    return codes, scale


def fp4_dequantize(codes, scale):
    """Inverse map of fp4_quantize's codes: sign * E2M1 value * scale, fp64."""
    c = _c(codes, np.uint8)
    s = _c(scale, np.float32)
    D = c.shape[-1] * 2
    n = c.size // (D // 2)
    out = np.empty(c.shape[:-1] + (D,), dtype=np.float64)
    _lib().oracle_fp4_dequantize(n, D, _p(c, _u8p), _p(s, _f32p), _p(out, _f64p))
    return out


# ---------------------------------------------------------- attention --
def sparse_attn(Q, K, V, I, kv_base=None, scale=None, key_valid=None, q_pos=None):
    """Q [rows, n_q, D]; K, V [tokens, n_kv, D]; I [rows, n_lists, max_idx]
    (n_lists = n_kv or 1); kv_base [rows] token offset of each row's sequence;
    key_valid [tokens] (non-zero = the key may be attended; None = all) and
    q_pos [rows] (entry j of row t is used only if j <= q_pos[t]; None = no
    causal limit).  Returns (O [rows, n_q, D], lse [rows, n_q])."""
    Q = _c(Q, np.float64)
    K = _c(K, np.float64)
    V = _c(V, np.float64)
    I = _c(I, np.int32)
    rows, n_q, D = Q.shape
    n_kv = K.shape[1]
    if I.ndim == 2:
        I = I[:, None, :].copy()
    n_lists, max_idx = I.shape[1], I.shape[2]
    if kv_base is None:
        kv_base = np.zeros(rows, dtype=np.int64)
    kb = _c(kv_base, np.int64)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    kv = None if key_valid is None else _c(np.asarray(key_valid) != 0, np.uint8)
    qp = None if q_pos is None else _c(q_pos, np.int32)
    O = np.empty((rows, n_q, D), dtype=np.float64)
    lse = np.empty((rows, n_q), dtype=np.float64)
    _lib().oracle_sparse_attn(rows, n_q, n_kv, D, float(scale), _p(Q, _f64p), _p(K, _f64p),
                              _p(V, _f64p), _p(kb, _i64p), _p(I, _i32p), n_lists, max_idx,
                              None if kv is None else _p(kv, _u8p),
                              None if qp is None else _p(qp, _i32p),
                              _p(O, _f64p), _p(lse, _f64p))
    return O, lse
