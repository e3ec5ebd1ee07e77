"""Pins for the indexer part of the oracle (score, token top-k).

Structured inputs make the right top-k known by construction; invariants from
PaperTrace 2.2 "细粒度索引" (|S_t| = min(k, t+1); the streaming 2k -> k merge
equals the global top-k; the cutoff margin) hold for any input.
"""
import numpy as np
import pytest

import oracle


def test_single_head_known_order():
    """One head, w = 1, keys k_s = a_s u, query u: score = ReLU(a_s)|u|^2, so the
    top-k is the k largest a_s; non-positive a_s score exactly 0 and tie by index."""
    rng = np.random.default_rng(0)
    d, n, k = 8, 50, 12
    u = rng.standard_normal(d)
    a = rng.permutation(np.concatenate([np.linspace(0.5, 3.0, 20), -np.linspace(0.1, 2.0, 30)]))
    K = a[:, None] * u[None, :]
    idx, cnt, cut, nxt = oracle.indexer_topk(u[None, None, :], np.ones((1, 1)), K,
                                             np.zeros(1, np.int64), np.array([n], np.int32), k)
    want = np.sort(np.argsort(-a, kind="stable")[:k])
    assert cnt[0] == k and (idx[0] == want).all()
    # budget beyond the positive keys: the zeros come in index order
    k2 = 26
    idx2, cnt2, _, _ = oracle.indexer_topk(u[None, None, :], np.ones((1, 1)), K,
                                           np.zeros(1, np.int64), np.array([n], np.int32), k2)
    pos = np.flatnonzero(a > 0)
    zeros = np.flatnonzero(a <= 0)[: k2 - len(pos)]
    assert (idx2[0] == np.sort(np.concatenate([pos, zeros]))).all()


def test_negative_weight_prefers_relu_zeros():
    """w = -1: score = -ReLU(q.k) <= 0; the maxima are the clipped keys (score 0),
    taken smallest index first."""
    rng = np.random.default_rng(1)
    d, n, k = 4, 30, 5
    q = rng.standard_normal(d)
    K = rng.standard_normal((n, d))
    idx, cnt, cut, _ = oracle.indexer_topk(q[None, None], -np.ones((1, 1)), K,
                                           np.zeros(1, np.int64), np.array([n], np.int32), k)
    clipped = np.flatnonzero(K @ q <= 0)
    assert len(clipped) >= k
    assert (idx[0] == clipped[:k]).all() and cut[0] == 0.0


def test_head_weights_combine_disjoint_supports():
    """Heads reading disjoint coordinates: head h sees only coordinate h, so the
    score of a key with coordinates c is sum_h w_h max(c_h, 0)."""
    rng = np.random.default_rng(2)
    H, n, k = 3, 40, 7
    q = np.eye(H)                       # head h projects onto coordinate h
    w = np.array([2.0, -1.0, 0.5])
    K = rng.standard_normal((n, H))
    idx, cnt, cut, nxt = oracle.indexer_topk(q[None], w[None], K, np.zeros(1, np.int64),
                                             np.array([n], np.int32), k)
    s = sum(w[h] * np.maximum(K[:, h], 0) for h in range(H))
    order = np.lexsort((np.arange(n), -s))
    assert (idx[0] == np.sort(order[:k])).all()
    assert cut[0] == pytest.approx(s[order[k - 1]]) and nxt[0] == pytest.approx(s[order[k]])


def test_causal_prefix_counts_and_invalid_slots():
    """|S_t| = min(k, t+1), the rest -1 (PaperTrace 2.2 §2.1)."""
    rng = np.random.default_rng(3)
    n, H, d, k = 40, 2, 6, 16
    q = rng.standard_normal((n, H, d))
    w = rng.standard_normal((n, H))
    K = rng.standard_normal((n, d))
    t = np.arange(n)
    idx, cnt, _, _ = oracle.indexer_topk(q, w, K, np.zeros(n, np.int64),
                                         (t + 1).astype(np.int32), k)
    assert (cnt == np.minimum(k, t + 1)).all()
    for r in range(n):
        sel = idx[r, : cnt[r]]
        assert (idx[r, cnt[r]:] == -1).all()
        assert (np.diff(sel) > 0).all() and sel.max() <= r
        if r + 1 <= k:
            assert (sel == np.arange(r + 1)).all()


def test_streaming_merge_equals_global_topk():
    """Per-tile top-k then a 2k -> k merge gives the global top-k (PaperTrace 2.2 §2.1)."""
    rng = np.random.default_rng(4)
    H, d, n, k, tile = 4, 16, 300, 20, 64
    q = rng.standard_normal((1, H, d))
    w = rng.standard_normal((1, H))
    K = rng.standard_normal((n, d))
    K[50] = K[10]                       # an exact tie across tiles
    gidx, _, _, _ = oracle.indexer_topk(q, w, K, np.zeros(1, np.int64), np.array([n], np.int32), k)
    keep = np.zeros(0, np.int64)
    for t0 in range(0, n, tile):
        t1 = min(n, t0 + tile)
        li, lc, _, _ = oracle.indexer_topk(q, w, K[t0:t1], np.zeros(1, np.int64),
                                           np.array([t1 - t0], np.int32), k)
        cand = np.concatenate([keep, t0 + li[0, : lc[0]]])
        mi, mc, _, _ = oracle.indexer_topk(q, w, K[cand], np.zeros(1, np.int64),
                                           np.array([len(cand)], np.int32), k)
        keep = np.sort(cand[mi[0, : mc[0]]])
    assert (keep == gidx[0]).all()


def test_cutoff_margin_invariance():
    """Scores perturbed by less than delta_k / 2 keep the same set (PaperTrace 2.2 §3.1 Eq.(9))."""
    rng = np.random.default_rng(5)
    H, d, n, k = 2, 8, 200, 30
    q = rng.standard_normal((1, H, d))
    w = np.abs(rng.standard_normal((1, H)))
    K = rng.standard_normal((n, d))
    idx, _, cut, nxt = oracle.indexer_topk(q, w, K, np.zeros(1, np.int64), np.array([n], np.int32), k)
    s = oracle.indexer_score(q[0], w[0], K)
    sel = set(idx[0].tolist())
    assert min(s[list(sel)]) >= max(np.delete(s, list(sel)))
    delta = cut[0] - nxt[0]
    assert delta > 0
    # scaling every score by a positive factor is a perturbation that keeps the order
    idx2, _, _, _ = oracle.indexer_topk(q, 3.0 * w, K, np.zeros(1, np.int64), np.array([n], np.int32), k)
    assert (idx2 == idx).all()


def test_ragged_sequences_use_key_base():
    rng = np.random.default_rng(6)
    lens = [5, 33, 17]
    d, H, k = 8, 4, 10
    K = rng.standard_normal((sum(lens), d))
    base = np.cumsum([0] + lens[:-1]).astype(np.int64)
    q = rng.standard_normal((3, H, d))
    w = rng.standard_normal((3, H))
    idx, cnt, _, _ = oracle.indexer_topk(q, w, K, base, np.array(lens, np.int32), k)
    for r in range(3):
        li, lc, _, _ = oracle.indexer_topk(q[r:r + 1], w[r:r + 1], K[base[r]: base[r] + lens[r]],
                                           np.zeros(1, np.int64), np.array([lens[r]], np.int32), k)
        assert cnt[r] == lc[0] and (idx[r] == li[0]).all()
