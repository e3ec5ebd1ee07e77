"""Pins for the prefill (causal) form of the hierarchical indexer in the oracle ("细粒度索引"
page, §2.2 Eq.(7) and the three cost-cutting directions; the flat indexer's prefill rows
see keys 0..i, §2.1 Eq.(4)).  Query i keeps the top blocks among the sequence's complete
blocks j < (i + 1) / b and runs the token indexer on their keys and on its open block.
Checks: equality with the flat prefill indexer when every block is kept, a pure-Python
brute force on a tiny sequence, causality, equality with the decode form on each prefix,
tie order, and rows that have no complete block yet."""
import numpy as np

import oracle


def _seq(rng, n, heads=3, d=8):
    K = rng.standard_normal((n, d))
    q = rng.standard_normal((n, heads, d))
    w = np.abs(rng.standard_normal((n, heads)))
    return q, w, K


def _score(q, w, k):
    """sum_h w_h ReLU(q_h . k) for one query and one key, written out."""
    s = 0.0
    for h in range(q.shape[0]):
        s += w[h] * max(0.0, float(np.dot(q[h], k)))
    return s


def test_keeping_every_block_is_the_flat_prefill_indexer():
    rng = np.random.default_rng(31)
    n, blk, topk = 8 * 9 + 3, 8, 12
    q, w, K = _seq(rng, n)
    rep, _ = oracle.hisa_describe(K, np.array([0, n]), blk)
    _, idx, cnt = oracle.hisa_topk_prefill(q, w, K, rep, topk, blk, top_blocks=n // blk)
    f_idx, f_cnt, _, _ = oracle.indexer_topk(q, w, K, np.zeros(n, np.int64), np.arange(1, n + 1, dtype=np.int32),
                                             topk)
    assert np.array_equal(cnt, f_cnt)
    assert np.array_equal(idx, f_idx)


def test_brute_force_tiny_sequence():
    rng = np.random.default_rng(32)
    n, blk, top_blocks, topk = 37, 4, 3, 5
    q, w, K = _seq(rng, n, heads=2, d=4)
    rep, _ = oracle.hisa_describe(K, np.array([0, n]), blk)
    blocks, idx, cnt = oracle.hisa_topk_prefill(q, w, K, rep, topk, blk, top_blocks)
    means = [K[j * blk:(j + 1) * blk].mean(axis=0) for j in range(n // blk)]
    for i in range(n):
        nb = (i + 1) // blk
        coarse = sorted(range(nb), key=lambda j: (-_score(q[i], w[i], means[j]), j))
        kept = sorted(coarse[:top_blocks])
        exp_blocks = kept + [-1] * (top_blocks - len(kept))
        cand = [p for b in kept for p in range(b * blk, b * blk + blk)] + list(range(nb * blk, i + 1))
        fine = sorted(cand, key=lambda p: (-_score(q[i], w[i], K[p]), p))
        sel = sorted(fine[:topk])
        assert list(blocks[i]) == exp_blocks, i
        assert list(idx[i]) == sel + [-1] * (topk - len(sel)), i
        assert cnt[i] == len(sel)


def test_rows_do_not_see_later_keys():
    rng = np.random.default_rng(33)
    n, blk = 64, 8
    q, w, K = _seq(rng, n)
    rep, _ = oracle.hisa_describe(K, np.array([0, n]), blk)
    b0, i0, c0 = oracle.hisa_topk_prefill(q, w, K, rep, 6, blk, 2)
    cut = 29
    K2 = K.copy()
    K2[cut + 1:] = rng.standard_normal(K2[cut + 1:].shape) * 5.0
    rep2, _ = oracle.hisa_describe(K2, np.array([0, n]), blk)
    b1, i1, c1 = oracle.hisa_topk_prefill(q, w, K2, rep2, 6, blk, 2)
    assert np.array_equal(b0[:cut + 1], b1[:cut + 1])
    assert np.array_equal(i0[:cut + 1], i1[:cut + 1])
    assert np.array_equal(c0[:cut + 1], c1[:cut + 1])


def test_each_row_equals_the_decode_form_on_its_prefix():
    rng = np.random.default_rng(34)
    n, blk, top_blocks, topk = 50, 6, 3, 7
    q, w, K = _seq(rng, n)
    rep, _ = oracle.hisa_describe(K, np.array([0, n]), blk)
    blocks, idx, cnt = oracle.hisa_topk_prefill(q, w, K, rep, topk, blk, top_blocks)
    for i in range(n):
        ko = np.array([0, i + 1], dtype=np.int64)
        rep_i, bo_i = oracle.hisa_describe(K[: i + 1], ko, blk)
        db, di, dc, _ = oracle.hisa_topk(q[i:i + 1], w[i:i + 1], K[: i + 1], ko, rep_i, bo_i, topk, blk, top_blocks)
        assert np.array_equal(db[0], blocks[i]) and np.array_equal(di[0], idx[i]) and dc[0] == cnt[i], i


def test_ties_and_rows_without_a_complete_block():
    n, blk = 20, 4
    K = np.ones((n, 4))                       # every key and every block mean equal
    q = np.ones((n, 2, 4))
    w = np.ones((n, 2))
    rep, _ = oracle.hisa_describe(K, np.array([0, n]), blk)
    blocks, idx, cnt = oracle.hisa_topk_prefill(q, w, K, rep, 3, blk, 2)
    for i in range(n):
        nb = (i + 1) // blk
        kept = list(range(min(nb, 2)))        # equal coarse scores: the smaller blocks
        assert list(blocks[i]) == kept + [-1] * (2 - len(kept)), i
        cand = [p for b in kept for p in range(b * blk, b * blk + blk)] + list(range(nb * blk, i + 1))
        sel = sorted(cand)[:3]                # equal token scores: the smaller positions
        assert list(idx[i]) == sel + [-1] * (3 - len(sel)), i
    assert cnt[0] == 1 and list(idx[0]) == [0, -1, -1]    # query 0: only itself, no block
