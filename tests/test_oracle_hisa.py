"""Pins for the hierarchical indexer (HISA) of the oracle ("细粒度索引" page: the
three cost-cutting directions, §2.2 Eq.(7), the HISA cost C = O(B d_c + k_b b d_r)).
Checks: a hand-worked representative, equality with the flat indexer when every block
is kept, the final set inside the coarse candidates (Eq.(7) rests on S within C), a
planted block, tie order, and the open block that has no representative."""
import numpy as np

import oracle


def _row(rng, ctx, heads=4, d=8):
    K = rng.standard_normal((ctx, d))
    q = rng.standard_normal((1, heads, d))
    w = np.abs(rng.standard_normal((1, heads)))
    return K, q, w, np.array([0, ctx], dtype=np.int64)


def test_representatives_hand_example():
    K = np.array([[1.0, 2.0], [3.0, 4.0], [5.0, 6.0], [7.0, 8.0], [9.0, 10.0]])
    rep, bo = oracle.hisa_describe(K, np.array([0, 5]), 2)
    assert list(bo) == [0, 2]                                  # the fifth key is the open block
    assert np.array_equal(rep, [[2.0, 3.0], [6.0, 7.0]])


def test_keeping_every_block_is_the_flat_indexer():
    rng = np.random.default_rng(21)
    K, q, w, ko = _row(rng, 8 * 12 + 5)
    rep, bo = oracle.hisa_describe(K, ko, 8)
    _, idx, cnt, _ = oracle.hisa_topk(q, w, K, ko, rep, bo, topk=20, blk=8, top_blocks=12)
    f_idx, f_cnt, _, _ = oracle.indexer_topk(q, w, K, np.array([0]), np.array([K.shape[0]], dtype=np.int32), 20)
    assert cnt[0] == f_cnt[0] == 20
    assert np.array_equal(idx, f_idx)


def test_final_set_lies_in_the_coarse_candidates():
    rng = np.random.default_rng(22)
    K, q, w, ko = _row(rng, 16 * 40 + 9)
    rep, bo = oracle.hisa_describe(K, ko, 16)
    blocks, idx, cnt, _ = oracle.hisa_topk(q, w, K, ko, rep, bo, topk=32, blk=16, top_blocks=5)
    cand = set(int(p) for b in blocks[0] if b >= 0 for p in range(b * 16, b * 16 + 16))
    cand |= set(range(16 * 40, 16 * 40 + 9))
    sel = set(int(p) for p in idx[0, : cnt[0]])
    assert cnt[0] == 32 and sel <= cand
    # Eq.(7) then holds exactly for any teacher set G (here the flat top-32)
    f_idx, f_cnt, _, _ = oracle.indexer_topk(q, w, K, np.array([0]), np.array([K.shape[0]], dtype=np.int32), 32)
    G = set(int(p) for p in f_idx[0, : f_cnt[0]])
    r_total = len(sel & G) / len(G)
    r_coarse = len(cand & G) / len(G)
    r_fine = len(sel & cand & G) / max(1, len(cand & G))
    assert abs(r_total - r_coarse * r_fine) < 1e-12


def test_planted_block_and_ties():
    d, blk = 4, 4
    K = np.full((blk * 6, d), 0.01)
    K[3 * blk: 4 * blk] = 1.0                 # block 3 aligned with q
    K[1 * blk: 2 * blk] = K[5 * blk: 6 * blk] = 0.5   # blocks 1 and 5 tie for second
    q = np.ones((1, 1, d))
    w = np.ones((1, 1))
    ko = np.array([0, K.shape[0]])
    rep, bo = oracle.hisa_describe(K, ko, blk)
    blocks, idx, cnt, coarse = oracle.hisa_topk(q, w, K, ko, rep, bo, topk=4, blk=blk, top_blocks=2)
    assert list(blocks[0]) == [1, 3]
    assert list(idx[0, : cnt[0]]) == [12, 13, 14, 15]
    np.testing.assert_allclose(coarse, [0.04, 2.0, 0.04, 4.0, 0.04, 2.0])


def test_open_block_is_always_searched():
    rng = np.random.default_rng(23)
    d, blk, nb = 8, 8, 10
    K = 0.01 * rng.standard_normal((nb * blk + 3, d))
    q = np.ones((1, 1, d))
    w = np.ones((1, 1))
    K[nb * blk + 1] = 5.0                     # the best key sits in the open block
    ko = np.array([0, K.shape[0]])
    rep, bo = oracle.hisa_describe(K, ko, blk)
    _, idx, cnt, _ = oracle.hisa_topk(q, w, K, ko, rep, bo, topk=1, blk=blk, top_blocks=1)
    assert cnt[0] == 1 and idx[0, 0] == nb * blk + 1
