"""Pins for the Quest and mean-pool selectors of the oracle ("COBS 阅读笔记", Quest
section, Eq.(23)-(24) and Table 1).  Each check comes from outside the oracle's own
formula: a hand-worked box, the box maximum found by brute force over its corners,
the bound the box places on every key inside it, and linearity of the mean."""
import itertools

import numpy as np
import pytest

import oracle


def _head_scores(bs, G=1):
    # with one query head per KV head the block score is softmax_b(s_b): log-differences
    # recover s_b - s_0
    lb = np.log(bs)
    return lb - lb[..., :1]


def test_quest_describe_hand_example():
    # one sequence, two blocks of L = 2 keys, D = 2 (values worked by hand)
    K = np.array([[1.0, -2.0], [3.0, 0.0], [-1.0, 5.0], [-4.0, 2.0]]).reshape(1, 4, 1, 2)
    kmin, kmax = oracle.quest_describe(K, 2)
    assert np.array_equal(kmin[0, 0], [[1.0, -2.0], [-4.0, 2.0]])
    assert np.array_equal(kmax[0, 0], [[3.0, 0.0], [-1.0, 5.0]])


def test_quest_score_is_the_box_maximum():
    """Eq.(24) equals the largest q . k over the 2^D corners of the box (brute force)."""
    rng = np.random.default_rng(3)
    D, n_full, L = 4, 7, 2
    a = rng.standard_normal((1, 1, n_full, D))
    b = rng.standard_normal((1, 1, n_full, D))
    kmin, kmax = np.minimum(a, b), np.maximum(a, b)
    q = rng.standard_normal((1, 1, D))
    _, _, _, bs = oracle.quest_select(q, kmin, kmax, n_full * L, L, 2, 0, scale=1.0)
    brute = np.empty(n_full)
    for blk in range(n_full):
        best = -np.inf
        for pick in itertools.product((0, 1), repeat=D):
            corner = np.where(np.array(pick) == 1, kmax[0, 0, blk], kmin[0, 0, blk])
            best = max(best, float(q[0, 0] @ corner))
        brute[blk] = best
    np.testing.assert_allclose(_head_scores(bs[0, 0]), brute - brute[0], rtol=0, atol=1e-12)


def test_quest_box_bounds_every_key():
    """The box of a block contains its keys, so its score is >= q . k for each of them, and
    equal to the best key when one key is the largest in every coordinate."""
    rng = np.random.default_rng(4)
    n_full, L, D = 6, 4, 8
    K = rng.standard_normal((1, n_full * L, 1, D))
    K[0, 2 * L + 1, 0] = np.abs(K[0, 2 * L: 3 * L, 0]).max(axis=0) + 1.0   # dominating key, block 2
    q = np.abs(rng.standard_normal((1, 1, D)))                               # q >= 0
    kmin, kmax = oracle.quest_describe(K, L)
    _, _, _, bs = oracle.quest_select(q, kmin, kmax, n_full * L, L, 3, 0, scale=1.0)
    s = _head_scores(bs[0, 0])
    keys = K[0, :, 0].reshape(n_full, L, D)
    best_key = (keys @ q[0, 0]).max(axis=1)
    # s_b - s_0 >= (best key of b) - s_0 ... compare through block 2, where the bound is tight
    s2_abs = float(q[0, 0] @ kmax[0, 0, 2])            # q >= 0: the box maximum is q . kmax
    assert abs(best_key[2] - s2_abs) < 1e-12
    s_abs = s + (s2_abs - s[2])
    assert np.all(s_abs >= best_key - 1e-12)


def test_meanpool_is_the_average_key_score():
    """Rank 0 is the mean-pool selector: q . kbar_b, which by linearity is the average of
    q . k_r over the block's keys."""
    rng = np.random.default_rng(5)
    n_full, L, D = 9, 4, 16
    keys = rng.standard_normal((n_full, L, D))
    mu = keys.mean(axis=1).reshape(1, 1, n_full, D)
    xi = np.zeros((1, 1, n_full, 0, D))
    q = rng.standard_normal((1, 1, D))
    _, _, _, bs = oracle.block_select(q, mu, xi, n_full * L, L, 2, 0, scale=1.0)
    avg = (keys @ q[0, 0]).mean(axis=1)
    np.testing.assert_allclose(_head_scores(bs[0, 0]), avg - avg[0], rtol=0, atol=1e-12)


def test_quest_selects_the_aligned_block_and_breaks_ties_by_block():
    """A block stretched along q wins; two identical boxes tie and the smaller block is kept."""
    n_full, L, D, T = 8, 4, 4, 32
    kmin = np.zeros((1, 1, n_full, D))
    kmax = np.full((1, 1, n_full, D), 0.1)
    kmax[0, 0, 5] = 2.0                        # aligned with q = (1, 1, 1, 1)
    kmax[0, 0, 1] = kmax[0, 0, 6] = 1.0        # tie for the second place
    q = np.ones((1, 1, D))
    tok, cnt, blk, _ = oracle.quest_select(q, kmin, kmax, T, L, 2, 0, scale=1.0)
    assert list(blk[0, 0]) == [1, 5]
    assert list(tok[0, 0, : cnt[0, 0]]) == list(range(4, 8)) + list(range(20, 24))
