"""Pins for the LSH part of the oracle (hash, sort, candidate sets, attention).

Each check ties the oracle to something other than itself: a printed worked
example, a library sort, a brute-force enumeration of the definition, or a
degenerate case that reduces to plain (windowed) causal attention computed by
torch's SDPA.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import golden


def _x_example():
    g = golden("p1_lsh_2d_example.json")
    X = np.array(g["x"], dtype=np.float32)[None, None]
    R = np.array(g["R"], dtype=np.float32)[None, None]
    return g, X, R


def test_p1_2d_example_buckets_sort_sizes():
    g, X, R = _x_example()
    pr = g["printed"]
    b = oracle.lsh_hash(X, R, n_buckets=4)[0, 0, 0]
    assert list(b + 1) == pr["bucket_ids_1based"]
    perm, inv = oracle.lsh_sort(b[None])
    assert list(perm[0] + 1) == pr["sort_order_1based"]
    sizes = [int((b == k).sum()) for k in sorted(set(b.tolist()))]
    assert sizes == pr["bucket_sizes"]
    for key in ("x3_variant_a", "x3_variant_b"):
        v = pr[key]
        X2 = X.copy()
        X2[0, 0, 2] = np.array(v["x3"], dtype=np.float32)
        assert oracle.lsh_hash(X2, R, 4)[0, 0, 0, 2] + 1 == v["bucket_1based"]


def test_p1_2d_example_scores_mass_output():
    g, X, R = _x_example()
    pr = g["printed"]
    x = np.array(g["x"], dtype=np.float64)   # the attention pin runs on the exact decimals
    V = np.zeros_like(x)
    V[0] = pr["values_v1_v2"][0]
    V[1] = pr["values_v1_v2"][1]
    bucket = oracle.lsh_hash(X, R, 4)
    perm, inv = oracle.lsh_sort(bucket)
    # raw dot products, no sqrt(d) scaling, self allowed, no causal mask (as on the page)
    O, lse, cnt = oracle.lsh_attn(x[None, None], V[None, None], bucket, perm, inv,
                                  np.array([4], np.int32), chunk=4, causal=0, no_self=0,
                                  key_norm=0, scale=1.0, rows=np.array([1], np.int32))
    assert cnt[0, 0, 0] == 2
    # the four printed scores with q = x2, through the oracle's dense attention route
    I_all = np.arange(4, dtype=np.int32)[None, None, :]
    Od, lse_d = oracle.sparse_attn(x[1][None, None], x[:, None], V[:, None], I_all, scale=1.0)
    assert math.exp(lse_d[0, 0]) == pytest.approx(pr["exp_sum_all_four"], abs=5e-3)
    dropped = 1.0 - math.exp(lse[0, 0, 0] - lse_d[0, 0])
    assert 100 * dropped == pytest.approx(pr["dropped_mass_percent"], abs=0.05)
    for j, s in enumerate(pr["scores_q_dot_x"]):
        _, l1 = oracle.sparse_attn(x[1][None, None], x[:, None], V[:, None],
                                   np.array([[[j]]], np.int32), scale=1.0)
        assert l1[0, 0] == pytest.approx(s, abs=1e-12)
    assert O[0, 0, 0] == pytest.approx(g["derived"]["output_q_x2_over_bucket"], abs=1e-3)


def test_sort_equals_library_stable_sort():
    rng = np.random.default_rng(5)
    b = rng.integers(0, 13, size=(3, 257)).astype(np.int32)
    perm, inv = oracle.lsh_sort(b)
    for s in range(3):
        ref = np.argsort(b[s], kind="stable")
        assert (perm[s] == ref).all()
        assert (perm[s][inv[s]] == np.arange(257)).all()
        assert (inv[s][perm[s]] == np.arange(257)).all()


def test_hash_argmax_ties_lowest_index_and_zero_rotation():
    X = np.ones((1, 1, 5, 8), np.float32)
    R = np.zeros((1, 2, 8, 3), np.float32)           # u = 0: every entry of [u; -u] ties
    assert (oracle.lsh_hash(X, R, 6) == 0).all()


def test_hash_matches_fp64_argmax_away_from_ties():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((1, 2, 300, 64)).astype(np.float32)
    R = rng.standard_normal((2, 3, 64, 16)).astype(np.float32)
    b = oracle.lsh_hash(X, R, 32)
    u = np.einsum("bhnd,hrdk->bhrnk", X.astype(np.float64), R.astype(np.float64))
    ref = np.concatenate([u, -u], axis=-1).argmax(-1)
    margin = oracle.lsh_margin(X, R, 32)
    ok = margin > 1e-4
    assert ok.mean() > 0.99
    assert (b[ok] == ref[ok]).all()


def _brute_candidates(bucket, inv, i, m, causal, no_self, valid_len):
    """U(i) enumerated pair by pair from the definition (P1 §2.1-2.2, Eq.(2))."""
    rounds, n = bucket.shape
    out = set()
    for r in range(rounds):
        ci = inv[r, i] // m
        for j in range(n):
            cj = inv[r, j] // m
            if cj not in (ci, ci - 1):
                continue
            if bucket[r, j] != bucket[r, i]:
                continue
            if causal and j > i:
                continue
            if no_self and j == i:
                continue
            if j >= valid_len:
                continue
            out.add(j)
    return sorted(out)


@pytest.mark.parametrize("causal,no_self", [(1, 1), (1, 0), (0, 0)])
def test_candidates_bruteforce(causal, no_self):
    rng = np.random.default_rng(7)
    rounds, n, m, nb = 3, 45, 8, 4
    bucket = rng.integers(0, nb, size=(rounds, n)).astype(np.int32)
    perm, inv = oracle.lsh_sort(bucket)
    vl = 41
    for i in range(n):
        got = oracle.lsh_candidates(bucket, perm, inv, i, m, causal, no_self, vl)
        assert got.tolist() == _brute_candidates(bucket, inv, i, m, causal, no_self, vl)


def test_candidates_invariants():
    rng = np.random.default_rng(11)
    n, m, nb = 200, 16, 8
    bucket = rng.integers(0, nb, size=(1, n)).astype(np.int32)
    perm, inv = oracle.lsh_sort(bucket)
    assert np.bincount(bucket[0], minlength=nb).sum() == n
    # cost identity C = n/m: every slot belongs to exactly one of ceil(n/m) chunks
    assert len(set((inv[0] // m).tolist())) == math.ceil(n / m)
    for i in range(n):
        c = oracle.lsh_candidates(bucket, perm, inv, i, m, 0, 0, n)
        assert len(c) <= 2 * m
        assert i in c.tolist()  # self is always a legal edge without masks


def test_causal_uses_original_position_leak_example():
    """P1 §"8.2 排序键必须保持因果信息": positions [0,1,2,3] stored in the order
    [2,0,3,1]; a mask on sorted slots would let position 0 see position 2."""
    perm = np.array([[2, 0, 3, 1]], np.int32)
    inv = np.empty_like(perm)
    inv[0, perm[0]] = np.arange(4)
    bucket = np.zeros((1, 4), np.int32)
    got = {i: oracle.lsh_candidates(bucket, perm, inv, i, 4, 1, 0, 4).tolist() for i in range(4)}
    assert got == {0: [0], 1: [0, 1], 2: [0, 1, 2], 3: [0, 1, 2, 3]}


def test_p4_causal_pair_count():
    g = golden("p4_counts.json")["printed"]
    bucket = np.zeros((1, 6), np.int32)
    perm, inv = oracle.lsh_sort(bucket)
    total = sum(len(oracle.lsh_candidates(bucket, perm, inv, i, 6, 1, 0, 6)) for i in range(6))
    assert total == g["causal_pairs_n6_with_self"]


def _sdpa(q, k, v, mask):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        attn_mask=torch.from_numpy(mask)).numpy()


def test_degenerate_one_bucket_one_chunk_is_dense_causal_no_self():
    """P1 "最小正确性测试": candidates = everything -> dense (causal, no-self)."""
    rng = np.random.default_rng(3)
    n, d = 70, 16
    q = rng.standard_normal((1, 1, n, d))
    v = rng.standard_normal((1, 1, n, d))
    R = np.zeros((1, 1, d, 2), np.float32)  # all in bucket 0
    b = oracle.lsh_hash(q.astype(np.float32), R, 2)
    perm, inv = oracle.lsh_sort(b)
    O, lse, cnt = oracle.lsh_attn(q, v, b, perm, inv, np.array([n], np.int32), chunk=n,
                                  causal=1, no_self=1, key_norm=1)
    k = q / np.linalg.norm(q, axis=-1, keepdims=True)
    mask = np.tril(np.ones((n, n), bool), -1)
    ref = _sdpa(q[0, 0, 1:][None], k[0, 0][None], v[0, 0][None], mask[1:][None])[0]
    assert np.abs(O[0, 0, 1:] - ref).max() < 1e-12
    assert (O[0, 0, 0] == 0).all() and lse[0, 0, 0] == -np.inf   # no legal key


def test_degenerate_position_sort_is_chunk_window():
    """P1 "最小正确性测试": a position-only sort turns chunk+previous into a window."""
    rng = np.random.default_rng(4)
    n, d, m = 64, 8, 8
    q = rng.standard_normal((1, 1, n, d))
    v = rng.standard_normal((1, 1, n, d))
    b = np.zeros((1, 1, 1, n), np.int32)
    perm, inv = oracle.lsh_sort(b)
    O, _, _ = oracle.lsh_attn(q, v, b, perm, inv, np.array([n], np.int32), chunk=m,
                              causal=1, no_self=0, key_norm=0)
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    mask = (j <= i) & (j >= (i // m - 1) * m)
    ref = _sdpa(q[0], q[0], v[0], mask[None])
    assert np.abs(O[0, 0] - ref[0]).max() < 1e-12


def test_multi_round_union_equals_attention_over_union():
    """The oracle's LSH attention equals its plain attention over U(i) with
    normalised keys (two independent code paths for the softmax)."""
    rng = np.random.default_rng(9)
    B, H, n, d, rounds, m, nb = 1, 2, 96, 8, 3, 8, 4
    q = rng.standard_normal((B, H, n, d)).astype(np.float32)
    v = rng.standard_normal((B, H, n, d))
    R = rng.standard_normal((H, rounds, d, nb // 2)).astype(np.float32)
    b = oracle.lsh_hash(q, R, nb)
    perm, inv = oracle.lsh_sort(b)
    vl = 90
    O, lse, cnt = oracle.lsh_attn(q, v, b, perm, inv, np.array([vl], np.int32), chunk=m,
                                  causal=1, no_self=1)
    qd = q.astype(np.float64)
    k = qd / np.linalg.norm(qd, axis=-1, keepdims=True)
    for h in range(H):
        for i in range(n):
            if i >= vl:
                assert (O[0, h, i] == 0).all()
                continue
            U = oracle.lsh_candidates(b[0, h], perm[0, h], inv[0, h], i, m, 1, 1, vl)
            assert cnt[0, h, i] == len(U)
            if len(U) == 0:
                assert lse[0, h, i] == -np.inf
                continue
            Oi, li = oracle.sparse_attn(qd[0, h, i][None, None], k[0, h][:, None],
                                        v[0, h][:, None], U[None, None, :])
            assert np.abs(O[0, h, i] - Oi[0, 0]).max() < 1e-12
            assert abs(lse[0, h, i] - li[0, 0]) < 1e-12
