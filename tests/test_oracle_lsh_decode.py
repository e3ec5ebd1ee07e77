"""Pins for the LSH decode step of the oracle (PaperTrace 2.1.1 §5.2: fixed hash, bucket
lists appended per new key, the new query reads its buckets' lists).  Checks: the page's
two-dimensional worked example, agreement with the prefill oracle when one chunk spans
the sequence (the same neighbourhood by another route), the single-bucket case, where
the step is dense causal attention, a brute force of the union over rounds on rows of
different lengths, and the empty set of a first token without itself."""
import math

import numpy as np

import oracle
from conftest import golden


def test_worked_example_query_x2():
    g = golden("p1_lsh_2d_example.json")
    x = np.array(g["x"])[:2].reshape(1, 1, 2, 2)             # history x1, then the new token x2
    v = np.array(g["printed"]["values_v1_v2"]).reshape(1, 1, 2, 2)
    R = np.array(g["R"], dtype=np.float32).reshape(1, 1, 2, 2)
    O, lse, cnt = oracle.lsh_decode(x, v, R, 4, np.array([2]), no_self=False, key_norm=False, scale=1.0)
    assert cnt[0, 0] == 2
    np.testing.assert_allclose(O[0, 0], g["derived"]["output_q_x2_over_bucket"], atol=5e-5)
    s = g["printed"]["scores_q_dot_x"]
    assert abs(lse[0, 0] - math.log(math.exp(s[0]) + math.exp(s[1]))) < 1e-12


def test_matches_prefill_oracle_over_one_chunk():
    rng = np.random.default_rng(41)
    H, n, d, b, rounds = 2, 40, 8, 8, 3
    X = rng.standard_normal((1, H, n, d)).astype(np.float32)
    V = rng.standard_normal((1, H, n, d))
    R = rng.standard_normal((H, rounds, d, b // 2)).astype(np.float32)
    for no_self in (True, False):
        O, lse, cnt = oracle.lsh_decode(X, V, R, b, np.array([n]), no_self=no_self)
        bucket = oracle.lsh_hash(X, R, b)
        perm, inv = oracle.lsh_sort(bucket)
        Op, lsep, cntp = oracle.lsh_attn(X.astype(np.float64), V, bucket, perm, inv, np.array([n], dtype=np.int32),
                                         chunk=n, causal=1, no_self=int(no_self), key_norm=1, rows=np.array([n - 1]))
        assert np.array_equal(cnt[0], cntp[0, :, 0])
        np.testing.assert_allclose(O[0], Op[0, :, 0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[0], lsep[0, :, 0], rtol=1e-12, atol=1e-12)


def test_single_bucket_is_dense_causal_attention():
    rng = np.random.default_rng(42)
    n, d = 17, 6
    X = rng.standard_normal((1, 1, n, d))
    X[..., 0] = np.abs(X[..., 0]) + 0.1                     # u = x . e1 > 0: every token in bucket 0
    V = rng.standard_normal((1, 1, n, d))
    R = np.zeros((1, 2, d, 1), dtype=np.float32)
    R[0, :, 0, 0] = 1.0
    O, lse, cnt = oracle.lsh_decode(X, V, R, 2, np.array([n]), no_self=True, key_norm=True, scale=0.5)
    q = X[0, 0, -1]
    K = X[0, 0, :-1] / np.linalg.norm(X[0, 0, :-1], axis=1, keepdims=True)
    lg = 0.5 * K @ q
    p = np.exp(lg - lg.max())
    assert cnt[0, 0] == n - 1
    np.testing.assert_allclose(O[0, 0], (p / p.sum()) @ V[0, 0, :-1], rtol=1e-12, atol=1e-12)


def test_union_over_rounds_by_brute_force():
    """Rows of different lengths, three rounds: the newest token t of each row attends to
    every j <= t sharing a bucket with it in some round, each j once (with and without
    itself), keys normalised; written out with Python sets and a plain softmax."""
    rng = np.random.default_rng(43)
    S, H, n_max, d, b, rounds = 3, 2, 20, 6, 4, 3
    X = rng.standard_normal((S, H, n_max, d)).astype(np.float32)
    V = rng.standard_normal((S, H, n_max, d))
    R = rng.standard_normal((H, rounds, d, b // 2)).astype(np.float32)
    lengths = np.array([5, 13, 20])
    bucket = oracle.lsh_hash(X, R, b)                      # [S, H, rounds, n_max]
    for no_self in (True, False):
        O, lse, cnt = oracle.lsh_decode(X, V, R, b, lengths, no_self=no_self, scale=0.7)
        for s in range(S):
            t = int(lengths[s]) - 1
            for h in range(H):
                cand = {j for j in range(t + 1) for r in range(rounds) if bucket[s, h, r, j] == bucket[s, h, r, t]}
                if no_self:
                    cand.discard(t)
                cand = sorted(cand)
                assert cnt[s, h] == len(cand)
                q = X[s, h, t].astype(np.float64)
                K = X[s, h, cand].astype(np.float64)
                K = K / np.linalg.norm(K, axis=1, keepdims=True)
                lg = 0.7 * (K @ q)
                m = lg.max()
                p = np.exp(lg - m)
                np.testing.assert_allclose(O[s, h], (p / p.sum()) @ V[s, h, cand], rtol=1e-12, atol=1e-12)
                assert abs(lse[s, h] - (m + math.log(p.sum()))) < 1e-12


def test_first_token_without_itself_has_an_empty_set():
    rng = np.random.default_rng(44)
    X = rng.standard_normal((1, 1, 4, 6)).astype(np.float32)
    V = rng.standard_normal((1, 1, 4, 6))
    R = rng.standard_normal((1, 2, 6, 2)).astype(np.float32)
    O, lse, cnt = oracle.lsh_decode(X, V, R, 4, np.array([1]), no_self=True)
    assert cnt[0, 0] == 0 and lse[0, 0] == -np.inf and not O[0, 0].any()
