"""Pins for routing (k-means) attention with quota execution (PaperTrace 2.1.1 §3.1-3.2):
the page's six-token worked example through the quota path, quota m = n reducing to
dense causal attention, and on integer-valued inputs (exact fp32 scores) the quotas equal
a brute-force ranking with the union of a query's centres counted once."""
import numpy as np

import oracle
from conftest import golden


def test_six_token_example_through_the_quota():
    g = golden("p1_kmeans_quota.json")
    keys = np.array(g["keys"])
    n = len(keys)
    Q = np.tile([0.0, 1.0], (n, 1))
    Q[0] = g["query"]                                   # row 0 carries q; the others point at centre 2
    V = np.zeros((n, 2))
    V[:, 0] = g["values"]
    M = np.array(g["centres"], dtype=np.float32)[None]
    JQ, JK, O, lse, cnt = oracle.kmeans_route(Q[None, None], keys[None, None], V[None, None], M, 3,
                                              causal=False, no_self=False, scale=1.0)
    assert list(JQ[0, 0, 0]) == [0, 1, 2] and 0 not in JQ[0, 0, 1]
    assert list(JK[0, 0, 0]) == [0, 1, 2] and list(JK[0, 0, 1]) == [3, 4, 5]
    assert cnt[0, 0, 0] == 3
    assert abs(O[0, 0, 0, 0] - g["derived"]["output"]) < 1e-3
    np.testing.assert_allclose(keys[:3] @ np.array(g["query"]), g["printed"]["scores_k1_k3"], atol=1e-12)
    np.testing.assert_allclose(keys[:3].mean(axis=0), g["printed"]["cluster1_mean"], atol=1e-12)
    assert abs(keys[5] @ np.array(g["query"]) - g["printed"]["k6_score"]) < 1e-12


def test_full_quota_is_dense_causal_attention():
    rng = np.random.default_rng(71)
    n, d, C = 12, 8, 3
    Q = rng.standard_normal((1, 1, n, d))
    K = rng.standard_normal((1, 1, n, d))
    V = rng.standard_normal((1, 1, n, d))
    M = rng.standard_normal((1, C, d)).astype(np.float32)
    _, _, O, lse, cnt = oracle.kmeans_route(Q, K, V, M, n, causal=True, scale=0.3)
    for i in range(n):
        lg = 0.3 * K[0, 0, : i + 1] @ Q[0, 0, i]
        p = np.exp(lg - lg.max())
        assert cnt[0, 0, i] == i + 1
        np.testing.assert_allclose(O[0, 0, i], (p / p.sum()) @ V[0, 0, : i + 1], rtol=1e-12, atol=1e-12)


def test_quotas_and_union_by_brute_force():
    rng = np.random.default_rng(72)
    n, d, C, m = 20, 4, 5, 6
    Q = rng.integers(-3, 4, (1, 1, n, d)).astype(np.float64)     # integer values: exact fp32 scores
    K = rng.integers(-3, 4, (1, 1, n, d)).astype(np.float64)
    V = rng.standard_normal((1, 1, n, d))
    M = rng.integers(-2, 3, (1, C, d)).astype(np.float32)
    JQ, JK, O, lse, cnt = oracle.kmeans_route(Q, K, V, M, m, causal=True, no_self=True)
    for J, X in ((JQ, Q), (JK, K)):
        for c in range(C):
            sc = X[0, 0] @ M[0, c]
            order = sorted(range(n), key=lambda i: (-sc[i], i))[:m]   # score desc, index asc
            assert list(J[0, 0, c]) == sorted(order)
    for i in range(n):
        U = {int(j) for c in range(C) if i in JQ[0, 0, c] for j in JK[0, 0, c] if j < i}
        assert cnt[0, 0, i] == len(U)
        if U:
            js = sorted(U)
            lg = K[0, 0, js] @ Q[0, 0, i] / np.sqrt(d)
            p = np.exp(lg - lg.max())
            np.testing.assert_allclose(O[0, 0, i], (p / p.sum()) @ V[0, 0, js], rtol=1e-12, atol=1e-12)
        else:
            assert np.all(O[0, 0, i] == 0) and lse[0, 0, i] == -np.inf
