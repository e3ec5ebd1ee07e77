"""Pins for the block-mass selector part of the oracle (descriptors, scores, selection)."""
import math

import numpy as np
import pytest

import oracle
from conftest import golden


def test_cobs_toy_mean_cov_and_gram_eigen():
    g = golden("p5_cobs_toy.json")
    gg = golden("p5_gram_example.json")
    K = np.array(g["keys"], dtype=np.float64)
    mu, xi, lam = oracle.block_describe(K[None], rank=2)
    assert mu[0] == pytest.approx(g["printed"]["mean"])
    assert lam[0] == pytest.approx(gg["printed"]["eigenvalues_top2"], abs=1e-12)
    for e in range(2):  # sign is free (squared in the score)
        want = np.array(gg["derived"]["xi_up_to_sign"][e])
        assert min(np.abs(xi[0, e] - want).max(), np.abs(xi[0, e] + want).max()) < 1e-12
    # sum xi xi^T reproduces the printed covariance (rank 2 = full rank here)
    cov = sum(np.outer(xi[0, e], xi[0, e]) for e in range(2))
    assert cov == pytest.approx(np.array(g["printed"]["covariance"]), abs=1e-12)


def test_cobs_toy_exact_first_second_order():
    g = golden("p5_cobs_toy.json")
    K = np.array(g["keys"], dtype=np.float64)
    L = g["L"]
    mu, xi, lam = oracle.block_describe(K[None], rank=2)
    for case in g["printed"]["cases"]:
        q = np.array(case["q"])
        assert oracle.block_log_mass(q, K) == pytest.approx(case["ln_mass_exact"], abs=5e-5)
        assert math.exp(oracle.block_log_mass(q, K)) == pytest.approx(case["mass"], abs=5e-4)
        # second order = ln L + block_select's score with scale 1; first order = rank 0
        for rank, key in ((2, "second_order"), (0, "first_order")):
            x = xi[:, :rank] if rank else np.zeros((1, 1, 2))
            # the score of one block is its softmax share; pair it with a zero block
            # (s = 0) so that s_b = log(score_b / score_zero)
            mu2 = np.concatenate([mu, np.zeros((1, 2))])[None, None]
            x2 = np.concatenate([x, np.zeros_like(x)])[None, None]
            _, _, _, bs2 = oracle.block_select(q[None, None], mu2, x2, T=8, L=4, top_blocks=1,
                                               window=0, scale=1.0)
            s_block = math.log(bs2[0, 0, 0] / bs2[0, 0, 1])   # s_b - s_zero, s_zero = 0
            assert math.log(L) + s_block == pytest.approx(case[key], abs=5e-5)


def test_gqa_group_score_example():
    """COBS notes Eq.(P6): masses (6,2) and (1,9) -> scores 0.85 and 1.15; block 2 wins."""
    g = golden("p5_gqa_example.json")["printed"]
    m1, m2 = g["mass_head1"], g["mass_head2"]
    # two heads reading coordinate 0 and 1; block means carry the log-masses
    Q = np.eye(2)[None]                                   # [1 seq, 2 q heads, D=2]
    mu = np.array([[math.log(m1[0]), math.log(m2[0])],
                   [math.log(m1[1]), math.log(m2[1])]])[None, None]
    xi = np.zeros((1, 1, 2, 1, 2))
    tok, cnt, blk, bs = oracle.block_select(Q, mu, xi, T=8, L=4, top_blocks=1, window=0, scale=1.0)
    assert bs[0, 0] == pytest.approx(g["score"], abs=1e-12)
    assert blk[0, 0, 0] + 1 == g["top1_block_1based"]
    assert tok[0, 0, :cnt[0, 0]].tolist() == [4, 5, 6, 7]


def test_gram_route_equals_covariance_route():
    """Eq.(20): Gram-route xi span the top eigen-directions of the D x D covariance
    (LAPACK eigh as the independent route)."""
    rng = np.random.default_rng(0)
    L, D, r = 32, 128, 4
    Kb = rng.standard_normal((3, L, D)) @ np.diag(np.linspace(0.2, 2.0, D))
    mu, xi, lam = oracle.block_describe(Kb, rank=r)
    for b in range(3):
        Kt = Kb[b] - Kb[b].mean(0)
        S = Kt.T @ Kt / L
        w, U = np.linalg.eigh(S)
        w, U = w[::-1], U[:, ::-1]
        assert lam[b] == pytest.approx(w[:r], rel=1e-10)
        P = sum(np.outer(xi[b, e], xi[b, e]) for e in range(r))
        Pref = (U[:, :r] * w[:r]) @ U[:, :r].T
        assert np.abs(P - Pref).max() < 1e-10
        assert mu[b] == pytest.approx(Kb[b].mean(0))


def test_rank_bound_and_trace():
    """Centred rank <= L-1 (COBS notes, '退化的秩'); sum of eigenvalues = tr(Sigma)."""
    rng = np.random.default_rng(1)
    L, D = 8, 20
    Kb = rng.standard_normal((1, L, D))
    mu, xi, lam = oracle.block_describe(Kb, rank=L)
    assert abs(lam[0, L - 1]) < 1e-12 and np.abs(xi[0, L - 1]).max() < 1e-6
    Kt = Kb[0] - Kb[0].mean(0)
    assert lam[0].sum() == pytest.approx(np.trace(Kt.T @ Kt / L), rel=1e-12)


def test_exact_low_rank_block_quadratic_term():
    """A block whose centred keys span 4 orthogonal directions: the rank-4 term is
    exactly 1/2 q^T Sigma q."""
    rng = np.random.default_rng(2)
    L, D = 32, 64
    U, _ = np.linalg.qr(rng.standard_normal((D, 4)))
    A = rng.standard_normal((L, 4)) * np.array([3.0, 2.0, 1.0, 0.5])
    A -= A.mean(0)
    Kb = 0.7 + A @ U.T
    mu, xi, lam = oracle.block_describe(Kb[None], rank=4)
    Sigma = (Kb - Kb.mean(0)).T @ (Kb - Kb.mean(0)) / L
    for _ in range(5):
        q = rng.standard_normal(D)
        quad = sum((xi[0, e] @ q) ** 2 for e in range(4))
        assert quad == pytest.approx(q @ Sigma @ q, rel=1e-10)


def test_partial_block_uses_own_count():
    rng = np.random.default_rng(3)
    L, D = 8, 6
    Kb = rng.standard_normal((1, L, D))
    mu, xi, lam = oracle.block_describe(Kb, rank=2, L_eff=np.array([5], np.int32))
    mu5, xi5, lam5 = oracle.block_describe(Kb[:, :5], rank=2)
    assert mu == pytest.approx(mu5) and lam == pytest.approx(lam5)


def test_window_union_dedup_and_mean_pool_case():
    rng = np.random.default_rng(4)
    n_full, L, D = 8, 4, 5
    Q = rng.standard_normal((1, 2, D))
    mu = rng.standard_normal((1, 1, n_full, D))
    xi = np.zeros((1, 1, n_full, 1, D))     # rank 0: the mean-pool selector
    tok, cnt, blk, bs = oracle.block_select(Q, mu, xi, T=32, L=L, top_blocks=3, window=8, scale=0.5)
    sel = blk[0, 0]
    want = set()
    for b in sel:
        want |= set(range(b * L, b * L + L))
    want |= set(range(24, 32))
    assert tok[0, 0, : cnt[0, 0]].tolist() == sorted(want)
    # mean-pool score order: sum_g softmax_b(0.5 q_g . mu_b)
    s = 0.5 * Q[0] @ mu[0, 0].T
    p = np.exp(s - s.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    assert bs[0, 0] == pytest.approx(p.sum(0))
    assert sorted(np.argsort(-p.sum(0), kind="stable")[:3].tolist()) == sel.tolist()
