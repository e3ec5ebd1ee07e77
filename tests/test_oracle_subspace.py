"""Pins for the query-subspace descriptors and selection of the oracle ("COBS 阅读笔记",
"子空间方法", Eq.(17)-(18)): the identity subspace reproduces the full-space descriptors,
the quadratic term equals the covariance quadratic form of the projected query computed
from the keys themselves, the eigenvalues are those of U^T Sigma U, and keys that lie in
the subspace are selected exactly as by the full-space selector."""
import numpy as np

import oracle


def _orthonormal(rng, D, s):
    q, _ = np.linalg.qr(rng.standard_normal((D, s)))
    return q


def test_identity_subspace_is_the_full_space():
    rng = np.random.default_rng(11)
    Kb = rng.standard_normal((5, 8, 6))
    mu0, xi0, lam0 = oracle.block_describe(Kb, 3)
    mu1, xi1, lam1 = oracle.block_describe_ss(Kb, np.eye(6), 3)
    np.testing.assert_allclose(mu1, mu0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lam1, lam0, rtol=1e-10, atol=1e-12)
    # eigenvector signs are arbitrary
    np.testing.assert_allclose(np.abs(np.einsum("bed,bed->be", xi1, xi0)),
                               np.einsum("bed,bed->be", xi0, xi0), rtol=1e-9, atol=1e-12)


def test_eigenvalues_are_those_of_the_projected_covariance():
    rng = np.random.default_rng(12)
    D, s, L = 10, 4, 8
    Kb = rng.standard_normal((3, L, D))
    U = _orthonormal(rng, D, s)
    _, _, lam = oracle.block_describe_ss(Kb, U, 4)
    for b in range(3):
        kt = Kb[b] - Kb[b].mean(axis=0)
        B = U.T @ (kt.T @ kt / L) @ U
        np.testing.assert_allclose(lam[b], np.sort(np.linalg.eigvalsh(B))[::-1], rtol=1e-9, atol=1e-12)


def test_quadratic_term_is_the_projected_query_form():
    """Eq.(18): with the rank covering the subspace, 1/2 sum_i (xi_i . U^T q)^2 equals
    1/2 (Pi q)^T Sigma_b (Pi q), here evaluated from the keys as (1/L) sum_r ((Pi q).(k_r - mu))^2."""
    rng = np.random.default_rng(13)
    D, s, L, n_full, rank = 8, 3, 4, 6, 3
    keys = rng.standard_normal((n_full, L, D))
    U = _orthonormal(rng, D, s)
    mu, xi, _ = oracle.block_describe_ss(keys, U, rank)
    q = rng.standard_normal((1, 1, D))
    _, _, _, bs = oracle.block_select_ss(q, U, mu.reshape(1, 1, n_full, D),
                                         xi.reshape(1, 1, n_full, rank, s), n_full * L, L, 2, 0, scale=1.0)
    lb = np.log(bs[0, 0])
    pq = U @ (U.T @ q[0, 0])
    direct = np.array([q[0, 0] @ keys[b].mean(axis=0)
                       + 0.5 * np.mean(((keys[b] - keys[b].mean(axis=0)) @ pq) ** 2) for b in range(n_full)])
    np.testing.assert_allclose(lb - lb[0], direct - direct[0], rtol=0, atol=1e-10)


def test_keys_inside_the_subspace_select_as_in_the_full_space():
    """Keys m + U z (a full-space mean plus a component in span U): every block covariance
    lies in span U, the full-space eigenvectors are U times the subspace ones, so the
    subspace selector's scores and picks equal the full-space selector's ([P5] Eq.(17)-(18)
    against Eq.(14)-(16))."""
    rng = np.random.default_rng(14)
    D, s, L, nb, rank = 10, 4, 8, 9, 3
    U = _orthonormal(rng, D, s)
    m = rng.standard_normal(D)
    z = rng.standard_normal((nb * L, s)) * np.linspace(0.5, 2.0, s)
    K = (m + z @ U.T).reshape(nb, L, D)
    mu, xi, _ = oracle.block_describe(K, rank)
    mu_s, xi_s, _ = oracle.block_describe_ss(K, U, rank)
    Q = rng.standard_normal((1, 2, D))
    T, top, win = nb * L, 3, 8
    full = oracle.block_select(Q, mu[None, None], xi[None, None], T, L, top, win, scale=0.5)
    sub = oracle.block_select_ss(Q, U, mu_s[None, None], xi_s[None, None], T, L, top, win, scale=0.5)
    np.testing.assert_allclose(sub[3], full[3], rtol=1e-9, atol=1e-9)     # block scores
    assert np.array_equal(sub[2], full[2])                                # picked blocks
    assert np.array_equal(sub[0], full[0]) and np.array_equal(sub[1], full[1])
