"""Pins of the attention-aware key transform oracle (oracle/attn_aware.py).

NOVA-KV summary, "Methodology > Key Transform Derivation": eq. 5 (the
logit error as an M_q-weighted key error), Theorem 1 (the optimal rank-p
transform) and Proposition 1 (the generalised Parseval relation), checked
against direct matrix products, random competitors, and the plain PCA basis
it must reduce to when the queries are isotropic.
"""
import numpy as np
import pytest

import oracle as O


def _data(seed, d=16, Nq=300, Nk=400):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((Nq, d)) * np.linspace(3.0, 0.2, d) @ np.linalg.qr(
        rng.standard_normal((d, d)))[0]
    K = rng.standard_normal((Nk, d)) @ rng.standard_normal((d, d)) * 0.4 + rng.standard_normal(d)
    return rng, Q, K


def test_logit_error_is_the_weighted_key_error():
    """Eq. 5: ||Q K^T - Q K_hat^T||_F^2 = sum_j (k_j - k_hat_j) Q^T Q (k_j - k_hat_j)^T."""
    rng, Q, K = _data(1)
    K_hat = K + 0.1 * rng.standard_normal(K.shape)
    lhs = ((Q @ K.T - Q @ K_hat.T) ** 2).sum()
    assert O.weighted_key_error(Q.T @ Q, K, K_hat) == pytest.approx(lhs, rel=1e-12)


def test_generalised_parseval_and_compander_condition():
    """Proposition 1: coefficient-domain MSE equals the M_q-weighted key error; the
    transform satisfies R R^T = M_q."""
    rng, Q, K = _data(2)
    T = O.key_transform(Q, K)
    assert np.abs(T.R @ T.R.T - T.M_q).max() <= 1e-10 * np.abs(T.M_q).max()
    k = rng.standard_normal((50, K.shape[1]))
    k_hat = k + rng.standard_normal(k.shape) * rng.uniform(0.01, 1.0, (50, 1))
    r, r_hat = (k - T.mu) @ T.R, (k_hat - T.mu) @ T.R
    for j in range(50):
        w = (k[j] - k_hat[j]) @ T.M_q @ (k[j] - k_hat[j])
        assert ((r[j] - r_hat[j]) ** 2).sum() == pytest.approx(w, rel=1e-10)


@pytest.mark.parametrize("p", [1, 4, 9, 15])
def test_theorem1_error_is_the_discarded_mass_and_is_optimal(p):
    """The rank-p reconstruction's weighted error equals the discarded eigenvalues of
    M_q^{1/2} S_k M_q^{1/2}; random rank-p maps and the unweighted PCA basis do no better."""
    rng, Q, K = _data(3 + p)
    T = O.key_transform(Q, K)
    best = O.weighted_key_error(T.M_q, K, T.reconstruct(K, p))
    assert best == pytest.approx(T.lam[p:].sum(), rel=1e-9, abs=1e-9 * T.lam[0])
    d = K.shape[1]
    for _ in range(20):
        A = rng.standard_normal((d, p)) @ rng.standard_normal((p, d))
        assert O.weighted_key_error(T.M_q, K, T.mu + (K - T.mu) @ A) >= best * (1 - 1e-12)
    mu = K.mean(axis=0)
    U, _ = O.fit_basis(K - mu, p)                 # plain PCA of the centred keys
    pca = O.weighted_key_error(T.M_q, K, mu + (K - mu) @ U @ U.T)
    assert pca >= best * (1 - 1e-12)
    if p < d:
        assert pca > best * (1 + 1e-6)           # anisotropic queries: strictly worse


def test_isotropic_queries_give_the_pca_basis():
    """M_q = c I: the key-side basis spans the top principal directions of the centred
    keys (fit_basis), and the query-side basis is the same up to the factor c."""
    rng, _, K = _data(4)
    d, p, c = K.shape[1], 6, 2.5
    Q = np.sqrt(c) * np.eye(d)
    T = O.key_transform(Q, K)
    U, _ = O.fit_basis(K - K.mean(axis=0), p)
    Wk, Wq = T.W_k(p), T.W_q(p)
    Pk = Wk @ np.linalg.pinv(Wk)
    assert np.abs(Pk - U @ U.T).max() < 1e-10
    assert np.abs(Wk - c * Wq).max() < 1e-10 * np.abs(Wk).max()


@pytest.mark.parametrize("p", [3, 8, 16])
def test_coefficient_space_logits(p):
    """q . k_hat = q . mu + (W_q^T q) . (W_k^T (k - mu)): a decode reads key
    coefficients against a query projected with the other factor (reading R22)."""
    rng, Q, K = _data(5)
    T = O.key_transform(Q, K)
    q = rng.standard_normal((7, K.shape[1]))
    k = rng.standard_normal((30, K.shape[1])) + T.mu
    direct = q @ T.reconstruct(k, p).T
    c = (k - T.mu) @ T.W_k(p)                     # [30, p]
    qt = q @ T.W_q(p)                             # [7, p]
    coef = (q @ T.mu)[:, None] + qt @ c.T
    np.testing.assert_allclose(coef, direct, rtol=1e-10, atol=1e-10 * np.abs(direct).max())


def test_full_rank_is_exact_and_singular_queries_are_rejected():
    rng, Q, K = _data(6)
    T = O.key_transform(Q, K)
    np.testing.assert_allclose(T.reconstruct(K, K.shape[1]), K, rtol=0, atol=1e-9 * np.abs(K).max())
    with pytest.raises(ValueError):
        O.key_transform(Q[:, :5] @ rng.standard_normal((5, K.shape[1])), K)
