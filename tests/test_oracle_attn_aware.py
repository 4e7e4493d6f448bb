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


# ---------------------------------------------------------------------------
# the transform inside a cache (reading R24): c = W_k^T (k - mu), k_hat = mu + W_q c
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("p", [3, 8, 16])
def test_cache_projection_reaches_the_discarded_mass(p):
    """The cache's own projection and reconstruction (oracle.project / reconstruct
    with the key-side basis W_k, the query-side basis W_q and the mean) give the
    Theorem 1 error: the M_q-weighted key error equals the discarded eigenvalues.
    A transposed basis, the wrong basis on either side or a dropped mean fails it."""
    rng, Q, K = _data(30 + p)
    T = O.key_transform(Q, K)
    C = O.project(T.W_k(p), K, T.mu)
    K_hat = O.reconstruct(T.W_q(p), C, T.mu)
    err = O.weighted_key_error(T.M_q, K, K_hat)
    assert err == pytest.approx(T.lam[p:].sum(), rel=1e-9, abs=1e-9 * T.lam[0])
    np.testing.assert_allclose(K_hat, T.reconstruct(K, p), rtol=1e-9, atol=1e-9)
    # the same keys through the cache's write path: e is ||k - k_hat|| / ||k||
    e = O.rel_error(T.W_k(p), K, U_rec=T.W_q(p), mu=T.mu)
    np.testing.assert_allclose(e, np.linalg.norm(K - K_hat, axis=1) / np.linalg.norm(K, axis=1),
                               rtol=1e-12)


def _exact_aware_setup(seed, d=128, p=40, T=60, Hq=4):
    """An attention-aware key basis whose arithmetic is exact in bf16: M_q diagonal
    with powers of four, so W_k = M_q^{1/2} E and W_q = M_q^{-1/2} E are signed,
    scaled coordinate columns (E a signed permutation); mu and the keys dyadic.
    Keys with nothing outside the kept p coordinates reconstruct exactly; the
    others are routed (their error is large)."""
    rng = np.random.default_rng(seed)
    perm = rng.permutation(d)[:p]
    sign = rng.choice([-1.0, 1.0], p)
    expo = rng.integers(-2, 3, p).astype(np.float64)            # M_q eigenvalues 4^expo
    W_k = np.zeros((1, d, p))
    W_q = np.zeros((1, d, p))
    W_k[0, perm, np.arange(p)] = sign * 2.0 ** expo
    W_q[0, perm, np.arange(p)] = sign * 2.0 ** -expo
    mu = O.bf16_round(rng.integers(-8, 9, d) / 8.0)[None]
    K = O.bf16_round(rng.standard_normal((1, T, 1, d)))
    kept = rng.random(T) < 0.7
    off = np.setdiff1d(np.arange(d), perm)
    for t in np.flatnonzero(kept):
        K[0, t, 0, :] = mu[0]                                     # the mean off the kept coordinates,
        K[0, t, 0, perm] = rng.integers(-64, 65, p) / 16.0        # dyadic values on them
    V = O.bf16_round(rng.standard_normal((1, T, 1, d)))
    U_v = np.eye(d)[None]                                          # values kept exactly
    q = O.bf16_round(rng.standard_normal((1, Hq, d)))
    assert np.all(K[0, kept][:, 0][:, off] == mu[0][off])
    return W_k, W_q, mu, K, V, U_v, q, kept


def _sdpa(q, K, V, g):
    import torch
    qt = torch.from_numpy(np.asarray(q, np.float64))[:, :, None, :]
    out = torch.nn.functional.scaled_dot_product_attention(
        qt, torch.from_numpy(np.asarray(K, np.float64)), torch.from_numpy(np.asarray(V, np.float64)),
        enable_gqa=(g > 1))
    return out[:, :, 0, :].numpy()


def test_aware_cache_with_exact_keys_is_dense_attention():
    """A cache with the attention-aware basis, its mean and both token sets:
    compressed keys reconstruct exactly (k_hat = mu + W_q W_k^T (k - mu) = k on the
    kept coordinates), routed keys are used as stored, so the decode over the cache
    must equal dense attention over the raw K, V (torch's SDPA) -- which pins the
    mean in the projection, the query-side basis in the reconstruction and the
    q . mu term of the coefficient-space logits."""
    W_k, W_q, mu, K, V, U_v, q, kept = _exact_aware_setup(5)
    d, p, T, Hq = 128, W_k.shape[2], K.shape[1], q.shape[1]
    D = O.Dims(B=1, Hq=Hq, Hkv=1, d=d, r_k=p, r_v=d, T_cap=64, F_cap=64)
    cache = O.Cache.empty(D, W_k, U_v, U_kq=W_q, mu_k=mu)
    e, ek, _ = O.compress(cache, K, V, tau=0.05)
    routed = cache.routed(0, 0, np.arange(T))
    assert np.array_equal(routed, ~kept) and np.all(ek[0, 0, kept] == 0.0)
    ref = _sdpa(q, K.transpose(0, 2, 1, 3), V.transpose(0, 2, 1, 3), Hq)
    np.testing.assert_allclose(O.decode_attn(cache, q), ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(O.decode_attn_coef(cache, q), ref, rtol=1e-12, atol=1e-13)
    # reading the same stored coefficients without the mean, or with the key-side
    # basis on the query side, is not dense attention
    import dataclasses
    for bad in (dataclasses.replace(cache, U_kq=W_k), dataclasses.replace(cache, mu_k=None)):
        assert np.abs(O.decode_attn(bad, q) - ref).max() > 1e-3
        assert np.abs(O.decode_attn_coef(bad, q) - ref).max() > 1e-3
