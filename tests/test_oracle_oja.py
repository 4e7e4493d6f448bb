"""Pins of the online basis update oracle (oracle/oja.py, Oja's subspace rule).

The rule itself is a reading (the page names Oja's algorithm without a rule
or step size), so these pin what Oja's rule fixes whatever the step: rows
inside the span change nothing, the principal subspace is a fixed point, the
update is orthogonal to the current span, it is the first-order form of the
normalised Hebbian update (Oja's derivation), and iterating it on fixed data
converges to the Eckart-Young subspace (the oracle's fit_basis).
"""
import numpy as np
import pytest

import oracle as O


def _rows(seed, N=500, d=24, k=6):
    rng = np.random.default_rng(seed)
    Qm = np.linalg.qr(rng.standard_normal((d, d)))[0]
    scales = np.concatenate([np.linspace(4.0, 2.0, k), np.linspace(0.5, 0.1, d - k)])
    return rng, (rng.standard_normal((N, d)) * scales) @ Qm.T


def _proj(U):
    return U @ U.T


def test_rows_inside_the_span_change_nothing():
    rng, _ = _rows(1)
    d, r = 24, 5
    U = np.linalg.qr(rng.standard_normal((d, r)))[0]
    X = rng.standard_normal((40, r)) @ U.T
    assert np.abs(O.oja_direction(U, X)).max() < 1e-12
    U2 = O.oja_step(U, X, 0.3)
    assert np.abs(_proj(U2) - _proj(U)).max() < 1e-12
    assert np.abs(U2.T @ U2 - np.eye(r)).max() < 1e-12


def test_principal_subspace_is_a_fixed_point():
    """U = top-r eigenvectors of X^T X: (I - U U^T) X^T X U = 0, so the step keeps the span."""
    _, X = _rows(2)
    r = 6
    U, _ = O.fit_basis(X, r)
    assert np.abs(O.oja_direction(U, X)).max() < 1e-10 * np.abs(X).max() ** 2
    assert np.abs(_proj(O.oja_step(U, X, 0.5)) - _proj(U)).max() < 1e-10


def test_update_is_orthogonal_to_the_span():
    rng, X = _rows(3)
    U = np.linalg.qr(rng.standard_normal((X.shape[1], 4)))[0]
    G = O.oja_direction(U, X)
    assert np.abs(U.T @ G).max() < 1e-12 * np.abs(G).max()


def test_first_order_normalised_hebbian_update():
    """r = 1: normalising u + eta y x (Hebbian) agrees with Oja's step to O(eta^2)."""
    rng, X = _rows(4)
    u = rng.standard_normal(X.shape[1])
    u /= np.linalg.norm(u)
    x = X[0]
    errs = []
    for eta in (1e-2, 1e-3, 1e-4):
        y = u @ x
        heb = u + eta * y * x
        heb /= np.linalg.norm(heb)
        oja = O.oja_step(u[:, None], x[None, :], eta)[:, 0]
        errs.append(np.abs(heb - oja).max())
    # shrinking eta tenfold shrinks the gap about a hundredfold
    assert errs[1] < errs[0] / 50 and errs[2] < errs[1] / 50


@pytest.mark.parametrize("r", [1, 3, 6])
def test_batch_steps_converge_to_the_eckart_young_subspace(r):
    rng, X = _rows(5 + r)
    U = np.linalg.qr(rng.standard_normal((X.shape[1], r)))[0]
    eta = 0.5 / np.linalg.eigvalsh(X.T @ X / X.shape[0]).max()
    for _ in range(3000):
        U = O.oja_step(U, X, eta)
    Ut, _ = O.fit_basis(X, r)
    assert np.abs(_proj(U) - _proj(Ut)).max() < 1e-8
    assert np.abs(U.T @ U - np.eye(r)).max() < 1e-12


def test_streaming_steps_track_the_principal_subspace():
    """One step per row over many rows from the same distribution: close to the
    principal subspace (stochastic approximation), and each step keeps orthonormal
    columns."""
    rng, X = _rows(9, N=6000)
    r = 6
    U = np.linalg.qr(rng.standard_normal((X.shape[1], r)))[0]
    U = O.oja_stream(U, X, 2e-3)
    Ut, _ = O.fit_basis(X, r)
    # sine of the largest principal angle between the subspaces
    s = np.linalg.svd((np.eye(X.shape[1]) - _proj(Ut)) @ U, compute_uv=False).max()
    assert s < 0.25
    assert np.abs(U.T @ U - np.eye(r)).max() < 1e-12
