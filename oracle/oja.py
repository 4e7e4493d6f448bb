"""Online basis update with Oja's subspace rule (fp64 CPU oracle).

Test infrastructure, under the same rules as ``lrkv_oracle``: only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import it; the CUDA library never does.

OjaKV repository README, "Method Summary > OjaKV": the low-rank subspace is
updated online with Oja's algorithm, during prefill and during decoding, so
that it follows the context.  The page gives no update rule, step size or
normalisation.  Reading R23 (the plainest form of Oja's algorithm for an
r-dimensional subspace):
    y = U^T x,   U <- U + eta (x - U y) y^T
averaged over the rows of a batch (a prefill chunk) or taken once per row
(a decode step), then re-orthonormalised by a QR factorisation whose R has a
positive diagonal (the columns stay a basis with orthonormal columns, as the
projection c = U^T x assumes).  How a cache treats coefficients written under
an older basis is not on the page and is not modelled here.
"""
import numpy as np


def _orthonormalise(A):
    """Q of A = Q R with R's diagonal positive (columns of A independent)."""
    Q, R = np.linalg.qr(A)
    s = np.sign(np.diag(R))
    s[s == 0] = 1.0
    return Q * s


def oja_direction(U, X):
    """Mean Oja update direction over rows X [N, d]: (1/N) sum_n (x_n - U y_n) y_n^T."""
    U = np.asarray(U, np.float64)
    X = np.asarray(X, np.float64)
    Y = X @ U                                     # rows y_n^T = x_n^T U
    return (X - Y @ U.T).T @ Y / X.shape[0]


def oja_step(U, X, eta):
    """One batch step (reading R23): U + eta * oja_direction(U, X), re-orthonormalised."""
    return _orthonormalise(np.asarray(U, np.float64) + eta * oja_direction(U, X))


def oja_stream(U, X, eta):
    """One step per row of X, in order (decode: one new token per step)."""
    U = np.asarray(U, np.float64)
    for x in np.asarray(X, np.float64):
        U = oja_step(U, x[None, :], eta)
    return U
