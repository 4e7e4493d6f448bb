"""Attention-aware key transform (fp64 CPU oracle).

Test infrastructure, under the same rules as ``lrkv_oracle``: only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import it; the CUDA library never does.

NOVA-KV summary, "Methodology > Key Transform Derivation":
* the key-side attention error of a reconstruction K_hat is
  ||Q K^T - Q K_hat^T||_F^2 = sum_j (k_j - k_hat_j) M_q (k_j - k_hat_j)^T with
  M_q = Q^T Q (eq. 5; keys and queries are row vectors);
* Theorem 1: the optimal rank-p key transform is R = M_q^{1/2} E_{1:p}, with
  E Lambda E^T the eigendecomposition of M_q^{1/2} S_k M_q^{1/2} and S_k the
  centred key scatter;
* Proposition 1 (generalised Parseval): with k = r R^{-1} (the full, square R),
  ||r - r_hat||^2 = ||k - k_hat||^2_{M_q}.

Reading R22 (what the page leaves open): the transform acts on centred keys,
r = (k - mu) R with mu the mean calibration key, and the rank-p reconstruction
keeps the first p transform coefficients:
    k_hat = mu + (k - mu) M_q^{1/2} E_p E_p^T M_q^{-1/2}.
In coefficient space (the form a decode kernel would read) a key is stored as
c = E_p^T M_q^{1/2} (k - mu)^T and a query is projected with the other
factor, q~ = E_p^T M_q^{-1/2} q^T, so that q . k_hat = q . mu + q~ . c: the
key-side basis W_k = M_q^{1/2} E_p and the query-side basis
W_q = M_q^{-1/2} E_p differ, and every compressed logit gains the bias q . mu.
M_q must be positive definite (at least d linearly independent queries).
"""
from dataclasses import dataclass

import numpy as np


def _sym_pow(M, power):
    """M^power of a symmetric positive definite matrix (eigendecomposition)."""
    m, V = np.linalg.eigh(M)
    if m.min() <= 1e-12 * m.max():                # singular up to rounding
        raise ValueError("M_q is not positive definite: more independent queries are needed")
    return (V * m ** power) @ V.T


@dataclass
class KeyTransform:
    """Theorem 1's transform of one kv head and what is derived from it."""
    mu: np.ndarray      # [d] mean calibration key
    M_q: np.ndarray     # [d, d] Q^T Q
    R: np.ndarray       # [d, d] M_q^{1/2} E, columns by decreasing eigenvalue
    lam: np.ndarray     # [d] eigenvalues of M_q^{1/2} S_k M_q^{1/2}, descending
    E: np.ndarray       # [d, d] their eigenvectors

    def W_k(self, p):
        """Key-side basis [d, p]: c = W_k^T (k - mu)."""
        return self.R[:, :p]

    def W_q(self, p):
        """Query-side basis [d, p]: q~ = W_q^T q."""
        return _sym_pow(self.M_q, -0.5) @ self.E[:, :p]

    def reconstruct(self, K, p):
        """k_hat of keys K [N, d] at rank p (reading R22)."""
        K = np.asarray(K, np.float64)
        A = self.R[:, :p] @ self.E[:, :p].T @ _sym_pow(self.M_q, -0.5)
        return self.mu + (K - self.mu) @ A


def key_transform(Q, K):
    """Theorem 1 from calibration queries Q [Nq, d] and keys K [Nk, d] (one kv head)."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    M_q = Q.T @ Q
    mu = K.mean(axis=0)
    Kc = K - mu
    S_k = Kc.T @ Kc
    Mh = _sym_pow(M_q, 0.5)
    lam, E = np.linalg.eigh(Mh @ S_k @ Mh)
    order = np.argsort(-lam, kind="stable")
    lam, E = lam[order], E[:, order]
    return KeyTransform(mu=mu, M_q=M_q, R=Mh @ E, lam=lam, E=E)


def weighted_key_error(M_q, K, K_hat):
    """sum_j (k_j - k_hat_j) M_q (k_j - k_hat_j)^T (eq. 5's right-hand side)."""
    D = np.asarray(K, np.float64) - np.asarray(K_hat, np.float64)
    return float(np.einsum("ji,ik,jk->", D, M_q, D))
