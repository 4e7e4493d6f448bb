"""Plain fp64 CPU oracle of low-rank compressed-KV decode attention.

Test infrastructure.  This module is the slow, obviously-correct statement
of what the CUDA library computes; it shares no code with it and never
imports it.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference arm may import, call or run anything here.  The
product path must never route through it.

What it follows
---------------
* OjaKV repository README, "Method Summary > StaticPCA": a fixed per-head
  low-rank basis, with keys and values reconstructed on the fly for
  standard attention.  The decode here is exactly that plain definition:
  rebuild K_hat = U_k c_k and V_hat = U_v c_v, then dense softmax attention.
* OjaKV repository README, "Method Summary > OjaKV": the hybrid storage
  policy -- tokens with a high reconstruction error are kept in full rank,
  the rest are compressed.
* The coefficient-space form of the same decode (logits (U_k^T q).c_k/sqrt(d),
  one softmax over compressed and full-rank tokens together,
  o = U_v sum_j p_j c_vj + sum_j p_j v_j) is the algebraic identity
  q.(U c) = (U^T q).c applied to the plain definition; ``decode_attn_coef``
  writes it out separately so the two can be checked against each other.

Readings taken where the pages are silent (each one is listed with its
reason in the design notes of the repository):
  R1  no mean-centring: c = U^T x.
  R2  one full-rank list per (batch row, kv head); a token is routed when
      max(e_k, e_v) > tau, and then both its key and value rows are kept.
  R3  strict ">" routes.          R4  ||x|| = 0 gives e = 0 (not routed).
  R5  routing uses the unrounded projection c (fp64 here).
  R6  the error is computed by direct reconstruction ||x - U c|| / ||x||.
  R7  coefficients of routed tokens are still stored at their position.
  R8  logits are scaled by 1/sqrt(d), d the head dimension.
  R10 a decode step appends first, then attends (the new token included).
  R12 every bfloat16 rounding is round-to-nearest-even.
Attention-aware key basis (NOVA-KV summary, Theorem 1 and Proposition 1;
reading R24 of how a cache uses it): a cache may carry a second key basis
U_kq (the query-side / reconstruction basis) and a key mean mu_k.  Then
c_k = U_k^T (k - mu_k), k_hat = mu_k + U_kq c_k, the key error is
||k - k_hat|| / ||k||, and the decode reads q~ = U_kq^T q with compressed
logits (q . mu_k + q~ . c_k) / sqrt(d).  Without them U_kq = U_k, mu_k = 0:
the plain StaticPCA cache above.  Values are never transformed this way.
Capacity: a sequence never grows past T_cap (the tokens that do not fit are
dropped and SEQ_OVERFLOW is raised); routed tokens beyond F_cap are kept
compressed instead (mask bit clear) and FULL_OVERFLOW is raised.  Routing is
order preserving: the full-rank list holds positions in ascending order.

Parity pins: every function here is checked in tests/ against closed forms,
invariants and library routines (Eckart-Young via numpy.linalg.eigh,
Parseval, dense attention via torch's scaled_dot_product_attention when
r = d and U = I or when K/V lie in span(U), softmax rows summing to one,
the softmax Lipschitz bound of the NOVA-KV summary, brute force on tiny
inputs).  No function is "parity unpinned".
"""
from dataclasses import dataclass, field

import numpy as np

from .bf16 import bf16_round

FULL_OVERFLOW = 0x1   # routed tokens exceeded F_cap: kept compressed instead
SEQ_OVERFLOW = 0x2    # seq_len + new tokens exceeded T_cap: the excess dropped


@dataclass
class Dims:
    B: int
    Hq: int
    Hkv: int
    d: int
    r_k: int
    r_v: int
    T_cap: int
    F_cap: int

    @property
    def g(self):
        return self.Hq // self.Hkv


@dataclass
class Cache:
    """One layer of compressed cache, laid out like the library's buffers.

    Shapes: U_k [Hkv,d,r_k], U_v [Hkv,d,r_v]; coef_k [B,Hkv,T_cap,r_k];
    coef_v [B,Hkv,T_cap,r_v]; route_mask [B,Hkv,T_cap/32] (bit p%32 of word
    p//32 set when position p is held in full rank); full_idx [B,Hkv,F_cap];
    full_k/full_v [B,Hkv,F_cap,d]; full_cnt [B,Hkv]; seq_len [B].
    Floating values are float64 holding bfloat16-representable numbers.
    """
    dims: Dims
    U_k: np.ndarray
    U_v: np.ndarray
    coef_k: np.ndarray = field(default=None)
    coef_v: np.ndarray = field(default=None)
    route_mask: np.ndarray = field(default=None)
    full_idx: np.ndarray = field(default=None)
    full_k: np.ndarray = field(default=None)
    full_v: np.ndarray = field(default=None)
    full_cnt: np.ndarray = field(default=None)
    seq_len: np.ndarray = field(default=None)
    status: int = 0
    U_kq: np.ndarray = field(default=None)    # [Hkv,d,r_k] key reconstruction basis, None: U_k
    mu_k: np.ndarray = field(default=None)    # [Hkv,d] key mean, None: 0

    @staticmethod
    def empty(dims, U_k, U_v, U_kq=None, mu_k=None):
        D = dims
        if D.T_cap % 32:
            raise ValueError("T_cap must be a multiple of 32")
        z = np.zeros
        return Cache(
            dims=D,
            U_kq=None if U_kq is None else np.asarray(U_kq, np.float64),
            mu_k=None if mu_k is None else np.asarray(mu_k, np.float64),
            U_k=np.asarray(U_k, np.float64), U_v=np.asarray(U_v, np.float64),
            coef_k=z((D.B, D.Hkv, D.T_cap, D.r_k)), coef_v=z((D.B, D.Hkv, D.T_cap, D.r_v)),
            route_mask=z((D.B, D.Hkv, D.T_cap // 32), np.uint32),
            full_idx=z((D.B, D.Hkv, D.F_cap), np.int32),
            full_k=z((D.B, D.Hkv, D.F_cap, D.d)), full_v=z((D.B, D.Hkv, D.F_cap, D.d)),
            full_cnt=z((D.B, D.Hkv), np.int32), seq_len=z((D.B,), np.int32), status=0)

    def key_rec_basis(self, h):
        """The basis keys of kv head h are reconstructed with (and q~ taken in)."""
        return self.U_k[h] if self.U_kq is None else self.U_kq[h]

    def key_mean(self, h):
        """The mean subtracted from keys of kv head h before projection."""
        return np.zeros(self.dims.d) if self.mu_k is None else self.mu_k[h]

    def routed(self, b, h, pos):
        """True where the mask marks position(s) ``pos`` of (b, h) as full rank."""
        pos = np.asarray(pos)
        words = self.route_mask[b, h, pos // 32]
        return ((words >> (pos % 32).astype(np.uint32)) & 1).astype(bool)


# ---------------------------------------------------------------------------
# write path: projection, error, routing (OjaKV README, Method Summary)
# ---------------------------------------------------------------------------

def project(U, X, mu=None):
    """Coefficients c = U^T (x - mu) for every row x of X.  U [d,r], X [...,d] -> [...,r].

    StaticPCA (OjaKV README, Method Summary): tokens are represented by their
    coordinates in the fixed per-head basis.  Reading R1: no mean-centring
    (mu = None); an attention-aware key basis (reading R24) subtracts its mean.
    """
    X = np.asarray(X, np.float64)
    if mu is not None:
        X = X - np.asarray(mu, np.float64)
    return X @ np.asarray(U, np.float64)


def reconstruct(U, C, mu=None):
    """x_hat = mu + U c for every row c of C (the on-the-fly reconstruction)."""
    Xh = np.asarray(C, np.float64) @ np.asarray(U, np.float64).T
    return Xh if mu is None else Xh + np.asarray(mu, np.float64)


def rel_error(U, X, C=None, U_rec=None, mu=None):
    """Per-token relative reconstruction error ||x - x_hat|| / ||x|| (readings R4, R6).

    OjaKV README, Method Summary > OjaKV: "reconstruction error" decides which
    tokens stay in full rank.  Computed by direct reconstruction,
    x_hat = mu + U_rec c with c = U^T (x - mu) (U_rec = U and mu = 0 unless an
    attention-aware key basis is used, reading R24); ||x|| = 0 gives 0.
    """
    X = np.asarray(X, np.float64)
    if C is None:
        C = project(U, X, mu)
    num = np.linalg.norm(X - reconstruct(U if U_rec is None else U_rec, C, mu), axis=-1)
    den = np.linalg.norm(X, axis=-1)
    return np.where(den > 0, num / np.where(den > 0, den, 1.0), 0.0)


# ---------------------------------------------------------------------------
# the offline basis (OjaKV README, Method Summary > StaticPCA; KV-CoRE page,
# abstract: the Frobenius-optimal low-rank approximation)
# ---------------------------------------------------------------------------

def fit_basis(X, r):
    """StaticPCA's offline basis of one kv head: the top-r eigenvectors of the
    (uncentred, reading R1) scatter matrix G = X^T X of the calibration rows.

    OjaKV README, "Method Summary > StaticPCA": an offline low-rank basis
    computed from a calibration corpus.  KV-CoRE page, abstract: the optimal
    low-rank approximation under the Frobenius norm; by Eckart-Young that is
    the span of G's leading eigenvectors, and the residual sum of squares is
    the discarded eigenvalue mass.

    X: [N, d] rows (bfloat16 values as float64).  Returns (U [d, r], lam [d])
    with lam descending and U's columns the matching unit eigenvectors.  Sign
    (reading R18): each column's entry of largest magnitude is positive (the
    lowest index on a tie).
    """
    X = np.asarray(X, np.float64)
    G = X.T @ X
    lam, V = np.linalg.eigh(G)               # ascending
    order = np.argsort(-lam, kind="stable")
    lam, V = lam[order], V[:, order]
    for j in range(V.shape[1]):
        i = int(np.argmax(np.abs(V[:, j])))  # first index of the largest magnitude
        if V[i, j] < 0:
            V[:, j] = -V[:, j]
    return V[:, :r], lam


def rank_for_budget(lam, budget):
    """Smallest rank whose discarded eigenvalue mass is within the error budget.

    OjaKV README (calibration command, `--error_budget`) and KV-CoRE page,
    abstract (Frobenius-optimal low-rank approximation).  Reading R20: the
    budget bounds the relative squared Frobenius error of the rank-r
    approximation of the calibration rows, which by Eckart-Young is the mass
    of the discarded eigenvalues over the total:
        r = min { r in 1..d : sum_{j >= r} lam_j <= budget * sum_j lam_j }
    with negative eigenvalues (rounding of a positive semi-definite matrix)
    counted as zero; the sums run from the smallest eigenvalue up, in fp64.

    lam: [d] eigenvalues, descending.  Returns an int.
    """
    lam = np.asarray(lam, np.float64)
    lam = np.where(lam > 0.0, lam, 0.0)
    d = lam.shape[0]
    tail = [0.0] * (d + 1)
    for j in range(d - 1, -1, -1):
        tail[j] = tail[j + 1] + float(lam[j])
    limit = float(budget) * tail[0]
    for r in range(1, d + 1):
        if tail[r] <= limit:
            return r
    return d


def route(e_k, e_v, tau):
    """Full-rank decision per token: max(e_k, e_v) > tau (readings R2, R3)."""
    return np.maximum(e_k, e_v) > tau


def compress(cache, k_new, v_new, tau, t_new_b=None):
    """Append new tokens to every sequence of ``cache`` (mutates it).

    k_new, v_new: [B, t_new, Hkv, d] (bfloat16 values as float64); row b uses
    its first t_new_b[b] tokens (all t_new when t_new_b is None).  Tokens go
    to positions seq_len[b], seq_len[b]+1, ...; each is projected, its
    error measured and routed; routed tokens are appended to the full-rank
    list in ascending position order.  Returns (e, e_k, e_v), each
    [B, Hkv, t_new] float64, NaN where no token was written.
    """
    D = cache.dims
    k_new = np.asarray(k_new, np.float64)
    v_new = np.asarray(v_new, np.float64)
    B, t_new, Hkv, d = k_new.shape
    assert (B, Hkv, d) == (D.B, D.Hkv, D.d) and v_new.shape == k_new.shape
    e_all = np.full((B, Hkv, t_new), np.nan)
    ek_all = np.full((B, Hkv, t_new), np.nan)
    ev_all = np.full((B, Hkv, t_new), np.nan)
    for b in range(B):
        n = t_new if t_new_b is None else int(t_new_b[b])
        if n < 0 or n > t_new:
            raise ValueError("t_new_b[b] must lie in [0, t_new]")
        start = int(cache.seq_len[b])
        n_eff = min(n, D.T_cap - start)
        if n_eff < n:
            cache.status |= SEQ_OVERFLOW
        if n_eff <= 0:
            continue
        for h in range(Hkv):
            K = k_new[b, :n_eff, h, :]
            V = v_new[b, :n_eff, h, :]
            mu = cache.key_mean(h)
            ck = project(cache.U_k[h], K, mu)
            cv = project(cache.U_v[h], V)
            ek = rel_error(cache.U_k[h], K, ck, U_rec=cache.key_rec_basis(h), mu=mu)
            ev = rel_error(cache.U_v[h], V, cv)
            full = route(ek, ev, tau)
            pos = start + np.arange(n_eff)
            cache.coef_k[b, h, pos] = bf16_round(ck)        # reading R7: stored for every token
            cache.coef_v[b, h, pos] = bf16_round(cv)
            for t in range(n_eff):
                p = start + t
                w, bit = p // 32, np.uint32(1 << (p % 32))
                keep_full = bool(full[t])
                if keep_full and cache.full_cnt[b, h] >= D.F_cap:
                    cache.status |= FULL_OVERFLOW
                    keep_full = False
                if keep_full:
                    slot = int(cache.full_cnt[b, h])
                    cache.full_idx[b, h, slot] = p
                    cache.full_k[b, h, slot] = K[t]
                    cache.full_v[b, h, slot] = V[t]
                    cache.full_cnt[b, h] = slot + 1
                    cache.route_mask[b, h, w] |= bit
                else:
                    cache.route_mask[b, h, w] &= ~bit
            e_all[b, h, :n_eff] = np.maximum(ek, ev)
            ek_all[b, h, :n_eff] = ek
            ev_all[b, h, :n_eff] = ev
        cache.seq_len[b] = start + n_eff
    return e_all, ek_all, ev_all


# ---------------------------------------------------------------------------
# read path: decode attention over the compressed cache
# ---------------------------------------------------------------------------

def effective_kv(cache, b, h):
    """K_hat, V_hat [T_b, d] of (b, kv head h): reconstructed or full-rank rows.

    OjaKV README, Method Summary > StaticPCA: keys and values are
    reconstructed on the fly; full-rank tokens (Method Summary > OjaKV)
    are used as stored.  The full-rank row of position p is the one whose
    full_idx entry equals p.
    """
    T = int(cache.seq_len[b])
    pos = np.arange(T)
    K = reconstruct(cache.key_rec_basis(h), cache.coef_k[b, h, :T], cache.key_mean(h))
    V = reconstruct(cache.U_v[h], cache.coef_v[b, h, :T])
    n_full = int(cache.full_cnt[b, h])
    idx = cache.full_idx[b, h, :n_full]
    full = cache.routed(b, h, pos) if T else np.zeros(0, bool)
    if not np.array_equal(np.sort(idx), np.flatnonzero(full)):
        raise ValueError("route mask and full-rank list disagree")
    K[idx] = cache.full_k[b, h, :n_full]
    V[idx] = cache.full_v[b, h, :n_full]
    return K, V


def softmax(s):
    """Numerically stable softmax of a 1-D vector (max subtracted first)."""
    s = np.asarray(s, np.float64)
    if s.size == 0:
        return s
    z = np.exp(s - s.max())
    return z / z.sum()


def decode_attn(cache, q):
    """Single-token decode attention, plain definition: reconstruct then attend.

    q [B, Hq, d] -> out [B, Hq, d] (float64).  Query head h reads kv head
    h // g with g = Hq / Hkv.  Logits q.k_hat/sqrt(d) (reading R8), one
    softmax over all T_b tokens, output p V_hat.  An empty sequence gives 0.
    """
    D = cache.dims
    q = np.asarray(q, np.float64)
    out = np.zeros((D.B, D.Hq, D.d))
    for b in range(D.B):
        if int(cache.seq_len[b]) == 0:
            continue
        for kvh in range(D.Hkv):
            K, V = effective_kv(cache, b, kvh)
            for h in range(kvh * D.g, (kvh + 1) * D.g):
                p = softmax(K @ q[b, h] / np.sqrt(D.d))
                out[b, h] = p @ V
    return out


def decode_attn_coef(cache, q):
    """The same decode written in coefficient space (the method's fast form).

    q_tilde = U_k^T q;  s_t = q_tilde.c_k,t / sqrt(d) for compressed t,
    s_t = q.k_t / sqrt(d) for full-rank t; one softmax over both sets;
    o = U_v (sum_C p_t c_v,t) + sum_F p_t v_t.  With an attention-aware key
    basis (reading R24): q_tilde = U_kq^T q and s_t = (q.mu_k + q_tilde.c_k,t) / sqrt(d).
    """
    D = cache.dims
    q = np.asarray(q, np.float64)
    out = np.zeros((D.B, D.Hq, D.d))
    for b in range(D.B):
        T = int(cache.seq_len[b])
        if T == 0:
            continue
        pos = np.arange(T)
        for kvh in range(D.Hkv):
            full = cache.routed(b, kvh, pos)
            comp = ~full
            n_full = int(cache.full_cnt[b, kvh])
            Fk = cache.full_k[b, kvh, :n_full]
            Fv = cache.full_v[b, kvh, :n_full]
            Ck = cache.coef_k[b, kvh, :T][comp]
            Cv = cache.coef_v[b, kvh, :T][comp]
            for h in range(kvh * D.g, (kvh + 1) * D.g):
                q_t = cache.key_rec_basis(kvh).T @ q[b, h]
                bias = q[b, h] @ cache.key_mean(kvh)
                s = np.concatenate([Ck @ q_t + bias, Fk @ q[b, h]]) / np.sqrt(D.d)
                p = softmax(s)
                pc, pf = p[:Ck.shape[0]], p[Ck.shape[0]:]
                out[b, h] = cache.U_v[kvh] @ (pc @ Cv) + pf @ Fv
    return out

