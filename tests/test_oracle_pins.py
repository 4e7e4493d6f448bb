"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each pin is independent of the oracle's own code: a library routine
(numpy.linalg.eigh, torch's scaled_dot_product_attention), a closed form,
an invariant, or a value worked out by hand.  They are chosen so that a
dropped term, a wrong sign or index, or a transposed operand anywhere in
the oracle fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O


def _dims(B=1, Hq=4, Hkv=1, d=128, r_k=32, r_v=32, T_cap=64, F_cap=64):
    return O.Dims(B=B, Hq=Hq, Hkv=Hkv, d=d, r_k=r_k, r_v=r_v, T_cap=T_cap, F_cap=F_cap)


def _sdpa(q, K, V, g):
    """Dense attention by torch (library routine), fp64.  q [B,Hq,d], K/V [B,Hkv,T,d]."""
    qt = torch.from_numpy(np.asarray(q, np.float64))[:, :, None, :]
    out = torch.nn.functional.scaled_dot_product_attention(
        qt, torch.from_numpy(np.asarray(K, np.float64)),
        torch.from_numpy(np.asarray(V, np.float64)), enable_gqa=(g > 1))
    return out[:, :, 0, :].numpy()


def _random_orthonormal(d, r, rng):
    q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    return q[:, :r]


# ---------------------------------------------------------------------------
# projection and reconstruction error
# ---------------------------------------------------------------------------

def test_eckart_young_discarded_eigenvalue_mass():
    """KV-CoRE summary: the best rank-r approximation under the Frobenius norm.

    With U = the top-r eigenvectors of X^T X, sum_t ||x_t - U U^T x_t||^2
    equals the sum of the discarded eigenvalues.
    """
    rng = np.random.default_rng(3)
    T, d, r = 400, 24, 7
    X = rng.standard_normal((T, d)) * np.linspace(3.0, 0.1, d)
    X = X @ _random_orthonormal(d, d, rng).T
    lam, E = np.linalg.eigh(X.T @ X)            # ascending eigenvalues
    U = E[:, ::-1][:, :r]
    e = O.rel_error(U, X)
    resid_energy = np.sum((e * np.linalg.norm(X, axis=1)) ** 2)
    discarded = lam[: d - r].sum()
    assert resid_energy == pytest.approx(discarded, rel=1e-10)
    # a non-optimal basis of the same rank leaves strictly more energy behind
    U2 = E[:, ::-1][:, 1: r + 1]
    e2 = O.rel_error(U2, X)
    assert np.sum((e2 * np.linalg.norm(X, axis=1)) ** 2) > discarded * (1 + 1e-6)


def test_parseval_with_orthonormal_basis():
    """NOVA-KV summary, Proposition 1 with M_q = I: ||x - U c||^2 = ||x||^2 - ||c||^2."""
    rng = np.random.default_rng(4)
    U = _random_orthonormal(128, 48, rng)
    X = rng.standard_normal((300, 128))
    C = O.project(U, X)
    lhs = (O.rel_error(U, X, C) * np.linalg.norm(X, axis=1)) ** 2
    rhs = np.sum(X ** 2, axis=1) - np.sum(C ** 2, axis=1)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-10)
    # the coefficients are the coordinates in the basis: U^T U = I gives x = U c back for x in span
    Xs = rng.standard_normal((5, 48)) @ U.T
    np.testing.assert_allclose(O.reconstruct(U, O.project(U, Xs)), Xs, atol=1e-12)


def test_error_hand_worked():
    """d=4, r=2, U picks coordinates 0 and 2 with signs: c and e by hand."""
    U = np.array([[1.0, 0], [0, 0], [0, -1.0], [0, 0]])
    X = np.array([[3.0, 4.0, 0.0, 0.0],     # c=(3,0), residual (0,4,0,0): e=4/5
                  [0.0, 0.0, 2.0, 0.0],     # in span: c=(0,-2), e=0
                  [0.0, 1.0, 0.0, 0.0],     # orthogonal: e=1
                  [0.0, 0.0, 0.0, 0.0]])    # zero row: e=0 by reading R4
    C = O.project(U, X)
    np.testing.assert_array_equal(C, [[3, 0], [0, -2], [0, 0], [0, 0]])
    np.testing.assert_allclose(O.rel_error(U, X, C), [0.8, 0.0, 1.0, 0.0], atol=1e-15)
    assert list(O.route(np.array([0.8, 0.0, 1.0, 0.0]), np.array([0.0, 0.9, 0.5, 0.0]), 0.85)) \
        == [False, True, True, False]
    assert list(O.route(np.array([0.3, 0.3000001]), np.zeros(2), 0.3)) == [False, True]   # strict


# ---------------------------------------------------------------------------
# write path: positions, routing, compaction, capacity
# ---------------------------------------------------------------------------

def _mixed_rows(U, e_target, rng, d):
    """Rows whose relative error against an exactly orthonormal U is e_target (by construction)."""
    r = U.shape[1]
    rows = []
    P = np.eye(d) - U @ U.T
    for e in e_target:
        a = U @ rng.standard_normal(r)
        b = P @ rng.standard_normal(d)
        a /= np.linalg.norm(a)
        b /= np.linalg.norm(b)
        rows.append(math.sqrt(1 - e * e) * a + e * b)
    return np.array(rows)


def test_compress_routing_and_compaction_by_construction():
    d, r = 16, 4
    U = np.eye(d)[:, [1, 5, 9, 12]] * np.array([1, -1, 1, -1])      # exact in bf16
    rng = np.random.default_rng(5)
    D = _dims(B=2, Hq=2, Hkv=1, d=d, r_k=r, r_v=r, T_cap=64, F_cap=64)
    e_k = np.array([0.1, 0.9, 0.2, 0.6, 0.05, 0.95, 0.3, 0.7])
    e_v = np.array([0.2, 0.1, 0.8, 0.1, 0.05, 0.2, 0.1, 0.1])
    K = _mixed_rows(U, e_k, rng, d)
    V = _mixed_rows(U, e_v, rng, d)
    k_new = np.stack([K, K[::-1]])[:, :, None, :]
    v_new = np.stack([V, V[::-1]])[:, :, None, :]
    cache = O.Cache.empty(D, U[None], U[None])
    cache.seq_len[:] = [3, 30]                     # existing tokens: writes start there
    e, ek, ev = O.compress(cache, k_new, v_new, tau=0.5)
    np.testing.assert_allclose(ek[0, 0], e_k, atol=1e-12)
    np.testing.assert_allclose(ev[0, 0], e_v, atol=1e-12)
    np.testing.assert_allclose(e[1, 0], np.maximum(e_k, e_v)[::-1], atol=1e-12)
    routed0 = [1, 2, 3, 5, 7]                      # max(e_k, e_v) > 0.5
    routed1 = [7 - i for i in routed0][::-1]
    assert list(cache.full_idx[0, 0, :5]) == [3 + i for i in routed0]
    assert list(cache.full_idx[1, 0, :5]) == [30 + i for i in routed1]
    assert list(cache.full_cnt[:, 0]) == [5, 5] and list(cache.seq_len) == [11, 38]
    np.testing.assert_array_equal(cache.full_k[0, 0, :5], K[routed0])
    np.testing.assert_array_equal(cache.full_v[1, 0, :5], V[::-1][routed1])
    # the mask holds exactly the routed positions (row 1 crosses a 32-bit word)
    assert np.flatnonzero(cache.routed(1, 0, np.arange(64))).tolist() == [30 + i for i in routed1]
    # coefficients: U picks signed coordinates, so c is those coordinates, rounded to bf16
    np.testing.assert_array_equal(cache.coef_k[0, 0, 3:11],
                                  O.bf16_round(K[:, [1, 5, 9, 12]] * [1, -1, 1, -1]))
    assert cache.status == 0


def test_compress_capacity_clamps_and_ragged_counts():
    d, r = 8, 2
    U = np.eye(d)[:, :r]
    D = _dims(B=3, Hq=1, Hkv=1, d=d, r_k=r, r_v=r, T_cap=32, F_cap=2)
    rng = np.random.default_rng(6)
    X = rng.standard_normal((3, 6, 1, d))           # random rows: e ~ 0.9, all routed at tau 0.5
    cache = O.Cache.empty(D, U[None], U[None])
    cache.seq_len[:] = [0, 29, 0]
    O.compress(cache, X, X, tau=0.5, t_new_b=[6, 6, 0])
    assert cache.status == (O.FULL_OVERFLOW | O.SEQ_OVERFLOW)
    assert list(cache.seq_len) == [6, 32, 0]        # row 1 clamped at T_cap, row 2 appended nothing
    assert list(cache.full_cnt[:, 0]) == [2, 2, 0]
    assert list(cache.full_idx[0, 0]) == [0, 1] and list(cache.full_idx[1, 0]) == [29, 30]
    # routed tokens that did not fit stay compressed: mask bit clear
    assert np.flatnonzero(cache.routed(0, 0, np.arange(32))).tolist() == [0, 1]
    assert np.flatnonzero(cache.routed(1, 0, np.arange(32))).tolist() == [29, 30]
    # a second call continues at seq_len; appending to a full row only raises SEQ_OVERFLOW
    cache.status = 0
    O.compress(cache, X[:, :1], X[:, :1], tau=2.0)
    assert list(cache.seq_len) == [7, 32, 1] and cache.status == O.SEQ_OVERFLOW


# ---------------------------------------------------------------------------
# read path: decode attention
# ---------------------------------------------------------------------------

def _cache_from(K, V, U_k, U_v, tau, Hq, F_cap=None, T_cap=None):
    """Compress K/V [B,T,Hkv,d] into a fresh oracle cache."""
    B, T, Hkv, d = K.shape
    T_cap = T_cap or max(32, -(-T // 32) * 32)
    D = _dims(B=B, Hq=Hq, Hkv=Hkv, d=d, r_k=U_k.shape[-1], r_v=U_v.shape[-1],
              T_cap=T_cap, F_cap=F_cap or T_cap)
    cache = O.Cache.empty(D, U_k, U_v)
    O.compress(cache, K, V, tau)
    return cache


@pytest.mark.parametrize("Hq,Hkv", [(4, 1), (4, 2), (3, 3)])
def test_identity_basis_is_dense_attention(Hq, Hkv):
    """r = d and U = I: nothing is lost, so the output is textbook dense attention."""
    rng = np.random.default_rng(7)
    B, T, d = 2, 37, 128
    K = O.bf16_round(rng.standard_normal((B, T, Hkv, d)))
    V = O.bf16_round(rng.standard_normal((B, T, Hkv, d)))
    q = O.bf16_round(rng.standard_normal((B, Hq, d)))
    I = np.broadcast_to(np.eye(d), (Hkv, d, d))
    cache = _cache_from(K, V, I, I, tau=0.3, Hq=Hq)
    assert cache.full_cnt.sum() == 0
    ref = _sdpa(q, K.transpose(0, 2, 1, 3), V.transpose(0, 2, 1, 3), Hq // Hkv)
    np.testing.assert_allclose(O.decode_attn(cache, q), ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(O.decode_attn_coef(cache, q), ref, rtol=1e-12, atol=1e-13)


def test_span_inputs_are_exact():
    """K, V inside span(U) with U a signed column subset of I: e = 0 and exact output."""
    rng = np.random.default_rng(8)
    B, T, Hkv, Hq, d, r = 1, 45, 2, 8, 128, 32
    cols = [rng.choice(d, r, replace=False) for _ in range(Hkv)]
    U = np.zeros((Hkv, d, r))
    for h in range(Hkv):
        U[h, cols[h], np.arange(r)] = rng.choice([-1.0, 1.0], r)
    K = np.zeros((B, T, Hkv, d))
    V = np.zeros((B, T, Hkv, d))
    for h in range(Hkv):
        K[:, :, h, cols[h]] = O.bf16_round(rng.standard_normal((B, T, r)))
        V[:, :, h, cols[h]] = O.bf16_round(rng.standard_normal((B, T, r)))
    q = O.bf16_round(rng.standard_normal((B, Hq, d)))
    cache = _cache_from(K, V, U, U, tau=1e-9, Hq=Hq)
    assert cache.full_cnt.sum() == 0
    ref = _sdpa(q, K.transpose(0, 2, 1, 3), V.transpose(0, 2, 1, 3), Hq // Hkv)
    np.testing.assert_allclose(O.decode_attn(cache, q), ref, rtol=1e-12, atol=1e-13)


def test_mixed_cache_equals_dense_attention():
    """Both token sets at once, against a library routine: tokens whose K and V lie
    in span(U) (U a signed column subset of I, so c and the reconstruction are exact
    in bf16) stay compressed; the other tokens are off the span (error well above
    tau) and go to the full-rank list.  The oracle's decode over that mixed cache
    must be dense attention over the raw K, V -- a wrong joint softmax, a lost
    full-rank row or a misplaced one would break it."""
    rng = np.random.default_rng(18)
    B, T, Hkv, Hq, d, r = 2, 77, 2, 8, 128, 32
    cols = [rng.choice(d, r, replace=False) for _ in range(Hkv)]
    U = np.zeros((Hkv, d, r))
    for h in range(Hkv):
        U[h, cols[h], np.arange(r)] = rng.choice([-1.0, 1.0], r)
    K = O.bf16_round(rng.standard_normal((B, T, Hkv, d)))
    V = O.bf16_round(rng.standard_normal((B, T, Hkv, d)))
    in_span = rng.random((B, T, Hkv)) < 0.6
    for b in range(B):
        for h in range(Hkv):
            off = np.setdiff1d(np.arange(d), cols[h])
            for t in np.flatnonzero(in_span[b, :, h]):
                K[b, t, h, off] = 0.0
                V[b, t, h, off] = 0.0
    q = O.bf16_round(rng.standard_normal((B, Hq, d)))
    cache = _cache_from(K, V, U, U, tau=0.5, Hq=Hq)
    for b in range(B):
        for h in range(Hkv):
            routed = cache.routed(b, h, np.arange(T))
            assert np.array_equal(routed, ~in_span[b, :, h])
            assert 0 < routed.sum() < T
    ref = _sdpa(q, K.transpose(0, 2, 1, 3), V.transpose(0, 2, 1, 3), Hq // Hkv)
    np.testing.assert_allclose(O.decode_attn(cache, q), ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(O.decode_attn_coef(cache, q), ref, rtol=1e-12, atol=1e-13)


def test_negative_tau_routes_everything_and_attends_raw_rows():
    rng = np.random.default_rng(9)
    B, T, Hkv, Hq, d = 1, 50, 1, 4, 128
    U = _random_orthonormal(d, 32, rng)[None]
    K = O.bf16_round(rng.standard_normal((B, T, Hkv, d)))
    V = O.bf16_round(rng.standard_normal((B, T, Hkv, d)))
    q = O.bf16_round(rng.standard_normal((B, Hq, d)))
    cache = _cache_from(K, V, U, U, tau=-1.0, Hq=Hq)
    assert cache.full_cnt[0, 0] == T and list(cache.full_idx[0, 0, :T]) == list(range(T))
    ref = _sdpa(q, K.transpose(0, 2, 1, 3), V.transpose(0, 2, 1, 3), Hq // Hkv)
    np.testing.assert_allclose(O.decode_attn(cache, q), ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(O.decode_attn_coef(cache, q), ref, rtol=1e-12, atol=1e-13)


def test_tau_above_one_routes_nothing():
    rng = np.random.default_rng(10)
    U = _random_orthonormal(128, 16, rng)[None]
    K = rng.standard_normal((1, 40, 1, 128))       # e close to 1 for random rows
    cache = _cache_from(K, K, U, U, tau=1.5, Hq=1)
    assert cache.full_cnt.sum() == 0 and cache.route_mask.sum() == 0


def test_softmax_rows_sum_to_one():
    """All value rows equal to w in span(U_v): the output is w whatever q and K are."""
    rng = np.random.default_rng(11)
    d, r, T = 128, 32, 70
    U = np.zeros((1, d, r))
    U[0, np.arange(r) * 4, np.arange(r)] = 1.0
    w = np.zeros(d)
    w[np.arange(r) * 4] = O.bf16_round(rng.standard_normal(r))
    K = O.bf16_round(3 * rng.standard_normal((1, T, 1, d)))
    off_span = np.setdiff1d(np.arange(d), np.arange(r) * 4)
    K[0, ::2, 0, off_span[:, None]] = 0.0            # even tokens lie in span(U_k): compressed
    V = np.broadcast_to(w, (1, T, 1, d)).copy()
    q = O.bf16_round(rng.standard_normal((1, 4, d)))
    cache = _cache_from(K, V, U, U, tau=0.5, Hq=4)
    assert 0 < cache.full_cnt[0, 0] < T                # both token sets take part
    out = O.decode_attn(cache, q)
    np.testing.assert_allclose(out, np.broadcast_to(w, out.shape), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(O.decode_attn_coef(cache, q), out, rtol=1e-12, atol=1e-14)


def test_softmax_lipschitz_bound():
    """NOVA-KV summary, key transform derivation: ||p - p_hat|| <= ||q (K - K_hat)^T|| / (2 sqrt d)."""
    rng = np.random.default_rng(12)
    d, T = 128, 300
    for trial in range(5):
        U = _random_orthonormal(d, 24 + 8 * trial, rng)[None]
        K = O.bf16_round(rng.standard_normal((1, T, 1, d)) * 2)
        cache = _cache_from(K, K, U, U, tau=0.97, Hq=1)
        q = O.bf16_round(rng.standard_normal(d) * 2)
        K_hat, _ = O.effective_kv(cache, 0, 0)
        p = O.softmax(K[0, :, 0] @ q / math.sqrt(d))
        p_hat = O.softmax(K_hat @ q / math.sqrt(d))
        bound = np.linalg.norm((K[0, :, 0] - K_hat) @ q) / (2 * math.sqrt(d))
        assert np.linalg.norm(p - p_hat) <= bound * (1 + 1e-12)
        assert np.linalg.norm(p - p_hat) > 0


def test_single_token_returns_its_value_row():
    rng = np.random.default_rng(13)
    U = _random_orthonormal(128, 32, rng)[None]
    V = O.bf16_round(rng.standard_normal((1, 1, 1, 128)))
    K = O.bf16_round(rng.standard_normal((1, 1, 1, 128)))
    q = O.bf16_round(rng.standard_normal((1, 2, 128)))
    c_full = _cache_from(K, V, U, U, tau=0.5, Hq=2)                # random row: routed
    np.testing.assert_allclose(O.decode_attn(c_full, q)[0], np.broadcast_to(V[0, 0, 0], (2, 128)),
                               rtol=1e-15)
    c_comp = _cache_from(K, V, U, U, tau=2.0, Hq=2)                # kept compressed
    v_hat = U[0] @ O.bf16_round(U[0].T @ V[0, 0, 0])
    np.testing.assert_allclose(O.decode_attn(c_comp, q)[0], np.broadcast_to(v_hat, (2, 128)),
                               rtol=1e-13, atol=1e-15)


def test_hand_worked_two_token_attention():
    """Logits 0 and ln 3 give p = (1/4, 3/4); values (4,0,0,0), (0,4,0,0) give o = (1, 3, 0, 0)."""
    d = 4
    U = np.eye(d)[:, :2][None]
    K = np.array([[0.0, 1, 0, 0], [1.0, 0, 0, 0]])[None, :, None, :]
    V = np.array([[4.0, 0, 0, 0], [0, 4.0, 0, 0]])[None, :, None, :]
    q = np.array([[[2 * math.log(3), 0, 0, 0]]])
    for tau in (-1.0, 2.0):                       # all full rank / all compressed (exact here)
        cache = _cache_from(K, V, U, U, tau=tau, Hq=1)
        np.testing.assert_allclose(O.decode_attn(cache, q)[0, 0], [1, 3, 0, 0], rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(O.decode_attn_coef(cache, q)[0, 0], [1, 3, 0, 0], rtol=1e-14,
                                   atol=1e-15)


def test_empty_sequence_outputs_zero():
    U = np.eye(128)[:, :16][None]
    cache = O.Cache.empty(_dims(B=2, Hq=2, Hkv=1, r_k=16, r_v=16), U, U)
    q = np.ones((2, 2, 128))
    assert not O.decode_attn(cache, q).any() and not O.decode_attn_coef(cache, q).any()


def test_coefficient_space_equals_reconstruct_then_attend():
    """q.(U c) = (U^T q).c: the two oracle read paths agree on a mixed cache."""
    rng = np.random.default_rng(14)
    B, T, Hkv, Hq, d = 2, 97, 2, 8, 128
    Qk = np.stack([_random_orthonormal(d, d, rng) for _ in range(Hkv)])
    Qv = np.stack([_random_orthonormal(d, d, rng) for _ in range(Hkv)])
    U_k = O.bf16_round(Qk[:, :, :48])
    U_v = O.bf16_round(Qv[:, :, :80])
    Z = rng.standard_normal((B, T, Hkv, 64)) * np.arange(1, 65) ** -0.5
    K = O.bf16_round(np.einsum("bthi,hdi->bthd", Z, Qk[:, :, :64]) + 0.02 * rng.standard_normal((B, T, Hkv, d)))
    V = O.bf16_round(np.einsum("bthi,hdi->bthd", Z, Qv[:, :, :64]) + 0.02 * rng.standard_normal((B, T, Hkv, d)))
    q = O.bf16_round(rng.standard_normal((B, Hq, d)))
    cache = _cache_from(K, V, U_k, U_v, tau=0.2, Hq=Hq)
    assert 0 < cache.full_cnt.sum() < B * Hkv * T
    a = O.decode_attn(cache, q)
    b = O.decode_attn_coef(cache, q)
    assert np.abs(a - b).max() <= 1e-12 * np.abs(a).max()


# ---- the offline basis (StaticPCA; Frobenius-optimal subspace) --------------------------

def _calib_rows(seed, N=600, d=32, rank_sig=12, noise=0.05):
    rng = np.random.default_rng(seed)
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    Z = rng.standard_normal((N, rank_sig)) * (np.arange(1, rank_sig + 1) ** -0.5)
    return Z @ Q[:, :rank_sig].T + noise * rng.standard_normal((N, d))


def test_fit_basis_matches_svd_and_eckart_young():
    """Against numpy's SVD of X (another library routine): singular values squared are
    the eigenvalues, the right singular vectors span the same subspace; the residual
    sum of squares equals the discarded eigenvalue mass."""
    X = _calib_rows(1)
    r = 8
    U, lam = O.fit_basis(X, r)
    _, sv, Vt = np.linalg.svd(X, full_matrices=False)
    assert np.allclose(lam[:len(sv)], sv ** 2, rtol=1e-10, atol=1e-9)
    P, Ps = U @ U.T, Vt[:r].T @ Vt[:r]
    assert np.abs(P - Ps).max() < 1e-10
    resid = ((X - X @ U @ U.T) ** 2).sum()
    assert abs(resid - lam[r:].sum()) <= 1e-10 * lam.sum()
    assert np.allclose(U.T @ U, np.eye(r), atol=1e-12)
    G = X.T @ X
    assert np.allclose(G @ U, U * lam[:r], atol=1e-9 * lam[0])


def test_fit_basis_beats_every_other_basis_and_sign_convention():
    """No other r-dim orthonormal basis has a smaller residual (random trials), and
    each column's largest-magnitude entry is positive."""
    X = _calib_rows(2)
    r = 6
    U, lam = O.fit_basis(X, r)
    best = ((X - X @ U @ U.T) ** 2).sum()
    rng = np.random.default_rng(3)
    for _ in range(50):
        Q, _ = np.linalg.qr(rng.standard_normal((X.shape[1], r)))
        assert ((X - X @ Q @ Q.T) ** 2).sum() >= best - 1e-9
    for j in range(r):
        i = int(np.argmax(np.abs(U[:, j])))
        assert U[i, j] > 0


def test_fit_basis_exact_low_rank_data():
    """Rows exactly in a rank-r span: the basis spans it and the rest of the spectrum is 0."""
    rng = np.random.default_rng(4)
    d, r = 16, 5
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    X = rng.standard_normal((200, r)) @ Q[:, :r].T
    U, lam = O.fit_basis(X, r)
    assert np.abs(U @ U.T - Q[:, :r] @ Q[:, :r].T).max() < 1e-10
    assert np.abs(lam[r:]).max() < 1e-9 * lam[0]


def test_rank_for_budget_worked_by_hand():
    """Spectrum 8, 4, 2, 1, 1 (total 16): discarded mass after r = 1..5 is 8, 4, 2, 1, 0."""
    lam = [8.0, 4.0, 2.0, 1.0, 1.0]
    assert O.rank_for_budget(lam, 0.5) == 1        # 8 <= 8
    assert O.rank_for_budget(lam, 0.49) == 2       # 4 <= 7.84
    assert O.rank_for_budget(lam, 0.125) == 3      # 2 <= 2, boundary inclusive
    assert O.rank_for_budget(lam, 0.1) == 4        # 2 > 1.6, 1 <= 1.6
    assert O.rank_for_budget(lam, 0.0) == 5
    assert O.rank_for_budget(lam, 1.0) == 1
    assert O.rank_for_budget([0.0, 0.0, 0.0], 0.0) == 1
    # a negative eigenvalue from rounding counts as zero
    assert O.rank_for_budget([3.0, 1.0, -1e-12], 0.0) == 2


def test_rank_for_budget_is_the_eckart_young_rank():
    """The chosen rank's projection residual, computed directly from the rows, is
    within the budget and one rank less is not (Eckart-Young: the discarded mass
    is the best rank-r residual)."""
    X = _calib_rows(5)
    total = (X ** 2).sum()
    for budget in (0.3, 0.1, 0.05, 0.02, 0.01, 0.004):
        U, lam = O.fit_basis(X, X.shape[1])
        r = O.rank_for_budget(lam, budget)
        res = lambda k: ((X - X @ U[:, :k] @ U[:, :k].T) ** 2).sum() / total
        assert res(r) <= budget + 1e-12
        if r > 1:
            assert res(r - 1) > budget - 1e-12


def test_rank_for_budget_monotone_and_exact_rank():
    rng = np.random.default_rng(6)
    lam = np.sort(rng.gamma(0.5, 1.0, 64))[::-1]
    ranks = [O.rank_for_budget(lam, b) for b in np.linspace(0.0, 1.0, 101)]
    assert all(a >= b for a, b in zip(ranks, ranks[1:]))
    assert ranks[0] == 64 and ranks[-1] == 1
    # rows exactly in a rank-5 span: any small budget gives 5
    d, k = 16, 5
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    X = rng.standard_normal((200, k)) @ Q[:, :k].T
    _, lam = O.fit_basis(X, d)
    assert O.rank_for_budget(lam, 1e-9) == k
