"""Pins of the quantised-coefficient oracle (oracle/coef_quant.py).

Independent of the oracle's own code: values worked out by hand, brute force
over every code, exact algebraic invariants of a symmetric absmax quantiser,
and the plain decode of the unquantised oracle where quantisation is exact.
"""
import numpy as np
import pytest

import oracle as O


def _dims(B=1, Hq=4, Hkv=1, d=128, r_k=32, r_v=32, T_cap=64, F_cap=64):
    return O.Dims(B=B, Hq=Hq, Hkv=Hkv, d=d, r_k=r_k, r_v=r_v, T_cap=T_cap, F_cap=F_cap)


def test_round_half_even_worked_by_hand():
    """Scale 1 exactly (max |c| = Q): codes are c rounded to nearest, ties to even."""
    q, s = O.quantize_coef(np.array([127, -63.5, 31.75, 0, -127, 2.5, -0.5, 1.5, 0.25]), 8)
    assert s == np.float32(1.0)
    assert q.tolist() == [127, -64, 32, 0, -127, 2, 0, 2, 0]
    q, s = O.quantize_coef(np.array([7, -3.5, 2.5, 0.5, -7, 1.25]), 4)
    assert s == np.float32(1.0)
    assert q.tolist() == [7, -4, 2, 0, -7, 1]
    # scale 2^-3: the same codes for the row divided by 8
    q, s = O.quantize_coef(np.array([127, -63.5, 31.75]) / 8, 8)
    assert s == np.float32(0.125) and q.tolist() == [127, -64, 32]


def test_int4_packing():
    """Element 2i in the low nibble, two's complement: [1, -1, 7, -7] -> 0xF1, 0x97."""
    assert O.pack_int4(np.array([1, -1, 7, -7])).tolist() == [0xF1, 0x97]
    a, b = np.meshgrid(np.arange(-8, 8), np.arange(-8, 8))
    codes = np.stack([a.ravel(), b.ravel()], axis=-1).astype(np.int8)
    assert np.array_equal(O.unpack_int4(O.pack_int4(codes)), codes)
    with pytest.raises(ValueError):
        O.pack_int4(np.zeros(3, np.int8))


@pytest.mark.parametrize("bits", [8, 4])
def test_codes_are_the_nearest_grid_points(bits):
    """Brute force: each code is the integer in [-Q, Q] whose grid point s*q is
    nearest to c (the larger |.| never wins a tie over the even one), the row's
    largest magnitude maps to +-Q, and every code is in range."""
    Q = O.QMAX[bits]
    rng = np.random.default_rng(bits)
    c = O.bf16_round(rng.standard_normal((200, 16)) * rng.uniform(0.01, 10.0, (200, 1)))
    q, s = O.quantize_coef(c, bits)
    grid = np.arange(-Q, Q + 1)
    for i in range(c.shape[0]):
        t = c[i].astype(np.float32) / s[i]                 # the fp32 quotient of the definition
        dist = np.abs(t.astype(np.float64)[:, None] - grid[None, :])
        best = dist.min(axis=1)
        chosen = np.abs(t.astype(np.float64) - q[i])
        assert np.all(chosen == best)
        ties = (np.sum(dist == best[:, None], axis=1) > 1)
        assert np.all(q[i][ties] % 2 == 0)
        j = int(np.argmax(np.abs(c[i])))
        assert abs(int(q[i, j])) == Q
    assert np.abs(q).max() <= Q


@pytest.mark.parametrize("bits", [8, 4])
def test_error_bound_symmetry_and_scale_invariance(bits):
    rng = np.random.default_rng(20 + bits)
    c = O.bf16_round(rng.standard_normal((64, 48)) * 3.0)
    q, s = O.quantize_coef(c, bits)
    c_hat = O.dequantize_coef(q, s)
    # |c - s q| <= s/2, up to the fp32 rounding of the quotient c/s (|c/s| <= Q,
    # one rounding of relative size 2^-24 can move a value just below a tie onto it)
    slack = 0.5 + O.QMAX[bits] * 2.0 ** -23
    assert np.all(np.abs(c - c_hat) <= s[:, None].astype(np.float64) * slack)
    assert np.all(s == np.abs(c).max(axis=1).astype(np.float32) / np.float32(O.QMAX[bits]))
    qn, sn = O.quantize_coef(-c, bits)
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)
    for k in (-6, 3):
        qk, sk = O.quantize_coef(c * 2.0 ** k, bits)
        assert np.array_equal(qk, q) and np.array_equal(sk, s * np.float32(2.0 ** k))
    qz, sz = O.quantize_coef(np.zeros((3, 8)), bits)
    assert not qz.any() and not sz.any()
    assert not O.dequantize_coef(qz, sz).any()


def _cache_with_rows(Ck, Cv, U_k, U_v, Hq):
    """An oracle cache [B=1] holding the given coefficient rows, none routed."""
    Hkv, T, r_k = Ck.shape
    r_v = Cv.shape[-1]
    d = U_k.shape[1]
    T_cap = -(-T // 32) * 32
    cache = O.Cache.empty(_dims(Hq=Hq, Hkv=Hkv, d=d, r_k=r_k, r_v=r_v, T_cap=T_cap, F_cap=T_cap),
                          U_k, U_v)
    cache.coef_k[0, :, :T] = Ck
    cache.coef_v[0, :, :T] = Cv
    cache.seq_len[0] = T
    return cache


def _orth(d, r, rng):
    return np.linalg.qr(rng.standard_normal((d, d)))[0][:, :r]


@pytest.mark.parametrize("bits", [8, 4])
def test_rows_on_the_grid_decode_exactly(bits):
    """Rows that are exactly s * q with max |q| = Q (power-of-two s) come back as
    those codes, and the quantised decode equals the plain unquantised decode."""
    Q = O.QMAX[bits]
    rng = np.random.default_rng(30 + bits)
    Hkv, T, r, d = 2, 40, 32, 128
    def rows():
        q = rng.integers(-Q, Q + 1, (Hkv, T, r))
        q[..., 0] = Q * rng.choice([-1, 1], (Hkv, T))
        return q, 2.0 ** rng.integers(-8, 3, (Hkv, T))
    qk, sk = rows()
    qv, sv = rows()
    Ck, Cv = qk * sk[..., None], qv * sv[..., None]
    U_k = np.stack([_orth(d, r, rng) for _ in range(Hkv)])
    U_v = np.stack([_orth(d, r, rng) for _ in range(Hkv)])
    cache = _cache_with_rows(Ck, Cv, U_k, U_v, Hq=8)
    codes = O.quantize_cache(cache, bits)
    assert np.array_equal(codes["qk"][0, :, :T], qk) and np.array_equal(codes["sk"][0, :, :T], sk)
    assert np.array_equal(codes["qv"][0, :, :T], qv) and np.array_equal(codes["sv"][0, :, :T], sv)
    qry = O.bf16_round(rng.standard_normal((1, 8, d)))
    ref = O.decode_attn(cache, qry)
    np.testing.assert_allclose(O.decode_attn_quant(cache, codes, qry), ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(O.decode_attn_quant_coef(cache, codes, qry), ref, rtol=1e-12,
                               atol=1e-13)


@pytest.mark.parametrize("bits,Hq,Hkv", [(8, 4, 1), (4, 8, 2), (8, 6, 3)])
def test_code_space_decode_equals_dequantise_then_decode(bits, Hq, Hkv):
    """Two writings of the quantised decode: per-row scales applied to integer codes
    (logits and folded into the value weights) against dequantise-then-attend, on a
    cache with compressed and full-rank tokens."""
    rng = np.random.default_rng(40 + bits + Hq)
    B, T, d, r_k, r_v = 2, 70, 128, 32, 48
    U_k = np.stack([_orth(d, r_k, rng) for _ in range(Hkv)])
    U_v = np.stack([_orth(d, r_v, rng) for _ in range(Hkv)])
    K = O.bf16_round(rng.standard_normal((B, T, Hkv, d)))
    V = O.bf16_round(rng.standard_normal((B, T, Hkv, d)))
    cache = O.Cache.empty(_dims(B=B, Hq=Hq, Hkv=Hkv, d=d, r_k=r_k, r_v=r_v, T_cap=96, F_cap=96),
                          U_k, U_v)
    O.compress(cache, K, V, tau=0.84)
    assert 0 < cache.full_cnt.sum() < B * Hkv * T
    codes = O.quantize_cache(cache, bits)
    qry = O.bf16_round(rng.standard_normal((B, Hq, d)))
    a = O.decode_attn_quant(cache, codes, qry)
    b = O.decode_attn_quant_coef(cache, codes, qry)
    np.testing.assert_allclose(b, a, rtol=1e-11, atol=1e-12)
    # the codes do change the output (the test would not see a dropped scale otherwise)
    assert np.abs(a - O.decode_attn(cache, qry)).max() > 1e-6


def test_full_rank_tokens_ignore_the_codes():
    """Every token routed (tau < 0): the codes are never read and the output is the
    unquantised one exactly."""
    rng = np.random.default_rng(50)
    B, T, Hkv, Hq, d, r = 1, 33, 2, 4, 128, 32
    U = np.stack([_orth(d, r, rng) for _ in range(Hkv)])
    K = O.bf16_round(rng.standard_normal((B, T, Hkv, d)))
    V = O.bf16_round(rng.standard_normal((B, T, Hkv, d)))
    cache = O.Cache.empty(_dims(B=B, Hq=Hq, Hkv=Hkv, d=d, r_k=r, r_v=r, T_cap=64, F_cap=64), U, U)
    O.compress(cache, K, V, tau=-1.0)
    assert (cache.full_cnt == T).all()
    qry = O.bf16_round(rng.standard_normal((B, Hq, d)))
    ref = O.decode_attn(cache, qry)
    for bits in (8, 4):
        codes = O.quantize_cache(cache, bits)
        np.testing.assert_allclose(O.decode_attn_quant(cache, codes, qry), ref, rtol=1e-13, atol=0)
        np.testing.assert_allclose(O.decode_attn_quant_coef(cache, codes, qry), ref, rtol=1e-12,
                                   atol=1e-13)


def test_bytes_per_token():
    """Fixed-width rows: codes plus one fp32 scale per tensor (64/96 ranks: 320 B in bf16)."""
    assert O.quant_bytes_per_token(64, 96, 8) == 168
    assert O.quant_bytes_per_token(64, 96, 4) == 88
    assert O.quant_bytes_per_token(48, 80, 4) == 72
