"""Quantised coefficients: per-vector scaled int8 / int4 codes of the stored
coefficient rows, and decode attention over them (fp64 CPU oracle).

Test infrastructure, under the same rules as ``lrkv_oracle``: only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import it; the CUDA library never does.

What it follows
---------------
* KVQuant record ("Quant method", "Methodology"): sub-8-bit KV storage with a
  per-vector scale, whose overhead is counted in the average bit width.
* NOVA-KV summary ("Introduction", requirements 2 and 3): the cache is read
  at every decoding step, so the read path must stay cheap, and every token
  must occupy the same number of bits (a fixed-width layout); the
  quantiser acts on transform coefficients and is judged by MSE.
Here the transform is the low-rank basis itself: each stored coefficient row
(c_k or c_v of one token and kv head) is quantised on its own.

Reading R21 (the pages fix no scheme): symmetric, uniform, absmax-scaled.
With Q = 127 (8 bits) or 7 (4 bits) and the row c as stored (bf16 values):
    s   = max_j |c_j| / Q                  fp32, correctly rounded
    q_j = round_half_even(c_j / s)         fp32 division, clamped to [-Q, Q]
    s = 0 (an all-zero row) gives q = 0
    c_hat_j = s * q_j
Every step that decides an integer is IEEE fp32 (no flush to zero), so a
kernel doing the same operations takes the same decisions.  4-bit codes are
stored two per byte, element 2i in the low nibble (two's complement).
Decode over the codes: logit_t = s_k,t (q~ . q_k,t) / sqrt(d) for compressed
tokens, o = U_v sum_t (p_t s_v,t) q_v,t + sum_F p_t v_t -- the plain decode
of ``lrkv_oracle`` run on the dequantised rows c_hat.
"""
import numpy as np

from .lrkv_oracle import Cache, decode_attn, softmax

QMAX = {8: 127, 4: 7}


def quantize_coef(c, bits):
    """Per-row codes and scales of coefficient rows c [..., r] (bf16 values).

    Returns (q int8 [..., r], s float32 [...]) following reading R21.
    """
    Q = np.float32(QMAX[bits])
    c32 = np.asarray(c, np.float64).astype(np.float32)     # exact: bf16 values
    amax = np.abs(c32).max(axis=-1) if c32.shape[-1] else np.zeros(c32.shape[:-1], np.float32)
    s = (amax / Q).astype(np.float32)
    q = np.zeros(c32.shape, np.int8)
    nz = s > 0
    t = c32[nz] / s[nz][..., None]                          # float32 / float32
    q[nz] = np.clip(np.rint(t), -Q, Q).astype(np.int8)      # rint: half to even
    return q, s


def dequantize_coef(q, s):
    """c_hat = s q (float64)."""
    return np.asarray(q, np.float64) * np.asarray(s, np.float64)[..., None]


def pack_int4(q):
    """[..., r] codes in [-8, 7] (r even) -> uint8 [..., r/2], element 2i low nibble."""
    q = np.asarray(q, np.int8)
    if q.shape[-1] % 2:
        raise ValueError("an even number of 4-bit codes is packed")
    u = (q.astype(np.int16) & 0xF).astype(np.uint8)
    return (u[..., 0::2] | (u[..., 1::2] << 4)).astype(np.uint8)


def unpack_int4(p):
    """Inverse of pack_int4: uint8 [..., r/2] -> int8 [..., r] (sign-extended nibbles)."""
    p = np.asarray(p, np.uint8)
    lo = (p & 0xF).astype(np.int16)
    hi = (p >> 4).astype(np.int16)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), np.int16)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return np.where(out > 7, out - 16, out).astype(np.int8)


def quantize_cache(cache, bits):
    """Codes and scales of every stored coefficient row of a cache.

    Returns dict(qk [B,Hkv,T_cap,r_k] int8, sk [B,Hkv,T_cap] f32, qv, sv).
    Rows past seq_len are quantised too (they hold zeros in a fresh cache).
    """
    qk, sk = quantize_coef(cache.coef_k, bits)
    qv, sv = quantize_coef(cache.coef_v, bits)
    return dict(qk=qk, sk=sk, qv=qv, sv=sv)


def dequantized_cache(cache, codes):
    """A copy of ``cache`` whose coefficient rows are the dequantised codes."""
    return Cache(dims=cache.dims, U_k=cache.U_k, U_v=cache.U_v, U_kq=cache.U_kq, mu_k=cache.mu_k,
                 coef_k=dequantize_coef(codes["qk"], codes["sk"]),
                 coef_v=dequantize_coef(codes["qv"], codes["sv"]),
                 route_mask=cache.route_mask, full_idx=cache.full_idx, full_k=cache.full_k,
                 full_v=cache.full_v, full_cnt=cache.full_cnt, seq_len=cache.seq_len,
                 status=cache.status)


def decode_attn_quant(cache, codes, q):
    """Decode over quantised coefficients, plain definition: dequantise the
    rows, then the reconstruct-and-attend decode of ``lrkv_oracle``."""
    return decode_attn(dequantized_cache(cache, codes), q)


def decode_attn_quant_coef(cache, codes, q):
    """The same decode in code space, as a kernel would run it: integer codes
    times per-row scales, the value scales folded into the weights.

    logit_t = s_k,t (q~ . q_k,t) / sqrt(d) (compressed t), q . k_t / sqrt(d)
    (full-rank t); one softmax; o = U_v sum_C (p_t s_v,t) q_v,t + sum_F p_t v_t.
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
            comp = ~cache.routed(b, kvh, pos)
            n_full = int(cache.full_cnt[b, kvh])
            Fk = cache.full_k[b, kvh, :n_full]
            Fv = cache.full_v[b, kvh, :n_full]
            Qk = codes["qk"][b, kvh, :T][comp].astype(np.float64)
            Sk = codes["sk"][b, kvh, :T][comp].astype(np.float64)
            Qv = codes["qv"][b, kvh, :T][comp].astype(np.float64)
            Sv = codes["sv"][b, kvh, :T][comp].astype(np.float64)
            for h in range(kvh * D.g, (kvh + 1) * D.g):
                q_t = cache.key_rec_basis(kvh).T @ q[b, h]
                bias = q[b, h] @ cache.key_mean(kvh)
                s = np.concatenate([Sk * (Qk @ q_t) + bias, Fk @ q[b, h]]) / np.sqrt(D.d)
                p = softmax(s)
                pc, pf = p[:len(Sk)], p[len(Sk):]
                out[b, h] = cache.U_v[kvh] @ ((pc * Sv) @ Qv) + pf @ Fv
    return out


def quant_bytes_per_token(r_k, r_v, bits):
    """Stored bytes of one token's coefficients per kv head: the codes plus one
    fp32 scale for keys and one for values (the fixed-width row)."""
    return (r_k + r_v) * bits // 8 + 8
