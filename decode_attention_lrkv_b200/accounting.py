"""Byte accounting for the compressed cache and its kernels (host logic).

These are the algorithmic byte counts that the measurements divide by the
kernels' durations: the bytes a kernel must move at minimum, not what it
happens to move.  The dense-cache formula is the one the KVQuant record
("KV bytes basis" field) and the Llama-3.1-NovaKV card (Results table,
"Cache, KB/token") use: layers x kv heads x head dim x 2 (K and V) x bytes.
"""
import math

BF16 = 2
FP32 = 4
INT32 = 4


def dense_kv_bytes_per_token(layers, kv_heads, d, elem_bytes=BF16):
    """Bytes one token takes in a dense K+V cache."""
    return layers * kv_heads * d * 2 * elem_bytes


def compressed_bytes_per_token_head(r_k, r_v, elem_bytes=BF16, coef_bits=16):
    """Coefficient bytes of one compressed token in one kv head: (r_k + r_v) values
    (bf16), or their codes plus one fp32 scale for keys and one for values
    (coef_bits 8 or 4)."""
    if coef_bits in (0, 16):
        return (r_k + r_v) * elem_bytes
    return (r_k + r_v) * coef_bits // 8 + 2 * FP32


def full_row_bytes(d, elem_bytes=BF16):
    """Bytes of one full-rank token in one kv head: its key row, value row and list index."""
    return 2 * d * elem_bytes + INT32


def decode_bytes(B, Hq, Hkv, d, r_k, r_v, lengths, full_cnt, coef_bits=16):
    """Algorithmic bytes of one decode-attention call over one layer.

    lengths: B sequence lengths; full_cnt: B x Hkv routed-token counts.
    Per (b, kv head): the coefficient rows of the compressed tokens, the key
    and value rows of the full-rank tokens (their list index is not needed
    to attend), and the route-mask words of the sequence.  Per kv head, the
    basis U_k, U_v once.  Plus the query (bf16) and the output (fp32).
    """
    total = 0
    for b in range(B):
        T = int(lengths[b])
        for h in range(Hkv):
            F = int(full_cnt[b][h])
            total += (T - F) * compressed_bytes_per_token_head(r_k, r_v, coef_bits=coef_bits)
            total += F * 2 * d * BF16
            total += math.ceil(T / 32) * 4
    total += Hkv * d * (r_k + r_v) * BF16
    total += B * Hq * d * (BF16 + FP32)
    return total


def compress_bytes(Hkv, d, r_k, r_v, n_tokens, n_routed, coef_bits=16):
    """Algorithmic bytes of compressing n_tokens positions (summed over batch rows).

    Each (token, kv head) reads its key and value rows and writes its
    coefficients (or codes and scales) and its mask bit; each routed (token,
    kv head) also writes its key and value rows and list index.  The basis is
    read once per kv head.
    """
    per_tok = Hkv * (2 * d * BF16 + compressed_bytes_per_token_head(r_k, r_v, coef_bits=coef_bits)) \
        + Hkv / 8.0
    return int(n_tokens * per_tok + n_routed * full_row_bytes(d) + Hkv * d * (r_k + r_v) * BF16)


def compress_tc_flops(Hkv, d, r_k, r_v, n_tokens):
    """Tensor-core flops the prefill projection executes per call.

    Per (token, kv head) and tensor: c = U^T x (2 d r) and the residual
    P x = (P_hi + P_lo) x with P = I - U U^T (2 * 2 d^2); the once-per-CTA
    U U^T products are not counted.
    """
    return int(n_tokens * Hkv * (2 * d * (r_k + r_v) + 2 * 4 * d * d))
