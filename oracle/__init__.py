"""fp64 CPU oracle for low-rank compressed-KV decode attention.

Test infrastructure only: ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arm may import it; the CUDA library
and its Python binding never do.
"""
from .bf16 import bf16_round, bf16_bits, bf16_from_bits, bf16_ulp
from .lrkv_oracle import (Dims, Cache, project, reconstruct, rel_error, route, fit_basis, rank_for_budget,
                          compress, effective_kv, softmax, decode_attn,
                          decode_attn_coef, FULL_OVERFLOW, SEQ_OVERFLOW)
from .coef_quant import (QMAX, quantize_coef, dequantize_coef, pack_int4, unpack_int4,
                         quantize_cache, dequantized_cache, decode_attn_quant,
                         decode_attn_quant_coef, quant_bytes_per_token)
from .attn_aware import KeyTransform, key_transform, weighted_key_error
from .oja import oja_direction, oja_step, oja_stream
