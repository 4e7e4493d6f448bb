// Parameters of the decode kernels (plain decode, and decode with a fused
// decode-time append).
#pragma once

#include "lrkv_common.cuh"

namespace lrkv {

struct DecodeParams {
  lrkv_dims D;
  lrkv_cache C;
  const lrkv_bf16* q;
  float* out;
  int32_t* tickets;   // [B][Hkv]
  float* partials;    // [B][Hkv][n_chunk_max][g][4 + r_v + d]
  int n_split;        // splits per (b, kv head) in the plain decode's grid (those of a full cache)
  // records per (b, kv head), and the fused call's grid: its last CTA appends,
  // the others hold at least the fewest splits any cached length needs
  int n_chunk_max;
  // query heads per kv head (Hq / Hkv), and the first of this launch's: the
  // streaming kernel serves up to its template's G of them per launch
  int g_all;
  int g_off;
  int num_sms;        // SMs of the device: each CTA sizes its split from the live length
  // fused decode-time append (lrkv_append_decode_attn); k_new null: plain decode
  const lrkv_bf16* k_new;   // [B][1][Hkv][d]
  const lrkv_bf16* v_new;   // [B][1][Hkv][d]
  const int32_t* t_new_b;   // [B] tokens of row b (0 or 1), nullable: 1 for every row
  float tau;
  float* err_out;           // [B][Hkv][1], nullable
  int32_t* seq_tickets;     // [B], zero between calls
};

}  // namespace lrkv
