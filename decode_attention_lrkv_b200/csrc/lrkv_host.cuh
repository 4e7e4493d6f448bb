// Host-side argument checks shared by every entry point of the C ABI, so that
// each call reports the same synchronous error for the same bad argument.
#pragma once

#include <cstdint>

#include "lrkv.h"
#include "lrkv_common.cuh"

namespace lrkv {

constexpr int kMaxG = 8;   // query heads per kv head handled by the decode kernels

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Sizes: LRKV_ERR_INVALID_ARG for values no build accepts, LRKV_ERR_UNSUPPORTED
// for valid sizes this build does not handle.
inline lrkv_status check_dims(const lrkv_dims* D) {
  if (!D) return LRKV_ERR_INVALID_ARG;
  if (D->B < 1 || D->Hq < 1 || D->Hkv < 1 || D->T_cap < 32 || D->F_cap < 0)
    return LRKV_ERR_INVALID_ARG;
  if (D->B > 65535 || D->Hkv > 65535) return LRKV_ERR_UNSUPPORTED;
  if (D->Hq % D->Hkv != 0) return LRKV_ERR_INVALID_ARG;
  if (D->T_cap % 32 != 0) return LRKV_ERR_INVALID_ARG;
  if (D->d != kD) return LRKV_ERR_UNSUPPORTED;
  if (D->r_k < 16 || D->r_k > D->d || D->r_k % 16 || D->r_v < 16 || D->r_v > D->d || D->r_v % 16)
    return LRKV_ERR_INVALID_ARG;
  if (D->Hq / D->Hkv > kMaxG) return LRKV_ERR_UNSUPPORTED;
  if (D->coef_bits != 0 && D->coef_bits != 16 && D->coef_bits != 8 && D->coef_bits != 4)
    return LRKV_ERR_INVALID_ARG;
  return LRKV_OK;
}

// The cache's pointers: present (the full-rank list only when F_cap > 0) and
// 16-byte aligned.
inline lrkv_status check_cache(const lrkv_dims* D, const lrkv_cache* C) {
  if (!C) return LRKV_ERR_INVALID_ARG;
  const void* need[] = {C->U_k, C->U_v, C->coef_k, C->coef_v, C->route_mask,
                        C->full_cnt, C->seq_len, C->dev_status};
  for (const void* p : need)
    if (!p) return LRKV_ERR_INVALID_ARG;
  const void* full[] = {C->full_idx, C->full_k, C->full_v};
  for (const void* p : full)
    if (!p && D->F_cap > 0) return LRKV_ERR_INVALID_ARG;
  for (const void* p : need)
    if (!aligned16(p)) return LRKV_ERR_ALIGNMENT;
  for (const void* p : full)
    if (!aligned16(p)) return LRKV_ERR_ALIGNMENT;
  if (!aligned16(C->U_kq) || !aligned16(C->mu_k)) return LRKV_ERR_ALIGNMENT;   // optional
  if (coef_quantised(*D)) {   // per-row scales of the codes
    if (!C->scale_k || !C->scale_v) return LRKV_ERR_INVALID_ARG;
    if (!aligned16(C->scale_k) || !aligned16(C->scale_v)) return LRKV_ERR_ALIGNMENT;
  }
  return LRKV_OK;
}

// A decode's query and output pointers.
inline lrkv_status check_q_out(const void* q, const void* out) {
  if (!q || !out) return LRKV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out)) return LRKV_ERR_ALIGNMENT;
  return LRKV_OK;
}

}  // namespace lrkv
