// liblrkv.so: the C ABI declared in include/lrkv.h.  Host-side validation,
// workspace carving and kernel launches; no allocation, no synchronisation.
#include <cmath>
#include <cstdint>

#include "compress_append.cuh"
#include "compress_simple.cuh"
#include "decode_launch.cuh"
#include "lrkv.h"
#include "lrkv_common.cuh"

namespace {

using namespace lrkv;

constexpr int kMaxG = 8;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

lrkv_status check_dims(const lrkv_dims* D) {
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
  return LRKV_OK;
}

lrkv_status check_cache(const lrkv_dims* D, const lrkv_cache* C) {
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
  return LRKV_OK;
}

lrkv_status check_ws(const lrkv_dims* D, void* ws, size_t ws_bytes, WsLayout* L) {
  *L = ws_layout(*D);
  if (!ws || ws_bytes < L->total) return LRKV_ERR_INVALID_ARG;
  if (!aligned16(ws)) return LRKV_ERR_ALIGNMENT;
  return LRKV_OK;
}

lrkv_status launched() {
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t lrkv_workspace_size(const lrkv_dims* dims) {
  if (check_dims(dims) != LRKV_OK) return 0;
  return ws_layout(*dims).total;
}

lrkv_status lrkv_compress(const lrkv_dims* dims, const lrkv_cache* cache,
                          const lrkv_bf16* k_new, const lrkv_bf16* v_new, int32_t t_new,
                          const int32_t* t_new_b, float tau, float* err_out, void* ws,
                          size_t ws_bytes, void* stream) {
  lrkv_status st = check_dims(dims);
  if (st != LRKV_OK) return st;
  if ((st = check_cache(dims, cache)) != LRKV_OK) return st;
  if (!k_new || !v_new || t_new < 0) return LRKV_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(t_new_b) || !aligned16(err_out))
    return LRKV_ERR_ALIGNMENT;
  WsLayout L;
  if ((st = check_ws(dims, ws, ws_bytes, &L)) != LRKV_OK) return st;
  if (t_new == 0) return LRKV_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  CompressParams p;
  p.D = *dims;
  p.C = *cache;
  p.k_new = k_new;
  p.v_new = v_new;
  p.t_new = t_new;
  p.t_new_b = t_new_b;
  p.tau = tau;
  p.err_out = err_out;
  p.flags = reinterpret_cast<uint8_t*>(w + L.flags);
  p.ticket = reinterpret_cast<int32_t*>(w + L.compress_ticket);
  if (t_new <= kAppendMaxTokens) {  // decode-time appends: one fused launch
    const size_t smem = append_smem_bytes(dims->r_k, dims->r_v);
    if (cudaFuncSetAttribute(append_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return launched(), LRKV_ERR_CUDA;
    append_kernel<<<dim3(dims->Hkv, dims->B), kAppendThreads, smem, s>>>(p);
    return launched();
  }
  const int tmax = t_new < dims->T_cap ? t_new : dims->T_cap;
  const size_t smem = proj_smem_bytes(dims->r_k > dims->r_v ? dims->r_k : dims->r_v);
  if (cudaFuncSetAttribute(project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return launched(), LRKV_ERR_CUDA;
  project_kernel<<<dim3((tmax + kProjTok - 1) / kProjTok, dims->Hkv, dims->B), kProjThreads, smem,
                   s>>>(p);
  if ((st = launched()) != LRKV_OK) return st;
  compact_kernel<<<dim3(dims->Hkv, dims->B), kCompactThreads, 0, s>>>(p);
  return launched();
}

lrkv_status lrkv_decode_attn(const lrkv_dims* dims, const lrkv_cache* cache, const lrkv_bf16* q,
                             float* out, void* ws, size_t ws_bytes, void* stream) {
  lrkv_status st = check_dims(dims);
  if (st != LRKV_OK) return st;
  if ((st = check_cache(dims, cache)) != LRKV_OK) return st;
  if (!q || !out) return LRKV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out)) return LRKV_ERR_ALIGNMENT;
  WsLayout L;
  if ((st = check_ws(dims, ws, ws_bytes, &L)) != LRKV_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  DecodeParams p;
  p.D = *dims;
  p.C = *cache;
  p.q = q;
  p.out = out;
  p.tickets = reinterpret_cast<int32_t*>(w + L.decode_tickets);
  p.partials = reinterpret_cast<float*>(w + L.partials);
  p.chunk = L.chunk;
  p.n_chunk_max = L.n_chunk_max;
  return launch_decode(p, s);
}

const char* lrkv_status_str(lrkv_status status) {
  switch (status) {
    case LRKV_OK: return "ok";
    case LRKV_ERR_INVALID_ARG: return "invalid argument (null pointer, bad size or workspace too small)";
    case LRKV_ERR_UNSUPPORTED: return "unsupported shape for this build";
    case LRKV_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case LRKV_ERR_CUDA: return "CUDA launch failed";
  }
  return "unknown status";
}

}  // extern "C"
