// lrkv_decode_attn_noalloc: decode attention whose scratch lives in a
// file-scope device array, for callers that cannot allocate device memory.
//
// The split-K decode needs scratch (one ticket per (batch row, kv head) and
// one partial softmax record per split).  lrkv_decode_attn takes it from a
// caller-allocated workspace; this entry point takes it from
// g_decode_scratch below instead, so the caller passes only the cache, the
// query and the output.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "decode_launch.cuh"
#include "lrkv.h"
#include "lrkv_common.cuh"

namespace {

using namespace lrkv;

// The scratch itself.  Every GPU that loads the library holds these
// LRKV_NOALLOC_SCRATCH_BYTES until the process exits; every call on a
// device shares them.
static __device__ __align__(256) unsigned char g_decode_scratch[LRKV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::once_flag g_once[kMaxDevices];
void* g_scratch[kMaxDevices];
cudaError_t g_setup_err[kMaxDevices];

// Device address of g_decode_scratch on the current device.  In host code the
// symbol name is only a stand-in; cudaGetSymbolAddress gives the address a
// kernel can use.  Done once per device, with that device current.
lrkv_status scratch_address(void** ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LRKV_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return LRKV_ERR_UNSUPPORTED;
  std::call_once(g_once[dev], [dev] {
    g_setup_err[dev] = cudaGetSymbolAddress(&g_scratch[dev], g_decode_scratch);
    if (g_setup_err[dev] != cudaSuccess) cudaGetLastError();
  });
  if (g_setup_err[dev] != cudaSuccess) return LRKV_ERR_CUDA;
  *ptr = g_scratch[dev];
  return LRKV_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

lrkv_status check_args(const lrkv_dims* D, const lrkv_cache* C, const void* q, const void* out) {
  if (!D || !C || !q || !out) return LRKV_ERR_INVALID_ARG;
  if (D->B < 1 || D->Hq < 1 || D->Hkv < 1 || D->T_cap < 32 || D->F_cap < 0 ||
      D->T_cap % 32 || D->Hq % D->Hkv)
    return LRKV_ERR_INVALID_ARG;
  if (D->B > 65535 || D->Hkv > 65535 || D->d != kD || D->Hq / D->Hkv > 8)
    return LRKV_ERR_UNSUPPORTED;
  if (D->r_k < 16 || D->r_k > D->d || D->r_k % 16 || D->r_v < 16 || D->r_v > D->d || D->r_v % 16)
    return LRKV_ERR_INVALID_ARG;
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
  if (!aligned16(q) || !aligned16(out)) return LRKV_ERR_ALIGNMENT;
  return LRKV_OK;
}

}  // namespace

extern "C" LRKV_API lrkv_status lrkv_decode_attn_noalloc(const lrkv_dims* dims,
                                                         const lrkv_cache* cache,
                                                         const lrkv_bf16* q, float* out,
                                                         void* stream) {
  lrkv_status st = check_args(dims, cache, q, out);
  if (st != LRKV_OK) return st;
  // scratch = tickets [B][Hkv] int32, then the split partials, as in the workspace
  const WsLayout L = ws_layout(*dims);
  const size_t ticket_bytes = align_up(sizeof(int32_t) * (size_t)dims->B * dims->Hkv, 256);
  const size_t partial_bytes = L.total - L.partials;
  if (ticket_bytes + partial_bytes > (size_t)LRKV_NOALLOC_SCRATCH_BYTES)
    return LRKV_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != LRKV_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(scratch);
  // the array keeps the previous call's contents: the tickets must start at zero
  if (cudaMemsetAsync(base, 0, ticket_bytes, s) != cudaSuccess) {
    cudaGetLastError();
    return LRKV_ERR_CUDA;
  }
  DecodeParams p = {};
  p.D = *dims;
  p.C = *cache;
  p.q = q;
  p.out = out;
  p.tickets = reinterpret_cast<int32_t*>(base);
  p.partials = reinterpret_cast<float*>(base + ticket_bytes);
  p.chunk = L.chunk;
  p.n_chunk_max = L.n_chunk_max;
  return launch_decode(p, s);
}
