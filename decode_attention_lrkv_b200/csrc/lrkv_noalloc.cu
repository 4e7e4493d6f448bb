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

#include "decode_dispatch.h"
#include "lrkv.h"
#include "lrkv_common.cuh"
#include "lrkv_host.cuh"

namespace {

using namespace lrkv;

// The scratch itself.  Every GPU that loads the library holds these
// LRKV_NOALLOC_SCRATCH_BYTES until the process exits; every call on a
// device shares them.
static __device__ __align__(256) unsigned char g_decode_scratch[LRKV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex[kMaxDevices];
void* g_scratch[kMaxDevices];   // non-null once looked up on that device

// Device address of g_decode_scratch on the current device.  In host code the
// symbol name is only a stand-in; cudaGetSymbolAddress gives the address a
// kernel can use.  Looked up once per device, with that device current, and
// kept only when the lookup succeeded: a failed lookup (for instance during a
// stream capture) is tried again by the next call.
lrkv_status scratch_address(void** ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LRKV_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return LRKV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex[dev]);
  if (!g_scratch[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return LRKV_ERR_CUDA;
    }
    g_scratch[dev] = p;
  }
  *ptr = g_scratch[dev];
  return LRKV_OK;
}

}  // namespace

extern "C" LRKV_API lrkv_status lrkv_decode_attn_noalloc(const lrkv_dims* dims,
                                                         const lrkv_cache* cache,
                                                         const lrkv_bf16* q, float* out,
                                                         void* stream) {
  // the sizes first (as lrkv_decode_attn checks them), then whether the scratch
  // holds this decode, then the pointers
  lrkv_status st = check_dims(dims);
  if (st != LRKV_OK) return st;
  // scratch = tickets [B][Hkv] int32, then the split partials, as in the workspace
  const WsLayout L = ws_layout(*dims);
  const size_t ticket_bytes = align_up(sizeof(int32_t) * (size_t)dims->B * dims->Hkv, 256);
  const size_t partial_bytes = L.total - L.partials;
  if (ticket_bytes + partial_bytes > (size_t)LRKV_NOALLOC_SCRATCH_BYTES)
    return LRKV_ERR_UNSUPPORTED;
  if ((st = check_cache(dims, cache)) != LRKV_OK) return st;
  if ((st = check_q_out(q, out)) != LRKV_OK) return st;
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
  p.n_split = L.n_split;
  p.n_chunk_max = L.n_chunk_max;
  p.num_sms = num_sms();
  return launch_decode(p, s);
}
