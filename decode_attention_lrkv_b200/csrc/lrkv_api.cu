// liblrkv.so: the C ABI declared in include/lrkv.h.  Host-side validation,
// workspace carving and kernel launches; no allocation, no synchronisation.
#include <cmath>
#include <cstdint>

#include <cuda.h>

#include "basis_fit.cuh"
#include "compress_append.cuh"
#include "compress_params.cuh"
#include "compress_tc.h"
#include "decode_dispatch.h"
#include "launch_util.cuh"
#include "lrkv.h"
#include "lrkv_common.cuh"
#include "lrkv_host.cuh"

namespace lrkv {
__global__ void stream_fence_kernel() {}
}  // namespace lrkv

namespace {

using namespace lrkv;

lrkv_status check_ws(const lrkv_dims* D, void* ws, size_t ws_bytes, WsLayout* L) {
  *L = ws_layout(*D);
  if (!ws || ws_bytes < L->total) return LRKV_ERR_INVALID_ARG;
  if (!aligned16(ws)) return LRKV_ERR_ALIGNMENT;
  return LRKV_OK;
}

lrkv_status launched() {
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

// Row splits of the Gram pass: about one wave of CTAs over the kv heads, each
// split a multiple of the ring's 64-row tile.
inline void fit_splits(int Hkv, int n_rows, int* splits, int* rows_per_split) {
  const int tiles = (n_rows + fit::kTileRows - 1) / fit::kTileRows;
  int sp = num_sms() / (Hkv > 0 ? Hkv : 1);
  if (sp < 1) sp = 1;
  if (sp > tiles) sp = tiles;
  const int tiles_per = (tiles + sp - 1) / sp;
  *rows_per_split = tiles_per * fit::kTileRows;
  *splits = (tiles + tiles_per - 1) / tiles_per;
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
  CompressParams p = {};
  p.D = *dims;
  p.C = *cache;
  p.k_new = k_new;
  p.v_new = v_new;
  p.t_new = t_new;
  p.t_new_b = t_new_b;
  p.tau = tau;
  p.err_out = err_out;
  p.ticket = reinterpret_cast<int32_t*>(w + L.compress_ticket);
  if (t_new <= kAppendMaxTokens) {  // decode-time appends: one fused launch
    const size_t smem = append_smem_bytes(dims->r_k, dims->r_v, cache->U_kq != nullptr);
    if (!set_smem(append_kernel, smem)) return LRKV_ERR_CUDA;
    return launch_pdl(append_kernel, dim3(dims->Hkv, dims->B), dim3(kAppendThreads), smem, s, p);
  }
  return compress_tc(*dims, *cache, k_new, v_new, t_new, t_new_b, tau, err_out, w, L, s);
}

lrkv_status lrkv_decode_attn(const lrkv_dims* dims, const lrkv_cache* cache, const lrkv_bf16* q,
                             float* out, void* ws, size_t ws_bytes, void* stream) {
  lrkv_status st = check_dims(dims);
  if (st != LRKV_OK) return st;
  if ((st = check_cache(dims, cache)) != LRKV_OK) return st;
  if ((st = check_q_out(q, out)) != LRKV_OK) return st;
  WsLayout L;
  if ((st = check_ws(dims, ws, ws_bytes, &L)) != LRKV_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  DecodeParams p = {};
  p.D = *dims;
  p.C = *cache;
  p.q = q;
  p.out = out;
  p.tickets = reinterpret_cast<int32_t*>(w + L.decode_tickets);
  p.partials = reinterpret_cast<float*>(w + L.partials);
  p.n_split = L.n_split;
  p.n_chunk_max = L.n_chunk_max;
  p.num_sms = num_sms();
  return launch_decode(p, s);
}

lrkv_status lrkv_append_decode_attn(const lrkv_dims* dims, const lrkv_cache* cache,
                                    const lrkv_bf16* k_new, const lrkv_bf16* v_new,
                                    const int32_t* t_new_b, float tau, float* err_out,
                                    const lrkv_bf16* q, float* out, void* ws, size_t ws_bytes,
                                    void* stream) {
  lrkv_status st = check_dims(dims);
  if (st != LRKV_OK) return st;
  if ((st = check_cache(dims, cache)) != LRKV_OK) return st;
  if (!k_new || !v_new || !q || !out) return LRKV_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(t_new_b) || !aligned16(err_out) ||
      !aligned16(q) || !aligned16(out))
    return LRKV_ERR_ALIGNMENT;
  WsLayout L;
  if ((st = check_ws(dims, ws, ws_bytes, &L)) != LRKV_OK) return st;
  if (!stream_decode_supported(*dims)) {   // the two launches it fuses
    st = lrkv_compress(dims, cache, k_new, v_new, 1, t_new_b, tau, err_out, ws, ws_bytes, stream);
    if (st != LRKV_OK) return st;
    return lrkv_decode_attn(dims, cache, q, out, ws, ws_bytes, stream);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  DecodeParams p = {};
  p.D = *dims;
  p.C = *cache;
  p.q = q;
  p.out = out;
  p.tickets = reinterpret_cast<int32_t*>(w + L.decode_tickets);
  p.partials = reinterpret_cast<float*>(w + L.partials);
  p.n_split = L.n_split;
  p.n_chunk_max = L.n_chunk_max;
  p.num_sms = num_sms();
  p.k_new = k_new;
  p.v_new = v_new;
  p.t_new_b = t_new_b;
  p.tau = tau;
  p.err_out = err_out;
  p.seq_tickets = reinterpret_cast<int32_t*>(w + L.seq_tickets);
  return launch_decode(p, s);
}

size_t lrkv_fit_workspace_size(const lrkv_dims* dims, int32_t n_rows) {
  if (!dims || dims->Hkv < 1 || dims->Hkv > 65535 || dims->d != kD || n_rows < 1) return 0;
  int splits, rps;
  fit_splits(dims->Hkv, n_rows, &splits, &rps);
  return sizeof(float) * (size_t)dims->Hkv * splits * kD * kD;
}

lrkv_status lrkv_fit_basis(const lrkv_dims* dims, const lrkv_bf16* X, int32_t n_rows, int32_t r,
                           lrkv_bf16* U_out, float* eigvals_out, void* ws, size_t ws_bytes,
                           void* stream) {
  if (!dims || !X || !U_out || n_rows < 1) return LRKV_ERR_INVALID_ARG;
  if (dims->Hkv < 1 || dims->Hkv > 65535) return LRKV_ERR_INVALID_ARG;
  if (dims->d != kD) return LRKV_ERR_UNSUPPORTED;
  if (r < 1 || r > kD) return LRKV_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(U_out) || !aligned16(eigvals_out) || !aligned16(ws))
    return LRKV_ERR_ALIGNMENT;
  const size_t need = lrkv_fit_workspace_size(dims, n_rows);
  if (!ws || ws_bytes < need) return LRKV_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  fit::GramParams gp;
  gp.X = X;
  gp.n_rows = n_rows;
  gp.Hkv = dims->Hkv;
  gp.partials = static_cast<float*>(ws);
  int splits;
  fit_splits(dims->Hkv, n_rows, &splits, &gp.rows_per_split);
  const size_t gsmem = 2 * fit::kStageBytes;
  if (!set_smem(fit::gram_kernel, gsmem)) return LRKV_ERR_CUDA;
  fit::gram_kernel<<<dim3(splits, dims->Hkv), fit::kThreads, gsmem, s>>>(gp);
  lrkv_status st = launched();
  if (st != LRKV_OK) return st;
  fit::EigParams ep;
  ep.partials = gp.partials;
  ep.splits = splits;
  ep.r = r;
  ep.U = U_out;
  ep.eigvals = eigvals_out;
  const size_t esmem = fit::eig_smem_bytes();
  if (!set_smem(fit::eig_kernel, esmem)) return LRKV_ERR_CUDA;
  fit::eig_kernel<<<dims->Hkv, fit::kEigThreads, esmem, s>>>(ep);
  if ((st = launched()) != LRKV_OK) return st;
  return launch_stream_fence(s);   // the bases are written: a decode may follow
}

lrkv_status lrkv_rank_for_budget(const float* eigvals, int32_t n_heads, int32_t d, double budget,
                                 int32_t* r_out) {
  if (!eigvals || !r_out || n_heads < 1 || d < 1 || d > 4096) return LRKV_ERR_INVALID_ARG;
  if (!(budget >= 0.0 && budget <= 1.0)) return LRKV_ERR_INVALID_ARG;   // NaN fails too
  double tail[4097];
  for (int32_t h = 0; h < n_heads; ++h) {
    const float* lam = eigvals + (size_t)h * d;
    // tail[j] = mass of eigenvalues j..d-1, summed from the smallest up
    tail[d] = 0.0;
    for (int32_t j = d - 1; j >= 0; --j) tail[j] = tail[j + 1] + (lam[j] > 0.f ? (double)lam[j] : 0.0);
    const double limit = budget * tail[0];
    int32_t r = 1;
    while (r < d && tail[r] > limit) ++r;
    r_out[h] = r;
  }
  return LRKV_OK;
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
