// lrkv_oja_update: the C ABI of the online basis update (oja.cuh), in its own
// translation unit.
#include "launch_util.cuh"
#include "lrkv.h"
#include "lrkv_common.cuh"
#include "lrkv_host.cuh"
#include "oja.cuh"

namespace {

using namespace lrkv;

// Row splits of the accumulation: about one wave of CTAs over the kv heads,
// each split a multiple of the 64-row tile.
void oja_splits(int Hkv, int n_rows, int* splits, int* rows_per_split) {
  const int tiles = (n_rows + oja::kTile - 1) / oja::kTile;
  int sp = num_sms() / (Hkv > 0 ? Hkv : 1);
  if (sp < 1) sp = 1;
  if (sp > tiles) sp = tiles;
  const int per = (tiles + sp - 1) / sp;
  *rows_per_split = per * oja::kTile;
  *splits = (tiles + per - 1) / per;
}

template <int RB>
lrkv_status launch_accum(const oja::AccumParams& p, int splits, cudaStream_t s) {
  const size_t smem = oja::accum_smem_bytes(RB * 16);
  if (!set_smem(oja::oja_accum_kernel<RB>, smem)) return LRKV_ERR_CUDA;
  oja::oja_accum_kernel<RB><<<dim3(splits, p.Hkv), oja::kThreads, smem, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

bool oja_args_ok(const lrkv_dims* dims, int32_t n_rows, int32_t r) {
  return dims && dims->Hkv >= 1 && dims->Hkv <= 65535 && n_rows >= 1 && r >= 16 && r <= kD &&
         r % 16 == 0;
}

}  // namespace

extern "C" {

size_t lrkv_oja_workspace_size(const lrkv_dims* dims, int32_t n_rows, int32_t r) {
  if (!oja_args_ok(dims, n_rows, r) || dims->d != kD) return 0;
  int splits, rps;
  oja_splits(dims->Hkv, n_rows, &splits, &rps);
  return sizeof(float) * (size_t)dims->Hkv * splits * ((size_t)kD * r + (size_t)r * r);
}

lrkv_status lrkv_oja_update(const lrkv_dims* dims, const lrkv_bf16* X, int32_t n_rows, int32_t r,
                            float eta, float* U, lrkv_bf16* U_out, void* ws, size_t ws_bytes,
                            void* stream) {
  if (!oja_args_ok(dims, n_rows, r) || !X || !U) return LRKV_ERR_INVALID_ARG;
  if (dims->d != kD) return LRKV_ERR_UNSUPPORTED;
  if (!(eta >= 0.f) || !(eta < 1e30f)) return LRKV_ERR_INVALID_ARG;   // NaN, negative, infinite
  if (!aligned16(X) || !aligned16(U) || !aligned16(U_out) || !aligned16(ws)) return LRKV_ERR_ALIGNMENT;
  const size_t need = lrkv_oja_workspace_size(dims, n_rows, r);
  if (!ws || ws_bytes < need) return LRKV_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  oja::AccumParams ap;
  ap.X = X;
  ap.U = U;
  ap.n_rows = n_rows;
  ap.Hkv = dims->Hkv;
  ap.r = r;
  ap.partials = static_cast<float*>(ws);
  int splits;
  oja_splits(dims->Hkv, n_rows, &splits, &ap.rows_per_split);
  lrkv_status st;
  switch (r / 16) {
    case 1: st = launch_accum<1>(ap, splits, s); break;
    case 2: st = launch_accum<2>(ap, splits, s); break;
    case 3: st = launch_accum<3>(ap, splits, s); break;
    case 4: st = launch_accum<4>(ap, splits, s); break;
    case 5: st = launch_accum<5>(ap, splits, s); break;
    case 6: st = launch_accum<6>(ap, splits, s); break;
    case 7: st = launch_accum<7>(ap, splits, s); break;
    default: st = launch_accum<8>(ap, splits, s); break;
  }
  if (st != LRKV_OK) return st;
  oja::FinishParams fp;
  fp.partials = ap.partials;
  fp.splits = splits;
  fp.r = r;
  fp.n_rows = n_rows;
  fp.eta = eta;
  fp.U = U;
  fp.U_bf16 = U_out;
  const size_t smem = oja::finish_smem_bytes(r);
  if (!set_smem(oja::oja_finish_kernel, smem)) return LRKV_ERR_CUDA;
  oja::oja_finish_kernel<<<dims->Hkv, oja::kFinishThreads, smem, s>>>(fp);
  if (cudaGetLastError() != cudaSuccess) return LRKV_ERR_CUDA;
  return launch_stream_fence(s);   // the bases are written: a decode may follow
}

}  // extern "C"
