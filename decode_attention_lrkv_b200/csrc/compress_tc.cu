// The prefill-sized write path: tensor-core projection and the two routing
// passes, in their own translation unit (declared in compress_tc.h).
#include <cuda.h>

#include <cstdlib>

#include "compress_tc.cuh"
#include "compress_tc.h"
#include "launch_util.cuh"

namespace lrkv {
namespace {

lrkv_status launched() {
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

// Limit of the projection's main-loop wait for each input tile.  The
// environment variable LRKV_MAIN_WAIT_ITERS (a positive integer) lowers it, so
// a test can make that bounded wait run out and check that the call reports
// LRKV_DEV_WAIT_TIMEOUT and leaves the GPU usable; the waits that drain copies
// and MMAs in flight keep their own limit.
uint32_t main_wait_iters() {
  const char* e = std::getenv("LRKV_MAIN_WAIT_ITERS");
  if (e && *e) {
    char* end = nullptr;
    const unsigned long v = std::strtoul(e, &end, 10);
    if (end && *end == '\0' && v > 0 && v < ptc::kWaitIters) return (uint32_t)v;
  }
  return ptc::kWaitIters;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// New key or value rows [B][t_new][Hkv][d] as a 3-d tensor (d, Hkv, B * t_new),
// boxes of 64 columns x 1 head x 128 tokens, 128-byte swizzle.
bool rows_map(CUtensorMap* map, const lrkv_bf16* base, const lrkv_dims& D, int t_new) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)D.Hkv, (cuuint64_t)D.B * t_new};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)D.Hkv * kD * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)ptc::kTile};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<lrkv_bf16*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Prefill-sized compress: tensor-core projection, then the two routing passes.
}  // namespace

lrkv_status compress_tc(const lrkv_dims& D, const lrkv_cache& C, const lrkv_bf16* k_new,
                        const lrkv_bf16* v_new, int t_new, const int32_t* t_new_b, float tau,
                        float* err_out, char* w, const WsLayout& L, cudaStream_t s) {
  ptc::Params pp = {};
  if (!rows_map(&pp.map_k, k_new, D, t_new) || !rows_map(&pp.map_v, v_new, D, t_new))
    return LRKV_ERR_CUDA;
  const int tmax = t_new < D.T_cap ? t_new : D.T_cap;
  pp.D = D;
  pp.C = C;
  pp.t_new = t_new;
  pp.t_new_b = t_new_b;
  pp.errs = reinterpret_cast<float*>(w + L.errs);
  pp.tiles_per_b = (tmax + ptc::kTile - 1) / ptc::kTile;
  pp.r_max = D.r_k > D.r_v ? D.r_k : D.r_v;
  pp.n_stages = ptc::stages_for(pp.r_max);
  pp.wait_iters = main_wait_iters();
  const int groups = 2 * D.Hkv;
  const int n_units = D.B * pp.tiles_per_b;
  int per_group = num_sms() / groups;
  if (per_group < 1) per_group = 1;
  if (per_group > n_units) per_group = n_units;
  const size_t smem = ptc::Layout(pp.r_max, pp.n_stages).bytes;
  const int bits = coef_bits_of(D);
  auto kern = bits == 8 ? ptc::project_tc_kernel<8> : bits == 4 ? ptc::project_tc_kernel<4>
                                                                : ptc::project_tc_kernel<16>;
  if (!set_smem(kern, smem) || !set_smem(ptc::route_count_kernel, 0) ||
      !set_smem(ptc::route_scatter_kernel, 0))
    return LRKV_ERR_CUDA;
  kern<<<dim3(per_group, groups), ptc::kThreads, smem, s>>>(pp);
  lrkv_status st = launched();
  if (st != LRKV_OK) return st;
  ptc::RouteParams rp = {};
  rp.D = D;
  rp.C = C;
  rp.k_new = k_new;
  rp.v_new = v_new;
  rp.t_new = t_new;
  rp.t_new_b = t_new_b;
  rp.tau = tau;
  rp.err_out = err_out;
  rp.errs = pp.errs;
  rp.tile_cnt = reinterpret_cast<int32_t*>(w + L.tile_cnt);
  rp.tile_bits = reinterpret_cast<uint32_t*>(w + L.tile_bits);
  rp.n_tiles = L.n_tiles;
  rp.bh_tickets = reinterpret_cast<int32_t*>(w + L.decode_tickets);
  rp.ticket = reinterpret_cast<int32_t*>(w + L.compress_ticket);
  const dim3 grid(pp.tiles_per_b, D.Hkv, D.B);
  ptc::route_count_kernel<<<grid, 128, 0, s>>>(rp);
  if ((st = launched()) != LRKV_OK) return st;
  ptc::route_scatter_kernel<<<grid, 128, 0, s>>>(rp);
  return launched();
}


}  // namespace lrkv
