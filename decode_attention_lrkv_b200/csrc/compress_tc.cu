// The prefill-sized write path: tensor-core projection and the two routing
// passes, in their own translation unit (declared in compress_tc.h).
#include <cuda.h>

#include <algorithm>
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

// The projection's grid over `groups` (kv head, K or V) groups of `n_units`
// tiles each (Params::per_group): k CTAs per group, or one range per SM over
// the groups' tiles laid end to end, a range that crosses into the next group
// finishing there as a second CTA.  The modelled makespan in tiles (with
// kCtaSetupTiles for each CTA on an SM: basis layouts, U U^T, the pipeline's
// fill and drain) picks one: 64 groups on 148 SMs leave 20 SMs idle in the
// first form.
int projection_grid(int groups, int n_units, int sms, ptc::Params* pp) {
  constexpr long long kCtaSetupTiles = 8;
  const long long total = (long long)groups * n_units;
  int k = sms / groups;
  if (k < 1) k = 1;
  if (k > n_units) k = n_units;
  const long long grid_a = (long long)k * groups;
  const long long cost_a = (grid_a + sms - 1) / sms * ((n_units + k - 1) / k + kCtaSetupTiles);
  const int n_ranges = (int)(total < sms ? total : sms);
  const long long per = (total + n_ranges - 1) / n_ranges;
  const long long cost_b = per + 2 * kCtaSetupTiles;
  pp->per_group = k;
  pp->n_ranges = 0;
  if (per > n_units || n_ranges > ptc::kMaxRanges || cost_b >= cost_a) return (int)grid_a;
  // ranges split at a group end: their second parts, longest first
  const int q = (int)(total / n_ranges), r = (int)(total % n_ranges);
  int order[ptc::kMaxRanges], rest[ptc::kMaxRanges], n2 = 0;
  for (int x = 0; x < n_ranges; ++x) {
    const int l0 = x * q + (x < r ? x : r), l1 = l0 + q + (x < r ? 1 : 0);
    const int end = (l0 / n_units + 1) * n_units;
    if (l1 > end) order[n2] = x, rest[x] = l1 - end, ++n2;
  }
  std::stable_sort(order, order + n2, [&](int a, int b) { return rest[a] > rest[b]; });
  for (int j = 0; j < n2; ++j) pp->second[j] = (uint16_t)order[j];
  pp->per_group = 0;
  pp->n_ranges = n_ranges;
  return n_ranges + n2;
}

// Prefill-sized compress: tensor-core projection, then the two routing passes.
}  // namespace

lrkv_status compress_tc(const lrkv_dims& D, const lrkv_cache& C, const lrkv_bf16* k_new,
                        const lrkv_bf16* v_new, int t_new, const int32_t* t_new_b, float tau,
                        float* err_out, char* w, const WsLayout& L, cudaStream_t s) {
  ptc::Params pp = {};
  const int tmax0 = t_new < D.T_cap ? t_new : D.T_cap;
  // the projection counts its tiles over every (kv head, K or V) group in 32 bits
  if (2LL * D.Hkv * D.B * ((tmax0 + ptc::kTile - 1) / ptc::kTile) >= (1LL << 31)) return LRKV_ERR_UNSUPPORTED;
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
  const int n_ctas = projection_grid(2 * D.Hkv, D.B * pp.tiles_per_b, num_sms(), &pp);
  const size_t smem = ptc::Layout(pp.r_max, pp.n_stages).bytes;
  const int bits = coef_bits_of(D);
  auto kern = bits == 8 ? ptc::project_tc_kernel<8> : bits == 4 ? ptc::project_tc_kernel<4>
                                                                : ptc::project_tc_kernel<16>;
  if (!set_smem(kern, smem) || !set_smem(ptc::route_count_kernel, 0) ||
      !set_smem(ptc::route_scatter_kernel, 0))
    return LRKV_ERR_CUDA;
  kern<<<n_ctas, ptc::kThreads, smem, s>>>(pp);
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
  // the scatter pass takes runs of tiles per CTA once the grid holds more than
  // 16 CTAs per SM (a wave of 128-thread CTAs) twice over
  const long long n_tiles_all = (long long)pp.tiles_per_b * D.Hkv * D.B;
  long long tpc = n_tiles_all / (16LL * num_sms());
  rp.tiles_per_cta = (int)(tpc < 1 ? 1 : tpc > ptc::kMaxScatterTiles ? ptc::kMaxScatterTiles : tpc);
  // the routing passes launch as dependents (programmatic dependent launch):
  // their launch overlaps the preceding kernel's tail, and each waits for it
  const dim3 grid(pp.tiles_per_b, D.Hkv, D.B);
  const dim3 grid_s((pp.tiles_per_b + rp.tiles_per_cta - 1) / rp.tiles_per_cta, D.Hkv, D.B);
  if ((st = launch_pdl(ptc::route_count_kernel, grid, dim3(128), 0, s, rp)) != LRKV_OK) return st;
  return launch_pdl(ptc::route_scatter_kernel, grid_s, dim3(128), 0, s, rp);
}


}  // namespace lrkv
