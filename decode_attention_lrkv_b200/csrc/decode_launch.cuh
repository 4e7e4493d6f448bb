// Launch templates of the decode kernels, instantiated by decode_g*.cu and
// decode_simple.cu (declared in decode_dispatch.h).
#pragma once

#include "decode_simple.cuh"
#include "decode_stream.cuh"
#include "launch_util.cuh"

namespace lrkv {

template <int G, int RK, int RV, int W, int NS, int CB>
inline lrkv_status launch_stream_cb(const DecodeParams& p, dim3 grid, cudaStream_t s) {
  using S = ds::Shape<G, RK, RV, W, NS, CB>;
  auto kern = p.k_new ? ds::decode_stream_kernel<G, RK, RV, W, NS, true, CB>
                      : ds::decode_stream_kernel<G, RK, RV, W, NS, false, CB>;
  if (!set_smem(kern, S::SMEM)) return LRKV_ERR_CUDA;
  return launch_pdl(kern, grid, dim3(S::kThreads), S::SMEM, s, p);
}

// bf16 coefficients, int8 or int4 codes
template <int G, int RK, int RV, int W, int NS>
inline lrkv_status launch_stream(const DecodeParams& p, dim3 grid, cudaStream_t s) {
  const int bits = coef_bits_of(p.D);
  if (bits == 8) return launch_stream_cb<G, RK, RV, W, NS, 8>(p, grid, s);
  if (bits == 4) return launch_stream_cb<G, RK, RV, W, NS, 4>(p, grid, s);
  return launch_stream_cb<G, RK, RV, W, NS, 16>(p, grid, s);
}

template <int G>
inline lrkv_status launch_simple(const DecodeParams& p, dim3 grid, cudaStream_t s) {
  const size_t smem = decode_simple_smem_bytes(G, p.n_chunk_max);
  if (!set_smem(decode_simple_kernel<G>, smem)) return LRKV_ERR_CUDA;
  decode_simple_kernel<G><<<grid, kDecThreads, smem, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

template <int G>
inline lrkv_status launch_stream_g(const DecodeParams& p, dim3 grid, cudaStream_t s, bool* done) {
  *done = true;
  const int rk = p.D.r_k, rv = p.D.r_v;
  // (warps per CTA, ring stages per warp) per shape: what shared memory holds
  // beside the mask words and the resident U_v
  if (rk == 32 && rv == 32) return launch_stream<G, 32, 32, 8, 3>(p, grid, s);
  if (rk == 48 && rv == 64) return launch_stream<G, 48, 64, 8, 3>(p, grid, s);
  if (rk == 48 && rv == 80) return launch_stream<G, 48, 80, 8, 2>(p, grid, s);
  if (rk == 64 && rv == 64) return launch_stream<G, 64, 64, 8, 2>(p, grid, s);
  if (rk == 64 && rv == 96) return launch_stream<G, 64, 96, 8, 2>(p, grid, s);
  *done = false;
  return LRKV_OK;
}

}  // namespace lrkv
