// Decode dispatch shared by lrkv_decode_attn and lrkv_decode_attn_noalloc:
// the tensor-core streaming kernel for the shapes it is instantiated for, the
// CUDA-core kernel for every other valid shape.
#pragma once

#include "decode_simple.cuh"
#include "decode_stream.cuh"
#include "launch_util.cuh"

namespace lrkv {

template <int G, int RK, int RV, int W, int NS>
inline lrkv_status launch_stream(const DecodeParams& p, dim3 grid, cudaStream_t s) {
  using S = ds::Shape<G, RK, RV, W, NS>;
  auto kern = p.k_new ? ds::decode_stream_kernel<G, RK, RV, W, NS, true>
                      : ds::decode_stream_kernel<G, RK, RV, W, NS, false>;
  if (!set_smem(kern, S::SMEM)) return LRKV_ERR_CUDA;
  return launch_pdl(kern, grid, dim3(S::kThreads), S::SMEM, s, p);
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

// Whether the streaming kernel covers these sizes.
inline bool stream_decode_supported(const lrkv_dims& D, int chunk) {
  const int g = D.Hq / D.Hkv;
  if (g != 1 && g != 2 && g != 4) return false;
  if (chunk > ds::kMaxChunk || chunk % 32) return false;
  const int rk = D.r_k, rv = D.r_v;
  return (rk == 32 && rv == 32) || (rk == 48 && rv == 64) || (rk == 48 && rv == 80) ||
         (rk == 64 && rv == 64) || (rk == 64 && rv == 96);
}

// p.k_new set: the fused append + decode, which only the streaming kernel has
// (the caller checks stream_decode_supported first).
inline lrkv_status launch_decode(const DecodeParams& p, cudaStream_t s) {
  const dim3 grid(p.n_chunk_max, p.D.Hkv, p.D.B);
  const int g = p.D.Hq / p.D.Hkv;
  if (stream_decode_supported(p.D, p.chunk)) {
    bool done = false;
    lrkv_status st = LRKV_OK;
    if (g == 1) st = launch_stream_g<1>(p, grid, s, &done);
    else if (g == 2) st = launch_stream_g<2>(p, grid, s, &done);
    else st = launch_stream_g<4>(p, grid, s, &done);
    if (done) return st;
  }
  if (p.k_new) return LRKV_ERR_UNSUPPORTED;
  switch (g) {
    case 1: return launch_simple<1>(p, grid, s);
    case 2: return launch_simple<2>(p, grid, s);
    case 3: return launch_simple<3>(p, grid, s);
    case 4: return launch_simple<4>(p, grid, s);
    case 5: return launch_simple<5>(p, grid, s);
    case 6: return launch_simple<6>(p, grid, s);
    case 7: return launch_simple<7>(p, grid, s);
    case 8: return launch_simple<8>(p, grid, s);
    default: return LRKV_ERR_UNSUPPORTED;
  }
}

}  // namespace lrkv
