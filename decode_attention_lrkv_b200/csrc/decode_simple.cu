// The CUDA-core decode kernel for every query group size, and the dispatch
// between it and the streaming kernel.
#include "decode_dispatch.h"
#include "decode_launch.cuh"

namespace lrkv {

lrkv_status launch_simple_any(const DecodeParams& p, dim3 grid, cudaStream_t s) {
  switch (p.D.Hq / p.D.Hkv) {
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

bool stream_decode_supported(const lrkv_dims& D) {
  const int g = D.Hq / D.Hkv;
  if (g != 1 && g != 2 && g != 4) return false;
  const int rk = D.r_k, rv = D.r_v;
  return (rk == 32 && rv == 32) || (rk == 48 && rv == 64) || (rk == 48 && rv == 80) ||
         (rk == 64 && rv == 64) || (rk == 64 && rv == 96);
}

lrkv_status launch_decode(const DecodeParams& p, cudaStream_t s) {
  const dim3 grid(p.n_chunk_max, p.D.Hkv, p.D.B);
  const int g = p.D.Hq / p.D.Hkv;
  if (stream_decode_supported(p.D)) {
    bool done = false;
    lrkv_status st = LRKV_OK;
    if (g == 1) st = launch_stream_g1(p, grid, s, &done);
    else if (g == 2) st = launch_stream_g2(p, grid, s, &done);
    else st = launch_stream_g4(p, grid, s, &done);
    if (done) return st;
  }
  if (p.k_new) return LRKV_ERR_UNSUPPORTED;
  return launch_simple_any(p, grid, s);
}

}  // namespace lrkv
