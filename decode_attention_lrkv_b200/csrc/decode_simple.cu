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
  if (D.Hkv < 1 || D.Hq < D.Hkv) return false;
  const int rk = D.r_k, rv = D.r_v;
  return (rk == 32 && rv == 32) || (rk == 48 && rv == 64) || (rk == 48 && rv == 80) ||
         (rk == 64 && rv == 64) || (rk == 64 && rv == 96);
}

// Query heads per launch of the streaming kernel: 1 or 2 as they are, else
// passes of 4 (the last one partly empty), each streaming the cache once.
int stream_heads_per_pass(int g) { return g <= 2 ? g : 4; }

// Grid: the plain decode's splits, or the fused call's (its last CTA appends).
static dim3 decode_grid(const DecodeParams& p) {
  return dim3(p.k_new ? p.n_chunk_max : p.n_split, p.D.Hkv, p.D.B);
}

lrkv_status launch_decode(const DecodeParams& p0, cudaStream_t s) {
  const int g = p0.D.Hq / p0.D.Hkv;
  if (stream_decode_supported(p0.D)) {
    DecodeParams p = p0;
    p.g_all = g;
    const int per = stream_heads_per_pass(g);
    for (int off = 0; off < g; off += per) {
      p.g_off = off;
      if (off > 0) {   // a fused append happens once, in the first pass; later passes read its result
        p.k_new = p.v_new = nullptr;
        p.t_new_b = nullptr;
        p.err_out = nullptr;
      }
      const dim3 grid = decode_grid(p);
      bool done = false;
      lrkv_status st = LRKV_OK;
      if (per == 1) st = launch_stream_g1(p, grid, s, &done);
      else if (per == 2) st = launch_stream_g2(p, grid, s, &done);
      else st = launch_stream_g4(p, grid, s, &done);
      if (st != LRKV_OK) return st;
      if (!done) return LRKV_ERR_UNSUPPORTED;   // not reached: the rank pairs above are instantiated
    }
    return LRKV_OK;
  }
  if (p0.k_new) return LRKV_ERR_UNSUPPORTED;
  return launch_simple_any(p0, decode_grid(p0), s);
}

}  // namespace lrkv
