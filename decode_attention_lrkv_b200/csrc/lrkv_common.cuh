// Shared device helpers and the workspace layout of liblrkv.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lrkv.h"

namespace lrkv {

constexpr int kD = 128;            // head dimension handled by this build
constexpr int kNumSMs = 148;       // B200; only used to size work splits
constexpr int kMaxDecodeChunk = 8192;   // positions per decode split, at most
constexpr float kLog2e = 1.4426950408889634f;

// bf16 <-> fp32.  A bf16 value is the top half of the fp32 with the same
// bits, so widening is a shift; narrowing uses round-to-nearest-even.
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf2f(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }
__device__ __forceinline__ uint16_t f2bf(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Number of new tokens sequence b contributes, and the status bits it raises.
__device__ __forceinline__ int new_tokens(const int32_t* t_new_b, int b, int t_new,
                                          uint32_t* flags) {
  int n = t_new;
  if (t_new_b) {
    n = t_new_b[b];
    if (n < 0 || n > t_new) {
      *flags |= LRKV_DEV_BAD_COUNT;
      n = n < 0 ? 0 : t_new;
    }
  }
  return n;
}

// Workspace layout, identical on host and device.  Offsets in bytes.
struct WsLayout {
  size_t decode_tickets;   // int32 [B][Hkv], zero between calls
  size_t compress_ticket;  // int32 [1], zero between calls
  size_t seq_tickets;      // int32 [B], zero between calls (fused append + decode)
  size_t errs;             // float [2][B][Hkv][T_cap] e_k, e_v of a prefill compress call
  size_t tile_cnt;         // int32 [B][Hkv][n_tiles] routed tokens per 128-token tile
  size_t tile_bits;        // uint32 [B][Hkv][n_tiles][4] routed bits per tile
  int n_tiles;             // ceil(T_cap / 128)
  size_t partials;         // float [B][Hkv][n_chunk_max][g][4 + r_v + d]
  size_t total;
  int chunk;               // decode: positions per split
  int n_chunk_max;         // decode: splits per (b, kv head)
  int partial_floats;      // floats per (split, q head)
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Positions per decode split: at least 128, a multiple of 32 (one mask word),
// at most kMaxDecodeChunk.  The split count n minimises the modelled makespan
//   ceil(B*Hkv*n / SMs) * (chunk + overhead)
// with one CTA per SM resident at a time; `overhead` is a CTA's fixed cost
// (bases, q~, merge) expressed in streamed positions.
inline int decode_chunk(const lrkv_dims& D) {
  const long long bh = (long long)D.B * D.Hkv;
  const long long overhead = 1024;
  long long best_cost = -1, best = kMaxDecodeChunk;
  const long long n_max = (D.T_cap + 127) / 128;
  for (long long n = 1; n <= n_max && n <= 1024; ++n) {
    long long ch = (D.T_cap + n - 1) / n;
    ch = (ch + 31) / 32 * 32;
    if (ch < 128) ch = 128;
    if (ch > kMaxDecodeChunk) continue;
    const long long splits = (D.T_cap + ch - 1) / ch;
    const long long waves = (bh * splits + kNumSMs - 1) / kNumSMs;
    const long long cost = waves * (ch + overhead);
    if (best_cost < 0 || cost < best_cost) best_cost = cost, best = ch;
  }
  return (int)best;
}

inline WsLayout ws_layout(const lrkv_dims& D) {
  WsLayout L;
  size_t off = 0;
  L.decode_tickets = off;
  off = align_up(off + sizeof(int32_t) * (size_t)D.B * D.Hkv, 256);
  L.compress_ticket = off;
  off = align_up(off + sizeof(int32_t), 256);
  L.seq_tickets = off;
  off = align_up(off + sizeof(int32_t) * (size_t)D.B, 256);
  L.n_tiles = (D.T_cap + 127) / 128;
  L.errs = off;
  off = align_up(off + sizeof(float) * 2 * (size_t)D.B * D.Hkv * D.T_cap, 256);
  L.tile_cnt = off;
  off = align_up(off + sizeof(int32_t) * (size_t)D.B * D.Hkv * L.n_tiles, 256);
  L.tile_bits = off;
  off = align_up(off + sizeof(uint32_t) * 4 * (size_t)D.B * D.Hkv * L.n_tiles, 256);
  L.chunk = decode_chunk(D);
  L.n_chunk_max = (D.T_cap + L.chunk - 1) / L.chunk;
  L.partial_floats = 4 + D.r_v + D.d;   // m, l, pad, pad, acc_c[r_v], acc_f[d]
  L.partials = off;
  int g = D.Hkv > 0 ? D.Hq / D.Hkv : 0;
  off = align_up(off + sizeof(float) * (size_t)D.B * D.Hkv * L.n_chunk_max * g *
                           L.partial_floats, 256);
  L.total = off;
  return L;
}

}  // namespace lrkv
