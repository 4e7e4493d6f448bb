// Shared device helpers and the workspace layout of liblrkv.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "lrkv.h"

namespace lrkv {

constexpr int kD = 128;            // head dimension handled by this build
constexpr int kDefaultSMs = 148;   // B200: used only when no device can be queried
constexpr int kMaxDecodeChunk = 8192;   // positions per decode split, at most
constexpr int kMinDecodeChunk = 128;    // positions per decode split, at least (when T allows)
constexpr int kDecodeOverhead = 1024;   // a decode CTA's fixed cost, in streamed positions
constexpr float kLog2e = 1.4426950408889634f;

// bf16 <-> fp32.  A bf16 value is the top half of the fp32 with the same
// bits, so widening is a shift; narrowing uses round-to-nearest-even.
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf2f(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }
__device__ __forceinline__ uint16_t f2bf(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}
// x rounded to bf16 (nearest even), as fp32
__device__ __forceinline__ float bf16_round(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
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

// Stored coefficient format: bits per coefficient (16 bf16, 8 or 4 integer codes).
__host__ __device__ __forceinline__ int coef_bits_of(const lrkv_dims& D) {
  return D.coef_bits == 0 ? 16 : D.coef_bits;
}
__host__ __device__ __forceinline__ bool coef_quantised(const lrkv_dims& D) {
  return coef_bits_of(D) < 16;
}

// Per-row quantisation of a stored coefficient row (codes with per-vector
// scales): Q = 127 for 8 bits, 7 for 4 bits; s = amax / Q with amax the largest
// |bf16(c_j)|; q_j = round_half_even(bf16(c_j) / s) clamped to [-Q, Q]; s = 0
// gives q = 0.  Every step is IEEE fp32 (correctly rounded division), so the
// decisions are those of any implementation of the same steps.
__device__ __forceinline__ float quant_scale(float amax, int bits) {
  return __fdiv_rn(amax, bits == 8 ? 127.f : 7.f);
}
__device__ __forceinline__ int quant_code(float cb, float s, int bits) {
  if (!(s > 0.f)) return 0;
  const int Q = bits == 8 ? 127 : 7;
  const int qv = __float2int_rn(__fdiv_rn(cb, s));
  return qv > Q ? Q : (qv < -Q ? -Q : qv);
}
// The same code from inv = 1/s (any rounding): t = cb * inv is within a few
// ulps of the correctly rounded quotient, so the nearest integer is the same
// unless t lies within 2^-15 of a half-integer (|t| <= Q + 1 < 128, where an
// ulp is at most 2^-17); those cases take the correctly rounded division.
__device__ __forceinline__ int quant_code_fast(float cb, float s, float inv, int bits) {
  if (!(s > 0.f)) return 0;
  const int Q = bits == 8 ? 127 : 7;
  float t = cb * inv;
  if (fabsf(fabsf(t - rintf(t)) - 0.5f) <= 3.0517578125e-05f || fabsf(t) > 128.f)
    t = __fdiv_rn(cb, s);   // rare
  const int qv = __float2int_rn(t);
  return qv > Q ? Q : (qv < -Q ? -Q : qv);
}

// The codes of 16 values of a row with scale s and inv = 1/s (any rounding),
// packed: 8-bit codes into cw[0..3] (byte k), 4-bit codes into cw[0..1]
// (nibble k).  The same decisions as quant_code, with plain ALU/FMA steps:
// rr = t + 1.5 * 2^23 for t = w * inv holds the nearest integer of t (half to
// even) in its low mantissa bits, so the code's two's-complement byte (nibble)
// is the low byte (nibble) of rr's bits; t is within 2^-15 of the correctly
// rounded quotient w / s (|t| <= Q + 2^-16 since s is the row's amax / Q, so
// no clamp is needed), and only a t that close to a half-integer redoes the
// correctly rounded division.
// bw: the 16 values, bf16, as pairs (element 2i in the low half of bw[i]).
__device__ __forceinline__ void quant_pack16_bf(const uint32_t (&bw)[8], float s, float inv, int bits,
                                                uint32_t (&cw)[4]) {
  uint32_t r[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint32_t pr = bw[k >> 1];
    const float b = (k & 1) ? __uint_as_float(pr & 0xffff0000u) : __uint_as_float(pr << 16);
    const float t = b * inv;
    float rr = t + 12582912.f;
    if (fabsf(t - (rr - 12582912.f)) >= 0.49996948f)   // within 2^-15 of a half-integer: rare
      rr = __int_as_float(0x4B400000 + (s > 0.f ? __float2int_rn(__fdiv_rn(b, s)) : 0));
    r[k] = __float_as_uint(rr);
  }
  if (bits == 8) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      cw[j] = __byte_perm(__byte_perm(r[4 * j], r[4 * j + 1], 0x0040), __byte_perm(r[4 * j + 2], r[4 * j + 3], 0x0040),
                          0x5410);
  } else {
#pragma unroll
    for (int j = 0; j < 2; ++j) {   // even codes' bytes, odd codes' bytes, then nibble pairs
      const uint32_t ev = __byte_perm(__byte_perm(r[8 * j], r[8 * j + 2], 0x0040),
                                      __byte_perm(r[8 * j + 4], r[8 * j + 6], 0x0040), 0x5410);
      const uint32_t od = __byte_perm(__byte_perm(r[8 * j + 1], r[8 * j + 3], 0x0040),
                                      __byte_perm(r[8 * j + 5], r[8 * j + 7], 0x0040), 0x5410);
      cw[j] = (ev & 0x0f0f0f0fu) | ((od << 4) & 0xf0f0f0f0u);
    }
    cw[2] = cw[3] = 0u;
  }
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
  int chunk;               // decode: positions per split of a full cache
  int n_split;             // decode: splits per (b, kv head) in the plain decode's grid
  int n_chunk_max;         // decode: records per (b, kv head), the fused call's grid
  int partial_floats;      // floats per (split, q head)
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Streaming multiprocessors of the current device, queried once per device.
// kDefaultSMs when no device is visible (a host-only size query).
inline int num_sms() {
  static std::atomic<int> cached[64];   // 0 until queried
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return kDefaultSMs;
  }
  if (dev >= 0 && dev < 64) {
    const int v = cached[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return kDefaultSMs;
  }
  if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

// How one (batch row, kv head) with T positions is split for decode: n splits
// of `chunk` positions (a multiple of 32, one mask word; at most
// kMaxDecodeChunk), n in [n_min, n_max] minimising the modelled makespan
//   ceil(BH * n / sms) * (chunk + kDecodeOverhead)
// with BH (batch row, kv head) pairs and one CTA per SM resident at a time.
// The cost only drops where n fills a wave, so the candidates are the largest
// n of the first four wave counts that n_min allows, and n_max.  Every CTA
// evaluates this for its own sequence, so the model is evaluated in fp32 (the
// choice only has to be good) and the chosen split in exact 32-bit integers.
// Returns the splits that hold positions (ceil(T / chunk) <= n).  tail_short:
// the chunk is sized for T + tail_short positions (still at most
// kMaxDecodeChunk), which leaves the last split that many positions fewer on
// average -- room for extra work its CTA does (the fused append).
__host__ __device__ inline int decode_split(int T, int n_max_grid, long long BH, int sms,
                                            int* chunk_out, int tail_short = 0) {
  if (T <= 0) {
    *chunk_out = kMinDecodeChunk;
    return 1;
  }
  const unsigned uT = (unsigned)T;
  const int n_min = (int)((uT + kMaxDecodeChunk - 1) / kMaxDecodeChunk);
  int n_max = (int)((uT + kMinDecodeChunk - 1) / kMinDecodeChunk);
  if (n_max > n_max_grid) n_max = n_max_grid;
  if (n_max < n_min) n_max = n_min;
  // The model only ranks candidates (the chunk itself is computed exactly
  // below), so on the device its quotients use the fast approximate divide
  // (relative error ~2.4e-7): every CTA runs this on its critical path, and
  // 21 IEEE divisions in a chain took ~1 us there.  Floor and ceil take the
  // quotient nudged by 1e-6 of itself, which keeps exact integers where the
  // exact model puts them (the smallest relative gap to an integer here is
  // above 1e-6 for T below a million positions).
#ifdef __CUDA_ARCH__
  auto q = [](float a, float b) { return __fdividef(a, b); };
#else
  auto q = [](float a, float b) { return a / b; };
#endif
  auto fl = [](float x) { return floorf(x * (1.f + 1e-6f)); };
  auto ce = [](float x) { return ceilf(x * (1.f - 1e-6f)); };
  const float fbh = (float)BH, fsm = (float)sms, ft = (float)T;
  const float w0 = ce(q(fbh * (float)n_min, fsm));   // waves at n_min
  float best_cost = -1.f;
  int best_n = n_min;
  for (int k = 0; k <= 4; ++k) {
    float nf = k < 4 ? fl(q((w0 + (float)k) * fsm, fbh)) : (float)n_max;
    nf = fminf(fmaxf(nf, (float)n_min), (float)n_max);
    const float ch = ce(q(ft, 32.f * nf)) * 32.f;
    const float waves = ce(q(fbh * ce(q(ft, ch)), fsm));
    const float cost = waves * (ch + (float)kDecodeOverhead);
    if (best_cost < 0.f || cost < best_cost) best_cost = cost, best_n = (int)nf;
  }
  const unsigned n = (unsigned)best_n;
  unsigned ch = ((uT + (unsigned)tail_short + n - 1) / n + 31) / 32 * 32;
  const unsigned ch_min = ((uT + n - 1) / n + 31) / 32 * 32;
  if (ch > kMaxDecodeChunk) ch = ch_min > kMaxDecodeChunk ? ch_min : kMaxDecodeChunk;
  *chunk_out = (int)ch;
  return (int)((uT + ch - 1) / ch);
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
  // decode: the plain decode's grid has the splits of a full cache; each CTA
  // re-splits the live length (decode_split) within them.  A fused append
  // takes the last CTA of its grid, and the other CTAs must still hold the
  // fewest splits a cached length can need (ceil(T_cap / kMaxDecodeChunk)), so
  // its grid, and the records per (b, kv head), are one more than that when
  // the plain grid has no CTA to spare.
  L.n_split = decode_split(D.T_cap, 1024, (long long)D.B * D.Hkv, num_sms(), &L.chunk);
  const int n_least = (D.T_cap + kMaxDecodeChunk - 1) / kMaxDecodeChunk;
  L.n_chunk_max = L.n_split > n_least ? L.n_split : n_least + 1;
  if (L.n_chunk_max < 2) L.n_chunk_max = 2;
  L.partial_floats = 4 + D.r_v + D.d;   // m, l, pad, pad, acc_c[r_v], acc_f[d]
  L.partials = off;
  // records per split: the query heads of a launch (the CUDA-core kernel
  // takes all g at once, the streaming kernel passes of up to 4)
  int g = D.Hkv > 0 ? D.Hq / D.Hkv : 0;
  if (g > 2 && g < 4) g = 4;
  off = align_up(off + sizeof(float) * (size_t)D.B * D.Hkv * L.n_chunk_max * g *
                           L.partial_floats, 256);
  L.total = off;
  return L;
}

}  // namespace lrkv
