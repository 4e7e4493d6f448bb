// Write path, CUDA-core version: projection, relative error, routing flags,
// then an order-preserving compaction of the routed tokens.
//
// OjaKV repository README, "Method Summary": a fixed per-head basis
// (StaticPCA) and the hybrid policy that keeps tokens with a high
// reconstruction error in full rank (OjaKV).
#pragma once

#include "lrkv_common.cuh"

namespace lrkv {

struct CompressParams {
  lrkv_dims D;
  lrkv_cache C;
  const lrkv_bf16* k_new;
  const lrkv_bf16* v_new;
  int t_new;
  const int32_t* t_new_b;
  float tau;
  float* err_out;
  uint8_t* flags;     // [B][Hkv][T_cap]
  int32_t* ticket;    // compaction CTAs done
};

constexpr int kProjTok = 32;      // tokens per projection CTA
constexpr int kProjThreads = 256;

// Shared memory of the projection kernel (floats):
//   U [d][r+1] (padded), X [kProjTok][d+1], Cf [kProjTok][r+1], R/N [kProjTok][d]
inline size_t proj_smem_bytes(int r_max) {
  return sizeof(float) * ((size_t)kD * (r_max + 1) + kProjTok * (kD + 1) +
                          kProjTok * (r_max + 1) + 2 * kProjTok * kD);
}

// One tensor (K or V) of one token tile: coefficients, stored bf16, and the
// relative reconstruction error per token into e_out[kProjTok].
__device__ void project_tile(const lrkv_bf16* __restrict__ U_g, int r,
                             const lrkv_bf16* __restrict__ X_g, int x_stride,
                             int ntok, lrkv_bf16* __restrict__ coef_g, float* smem,
                             float* e_out) {
  float* Us = smem;                              // [d][r+1]
  float* Xs = Us + kD * (r + 1);                 // [T][d+1]
  float* Cs = Xs + kProjTok * (kD + 1);          // [T][r+1]
  float* Rs = Cs + kProjTok * (r + 1);           // [T][d] squared residual
  float* Ns = Rs + kProjTok * kD;                // [T][d] squared input
  const int tid = threadIdx.x;
  for (int o = tid; o < kD * r; o += kProjThreads) {
    int i = o / r, j = o % r;
    Us[i * (r + 1) + j] = bf2f(U_g[o]);
  }
  for (int o = tid; o < kProjTok * kD; o += kProjThreads) {
    int t = o / kD, i = o % kD;
    Xs[t * (kD + 1) + i] = t < ntok ? bf2f(X_g[(size_t)t * x_stride + i]) : 0.f;
  }
  __syncthreads();
  for (int o = tid; o < kProjTok * r; o += kProjThreads) {
    int t = o / r, j = o % r;
    float acc = 0.f;
#pragma unroll 8
    for (int i = 0; i < kD; ++i) acc = fmaf(Xs[t * (kD + 1) + i], Us[i * (r + 1) + j], acc);
    Cs[t * (r + 1) + j] = acc;
  }
  __syncthreads();
  for (int o = tid; o < kProjTok * kD; o += kProjThreads) {
    int t = o / kD, i = o % kD;
    float xh = 0.f;
    for (int j = 0; j < r; ++j) xh = fmaf(Cs[t * (r + 1) + j], Us[i * (r + 1) + j], xh);
    float x = Xs[t * (kD + 1) + i];
    float dlt = x - xh;
    Rs[t * kD + i] = dlt * dlt;
    Ns[t * kD + i] = x * x;
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  for (int t = warp; t < kProjTok; t += kProjThreads / 32) {
    float rs = 0.f, ns = 0.f;
    for (int i = lane; i < kD; i += 32) {
      rs += Rs[t * kD + i];
      ns += Ns[t * kD + i];
    }
    rs = warp_sum(rs);
    ns = warp_sum(ns);
    if (lane == 0) e_out[t] = ns > 0.f ? sqrtf(rs / ns) : 0.f;
  }
  for (int o = tid; o < ntok * r; o += kProjThreads) {
    int t = o / r, j = o % r;
    coef_g[(size_t)t * r + j] = f2bf(Cs[t * (r + 1) + j]);
  }
  __syncthreads();
}

// grid (ceil(min(t_new, T_cap) / kProjTok), Hkv, B)
__global__ void __launch_bounds__(kProjThreads) project_kernel(CompressParams p) {
  extern __shared__ float smem[];
  __shared__ float e_k[kProjTok], e_v[kProjTok];
  const lrkv_dims& D = p.D;
  const int b = blockIdx.z, h = blockIdx.y;
  uint32_t st = 0;
  const int n = new_tokens(p.t_new_b, b, p.t_new, &st);
  const int start = min(max(p.C.seq_len[b], 0), D.T_cap);
  int n_eff = D.T_cap - start;
  if (n_eff > n) n_eff = n;
  if (n_eff < 0) n_eff = 0;
  const int t0 = blockIdx.x * kProjTok;
  if (t0 >= n_eff) return;
  const int ntok = min(kProjTok, n_eff - t0);
  const size_t x_off = (((size_t)b * p.t_new + t0) * D.Hkv + h) * kD;
  const int x_stride = D.Hkv * kD;
  const size_t row0 = ((size_t)b * D.Hkv + h) * D.T_cap + start + t0;
  project_tile(p.C.U_k + (size_t)h * kD * D.r_k, D.r_k, p.k_new + x_off, x_stride, ntok,
               p.C.coef_k + row0 * D.r_k, smem, e_k);
  project_tile(p.C.U_v + (size_t)h * kD * D.r_v, D.r_v, p.v_new + x_off, x_stride, ntok,
               p.C.coef_v + row0 * D.r_v, smem, e_v);
  for (int t = threadIdx.x; t < ntok; t += kProjThreads) {
    float e = fmaxf(e_k[t], e_v[t]);
    p.flags[((size_t)b * D.Hkv + h) * D.T_cap + t0 + t] = e > p.tau ? 1 : 0;
    if (p.err_out) p.err_out[((size_t)b * D.Hkv + h) * p.t_new + t0 + t] = e;
  }
}

constexpr int kCompactThreads = 256;

// Order-preserving compaction, one CTA per (kv head, batch row), walking the
// new positions one 32-bit mask word per warp: warp ballot for the mask word,
// block-wide prefix sum for the list slots.  The last CTA to finish advances
// seq_len (every CTA has read it by then).  grid (Hkv, B)
__global__ void __launch_bounds__(kCompactThreads) compact_kernel(CompressParams p) {
  const lrkv_dims& D = p.D;
  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kWarps = kCompactThreads / 32;
  __shared__ int warp_tot[kWarps];
  __shared__ int s_base;
  __shared__ bool s_last;
  uint32_t st = 0;
  const int n = new_tokens(p.t_new_b, b, p.t_new, &st);
  const int start = min(max(p.C.seq_len[b], 0), D.T_cap);
  int n_eff = D.T_cap - start;
  if (n_eff > n) n_eff = n;
  if (n_eff < 0) n_eff = 0;
  const size_t bh = (size_t)b * D.Hkv + h;
  const uint8_t* flags = p.flags + bh * D.T_cap;
  uint32_t* mask = p.C.route_mask + bh * (D.T_cap / 32);
  int32_t* fidx = p.C.full_idx + bh * D.F_cap;
  lrkv_bf16* fk = p.C.full_k + bh * D.F_cap * kD;
  lrkv_bf16* fv = p.C.full_v + bh * D.F_cap * kD;
  if (tid == 0) s_base = min(max(p.C.full_cnt[bh], 0), D.F_cap);
  __syncthreads();
  int base = s_base;
  bool overflow = false;
  if (n_eff > 0) {
    const int w_first = start / 32, w_last = (start + n_eff - 1) / 32;
    for (int w0 = w_first; w0 <= w_last; w0 += kWarps) {
      const int w = w0 + warp;
      const int pos = w * 32 + lane;
      const int t = pos - start;
      const bool inside = (w <= w_last) && t >= 0 && t < n_eff;
      const bool f = inside && flags[t];
      const uint32_t fb = __ballot_sync(0xffffffffu, f);
      if (lane == 0) warp_tot[warp] = __popc(fb);
      __syncthreads();
      int before = 0, total = 0;
      for (int i = 0; i < kWarps; ++i) {
        before += i < warp ? warp_tot[i] : 0;
        total += warp_tot[i];
      }
      const int slot = base + before + __popc(fb & ((1u << lane) - 1u));
      const bool ok = f && slot < D.F_cap;
      if (f && !ok) overflow = true;
      const uint32_t okb = __ballot_sync(0xffffffffu, ok);
      const uint32_t covered = __ballot_sync(0xffffffffu, inside);
      if (lane == 0 && covered) mask[w] = (mask[w] & ~covered) | okb;
      if (ok) fidx[slot] = pos;
      // copy the key/value rows of the routed tokens of this warp, one row per pass
      uint32_t todo = okb;
      while (todo) {
        const int src_lane = __ffs(todo) - 1;
        todo &= todo - 1;
        const int ts = w * 32 + src_lane - start;
        const int sl = base + before + __popc(fb & ((1u << src_lane) - 1u));
        const size_t x = (((size_t)b * p.t_new + ts) * D.Hkv + h) * kD;
        const uint2* ks = reinterpret_cast<const uint2*>(p.k_new + x);
        const uint2* vs = reinterpret_cast<const uint2*>(p.v_new + x);
        reinterpret_cast<uint2*>(fk + (size_t)sl * kD)[lane] = ks[lane];
        reinterpret_cast<uint2*>(fv + (size_t)sl * kD)[lane] = vs[lane];
      }
      base += total;
      __syncthreads();
    }
  }
  if (n_eff < n) st |= LRKV_DEV_SEQ_OVERFLOW;
  if (h != 0) st = 0;                       // per-sequence conditions: reported once
  if (__syncthreads_or(overflow)) st |= LRKV_DEV_FULL_OVERFLOW;
  if (tid == 0 && st) atomicOr(p.C.dev_status, st);
  if (tid == 0) {
    p.C.full_cnt[bh] = base < D.F_cap ? base : D.F_cap;
    __threadfence();
    const int done = atomicAdd(p.ticket, 1);
    s_last = (done == (int)(gridDim.x * gridDim.y) - 1);
  }
  __syncthreads();
  if (s_last) {
    __threadfence();
    for (int bb = tid; bb < D.B; bb += kCompactThreads) {
      uint32_t dummy = 0;
      const int nb = new_tokens(p.t_new_b, bb, p.t_new, &dummy);
      const int sb = min(max(p.C.seq_len[bb], 0), D.T_cap);
      int ne = D.T_cap - sb;
      if (ne > nb) ne = nb;
      if (ne < 0) ne = 0;
      p.C.seq_len[bb] = sb + ne;
    }
    if (tid == 0) *p.ticket = 0;
  }
}

}  // namespace lrkv
