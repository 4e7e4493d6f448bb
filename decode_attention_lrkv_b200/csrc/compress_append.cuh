// Write path for a few new tokens per sequence (decode-time appends): one
// CTA per (kv head, batch row) projects, measures and routes the row's new
// tokens in position order, all in one launch.
//
// OjaKV repository README, "Method Summary": the fixed per-head basis of
// StaticPCA, and the hybrid policy of OjaKV that keeps tokens with a high
// reconstruction error in full rank.  Per token x (key, then value):
//   c = U^T x (fp32), stored as bf16 at the token's position;
//   e = ||x - U c|| / ||x|| by direct reconstruction (0 when x = 0);
//   routed iff max(e_k, e_v) > tau: the k and v rows go to the next slot of
//   the full-rank list and the mask bit is set (kept compressed with
//   FULL_OVERFLOW when the list is full).
#pragma once

#include "compress_params.cuh"
#include "lrkv_common.cuh"
#include "ptx.cuh"

namespace lrkv {

constexpr int kAppendThreads = 256;    // two halves of 128: keys and values side by side
constexpr int kAppendMaxTokens = 16;   // larger appends take the tiled path
constexpr uint32_t kAppendWaitIters = 1u << 24;

// Shared memory: U_k, U_v as stored (bf16 [d][r]), the new tokens' key and
// value rows (bf16 [kAppendMaxTokens][d] each) and, with an attention-aware key
// basis, U_kq (bf16 [d][r_k]), all filled by bulk copies; then per half: x [d],
// partial c [4][d], c [d], reduction scratch; one mbarrier.
inline size_t append_smem_bytes(int r_k, int r_v, bool aware) {
  return sizeof(uint16_t) * (size_t)kD * (r_k + r_v + 2 * kAppendMaxTokens + (aware ? r_k : 0)) +
         sizeof(float) * 2 * (6 * kD + 8) + 16;
}

// One tensor (the key for half 0, the value for half 1) of one token: x (bf16
// [d] in shared memory) -> coefficients c = Us^T (x - mu) (bf16, global);
// returns the relative error ||x - mu - Urec c|| / ||x|| to every thread of the
// half (Urec = Us and mu = null except for an attention-aware key basis).  All
// 256 threads call it together.
// bits 16: coef_g receives the row as bf16; bits 8 or 4: as codes, with the
// row's scale in *scale_g (per-row quantisation of the stored row).
__device__ __forceinline__ float append_project(const uint16_t* __restrict__ x_s,
                                                const uint16_t* Us, const uint16_t* Urec,
                                                const float* mu, int r, int bits,
                                                unsigned char* __restrict__ coef_g,
                                                float* __restrict__ scale_g, float* ws) {
  const int tid = threadIdx.x & 127;
  const int warp = tid >> 5, lane = tid & 31;
  float* xs = ws;                 // [d]
  float* part = xs + kD;          // [4][d]
  float* cs = part + 4 * kD;      // [d]
  float* red = cs + kD;           // [8]
  const float xraw = bf2f(x_s[tid]);
  const float x = mu ? xraw - mu[tid] : xraw;
  xs[tid] = x;
  __syncthreads();
  // c_j = sum_i U[i][j] x_i: warp w sums rows 32w..32w+31, lane owns columns lane + 32k
  {
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    const uint16_t* U = Us + warp * 32 * r;
#pragma unroll 8
    for (int ii = 0; ii < 32; ++ii) {
      const float xi = xs[warp * 32 + ii];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (lane + 32 * k < r) a[k] = fmaf(bf2f(U[ii * r + lane + 32 * k]), xi, a[k]);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (lane + 32 * k < r) part[warp * kD + lane + 32 * k] = a[k];
  }
  __syncthreads();
  float c = 0.f;
  if (tid < r) {
    c = (part[tid] + part[kD + tid]) + (part[2 * kD + tid] + part[3 * kD + tid]);
    cs[tid] = c;
  }
  if (bits == 16) {
    if (tid < r) reinterpret_cast<lrkv_bf16*>(coef_g)[tid] = f2bf(c);
  } else {   // per-row codes: the row's amax over the half's warps, then one code per column
    const float cb = tid < r ? bf16_round(c) : 0.f;
    const float a = warp_max(fabsf(cb));
    if (lane == 0) red[warp] = a;
    __syncthreads();
    const float s = quant_scale(fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])), bits);
    const int qv = quant_code(cb, s, bits);
    const int qn = __shfl_down_sync(0xffffffffu, qv, 1);   // the odd neighbour's code (4-bit pairs)
    if (tid < r) {
      if (bits == 8) coef_g[tid] = (unsigned char)(qv & 0xff);
      else if ((tid & 1) == 0) coef_g[tid >> 1] = (unsigned char)((qv & 0xf) | ((qn & 0xf) << 4));
    }
    if (tid == 0) *scale_g = s;
  }
  __syncthreads();
  // x_hat_i = sum_j U[i][j] c_j: thread i walks row i two columns at a time,
  // starting at column pair (i mod r/2), so a warp's 32 rows hit 32 banks.
  const int npair = r >> 1;
  const uint32_t* row = reinterpret_cast<const uint32_t*>(Urec) + tid * npair;
  const float2* c2 = reinterpret_cast<const float2*>(cs);
  float h0 = 0.f, h1 = 0.f;
  int w = tid % npair;
#pragma unroll 8
  for (int k = 0; k < npair; ++k) {
    const uint32_t u = row[w];
    const float2 cc = c2[w];
    h0 = fmaf(bf_lo(u), cc.x, h0);
    h1 = fmaf(bf_hi(u), cc.y, h1);
    w = (w + 1 == npair) ? 0 : w + 1;
  }
  const float dlt = x - (h0 + h1);
  const float rs = warp_sum(dlt * dlt), ns = warp_sum(xraw * xraw);
  if (lane == 0) red[warp] = rs, red[4 + warp] = ns;
  __syncthreads();
  const float rsum = (red[0] + red[1]) + (red[2] + red[3]);
  const float nsum = (red[4] + red[5]) + (red[6] + red[7]);
  return nsum > 0.f ? sqrtf(rsum / nsum) : 0.f;
}

// grid (Hkv, B), kAppendThreads threads
__global__ void __launch_bounds__(kAppendThreads) append_kernel(CompressParams p) {
  extern __shared__ __align__(16) unsigned char sm_app[];
  const lrkv_dims& D = p.D;
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int r_k = D.r_k, r_v = D.r_v;
  const int bits = coef_bits_of(D);   // stored coefficient format
  uint16_t* Uks = reinterpret_cast<uint16_t*>(sm_app);
  uint16_t* Uvs = Uks + kD * r_k;
  uint16_t* Xks = Uvs + kD * r_v;                          // new key rows
  uint16_t* Xvs = Xks + kD * kAppendMaxTokens;             // new value rows
  const bool aware = p.C.U_kq != nullptr;
  uint16_t* Ukqs = Xvs + kD * kAppendMaxTokens;            // query-side key basis (aware only)
  float* ws0 = reinterpret_cast<float*>(Ukqs + (aware ? kD * r_k : 0));   // per-half scratch
  const int half = tid >> 7;
  float* ws = ws0 + half * (6 * kD + 8);
  uint64_t* bar = reinterpret_cast<uint64_t*>(ws0 + 2 * (6 * kD + 8));
  __shared__ int s_cnt;
  __shared__ bool s_last;
  __shared__ float s_err[2];

  // bases first: they do not depend on the preceding kernel of the stream
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    const uint32_t bk = kD * r_k * 2, bv = kD * r_v * 2;
    mbar_expect_tx(bar, bk + bv + (aware ? bk : 0));
    bulk_g2s(Uks, p.C.U_k + (size_t)h * kD * r_k, bk, bar);
    bulk_g2s(Uvs, p.C.U_v + (size_t)h * kD * r_v, bv, bar);
    if (aware) bulk_g2s(Ukqs, p.C.U_kq + (size_t)h * kD * r_k, bk, bar);
  }
  griddep_launch_dependents();
  griddep_wait();   // the new rows and the cache state come from earlier kernels

  uint32_t st = 0;
  const int n = new_tokens(p.t_new_b, b, p.t_new, &st);
  const size_t bh = (size_t)b * D.Hkv + h;
  // the new rows do not depend on the cache state: their copies go out first
  if (tid == 0) {
    mbar_arrive_expect_tx(bar, n * 4u * kD);   // the arrival that closes the phase
    for (int t = 0; t < n; ++t) {
      const size_t x = (((size_t)b * p.t_new + t) * D.Hkv + h) * kD;
      bulk_g2s(Xks + t * kD, p.k_new + x, 2u * kD, bar);
      bulk_g2s(Xvs + t * kD, p.v_new + x, 2u * kD, bar);
    }
  }
  const int start = min(max(p.C.seq_len[b], 0), D.T_cap);
  const int cnt0 = tid == 0 ? p.C.full_cnt[bh] : 0;
  int n_eff = D.T_cap - start;
  if (n_eff > n) n_eff = n;
  if (n_eff < 0) n_eff = 0;
  uint32_t* mask_row = p.C.route_mask + bh * (D.T_cap / 32);
  if (tid == 0) s_cnt = min(max(cnt0, 0), D.F_cap);
  // Every thread of this CTA holds its sequence's start: take the ticket now.
  // The CTA that takes the last one advances every sequence's length; the
  // other CTAs have all read theirs by then (acquire/release on the ticket).
  __syncthreads();
  if (tid == 0) s_last = atom_add_acq_rel_gpu(p.ticket, 1) == (int)(gridDim.x * gridDim.y) - 1;
  __syncthreads();
  if (s_last) {
    for (int bb = tid; bb < D.B; bb += kAppendThreads) {
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
  __syncthreads();
  // every copy (bases included) lands before anything else, also when there is no token
  if (!mbar_wait_bounded(bar, 0, kAppendWaitIters)) st |= LRKV_DEV_WAIT_TIMEOUT;
  if (__syncthreads_or(st & LRKV_DEV_WAIT_TIMEOUT)) {
    mbar_wait_bounded(bar, 0, kAppendWaitIters);   // one more bounded wait for the copies
    st |= LRKV_DEV_WAIT_TIMEOUT;
    if (tid == 0) atomicOr(p.C.dev_status, LRKV_DEV_WAIT_TIMEOUT);
    n_eff = 0;   // leave the cache untouched; the call's results are flagged invalid
  }
  if (n_eff > 0) {
    bool overflow = false;
    uint32_t m_or[2] = {0u, 0u}, m_and[2] = {~0u, ~0u};   // edits of the (at most two) mask words
    for (int t = 0; t < n_eff; ++t) {
      const int pos = start + t;
      const size_t row = bh * D.T_cap + pos;
      // one call site for both halves: every __syncthreads inside is reached by all threads
      const int r = half == 0 ? r_k : r_v;
      const float eh = append_project(half == 0 ? Xks + t * kD : Xvs + t * kD,
                                      half == 0 ? Uks : Uvs, half == 0 ? (aware ? Ukqs : Uks) : Uvs,
                                      half == 0 && p.C.mu_k ? p.C.mu_k + (size_t)h * kD : nullptr,
                                      r, bits,
                                      static_cast<unsigned char*>(half == 0 ? p.C.coef_k : p.C.coef_v) +
                                          row * (size_t)(r * bits / 8),
                                      bits < 16 ? (half == 0 ? p.C.scale_k : p.C.scale_v) + row : nullptr,
                                      ws);
      if ((tid & 127) == 0) s_err[half] = eh;
      __syncthreads();
      const float e = fmaxf(s_err[0], s_err[1]);
      const bool routed = e > p.tau;
      const int slot = s_cnt;
      const bool keep = routed && slot < D.F_cap;
      if (routed && !keep) overflow = true;
      if (keep) {
        const int i = tid & 127;
        if (half == 0) p.C.full_k[(bh * D.F_cap + slot) * kD + i] = Xks[t * kD + i];
        else p.C.full_v[(bh * D.F_cap + slot) * kD + i] = Xvs[t * kD + i];
      }
      if (tid == 0) {
        const uint32_t bit = 1u << (pos & 31);
        const int wsel = (pos >> 5) - (start >> 5);
        if (keep) m_or[wsel] |= bit;
        else m_and[wsel] &= ~bit;
        if (keep) {
          p.C.full_idx[bh * D.F_cap + slot] = pos;
          s_cnt = slot + 1;
        }
        if (p.err_out) p.err_out[bh * p.t_new + t] = e;
      }
      __syncthreads();
    }
    if (tid == 0) {
      p.C.full_cnt[bh] = s_cnt;
      // bits of earlier positions in the same words stay as they are
      const int nw = ((start + n_eff - 1) >> 5) - (start >> 5) + 1;
      for (int u = 0; u < nw; ++u) {
        if (m_or[u]) atomicOr(mask_row + (start >> 5) + u, m_or[u]);
        if (m_and[u] != ~0u) atomicAnd(mask_row + (start >> 5) + u, m_and[u]);
      }
      if (overflow) st |= LRKV_DEV_FULL_OVERFLOW;
    }
  }
  if (n_eff < n && !(st & LRKV_DEV_WAIT_TIMEOUT)) st |= LRKV_DEV_SEQ_OVERFLOW;
  if (h != 0) st &= LRKV_DEV_FULL_OVERFLOW;     // per-sequence conditions: reported once
  if (tid == 0 && st) atomicOr(p.C.dev_status, st);
}

}  // namespace lrkv
