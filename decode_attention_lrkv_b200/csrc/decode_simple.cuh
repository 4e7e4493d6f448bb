// Read path, CUDA-core reference version: split-K decode attention over the
// compressed cache with an LSE merge fused into the last CTA of each
// (batch row, kv head).
//
// Coefficient-space form of the StaticPCA read path (OjaKV repository
// README, "Method Summary > StaticPCA": keys and values reconstructed on the
// fly for standard attention): q.(U_k c_k) = (U_k^T q).c_k, so logits are
// taken against the coefficients directly, and the value side is
// accumulated in r_v-space and lifted by U_v once at the end.
#pragma once

#include "decode_params.cuh"
#include "lrkv_common.cuh"

namespace lrkv {


constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;

// Partial record of one split for one query head: m (running max of the
// base-2 logits), l (sum of 2^(s - m)), acc_c [r_v], acc_f [d].
__device__ __forceinline__ float* partial_ptr(const DecodeParams& p, int b, int h, int c,
                                              int gi, int g) {
  const int pf = 2 + p.D.r_v + kD;
  return p.partials +
         ((((size_t)b * p.D.Hkv + h) * p.n_chunk_max + c) * g + gi) * (size_t)pf;
}

// Shared memory (floats): qs [G][d], qt [G][d], per-warp state
// [warps][G][2 + d + d], merge weights [n_chunk_max][G].
inline size_t decode_simple_smem_bytes(int G, int n_chunk_max) {
  return sizeof(float) * ((size_t)2 * G * kD + (size_t)kDecWarps * G * (2 + 2 * kD) +
                          (size_t)n_chunk_max * G + 2 * G);
}

template <int G>
__global__ void __launch_bounds__(kDecThreads) decode_simple_kernel(DecodeParams p) {
  extern __shared__ float sm[];
  const lrkv_dims& D = p.D;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int T = p.C.seq_len[b];
  T = T < 0 ? 0 : (T > D.T_cap ? D.T_cap : T);
  int chunk;   // positions per split, from the live length
  const int n_chunks = decode_split(T, p.n_split, (long long)D.B * D.Hkv, p.num_sms, &chunk);
  if (c >= n_chunks) return;
  const int r_k = D.r_k, r_v = D.r_v;
  const size_t bh = (size_t)b * D.Hkv + h;

  float* qs = sm;                  // [G][d]  q * log2(e)/sqrt(d)
  float* qt = qs + G * kD;         // [G][d]  U_kq^T q * log2(e)/sqrt(d)  (r_k used)
  float* ws = qt + G * kD;         // per-warp state
  float* wts = ws + kDecWarps * G * (2 + 2 * kD);
  __shared__ float s_bias[G];      // q . mu_k * log2(e)/sqrt(d): added to compressed logits
  const float scale = kLog2e * rsqrtf((float)kD);

  for (int o = tid; o < G * kD; o += kDecThreads) {
    const int gi = o / kD, i = o % kD;
    qs[o] = bf2f(p.q[((size_t)b * D.Hq + h * G + gi) * kD + i]) * scale;
  }
  __syncthreads();
  // q~ in the query-side key basis (U_k unless an attention-aware U_kq is given)
  const lrkv_bf16* Uk = (p.C.U_kq ? p.C.U_kq : p.C.U_k) + (size_t)h * kD * r_k;
  for (int o = tid; o < G * r_k; o += kDecThreads) {
    const int gi = o / r_k, j = o % r_k;
    float acc = 0.f;
    for (int i = 0; i < kD; ++i) acc = fmaf(bf2f(Uk[i * r_k + j]), qs[gi * kD + i], acc);
    qt[gi * kD + j] = acc;
  }
  if (warp < G) {
    float s = 0.f;
    if (p.C.mu_k)
      for (int i = lane; i < kD; i += 32) s = fmaf(qs[warp * kD + i], p.C.mu_k[(size_t)h * kD + i], s);
    s = warp_sum(s);
    if (lane == 0) s_bias[warp] = s;
  }
  __syncthreads();

  float m[G], l[G], accc[G][4], accf[G][4];
#pragma unroll
  for (int gi = 0; gi < G; ++gi) {
    m[gi] = -INFINITY;
    l[gi] = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) accc[gi][k] = accf[gi][k] = 0.f;
  }

  // compressed tokens of this split
  const int c0 = c * chunk;
  const int c1 = min(T, c0 + chunk);
  const uint32_t* mask = p.C.route_mask + bh * (D.T_cap / 32);
  // stored coefficients: bf16, or integer codes (8 or 4 bits) with per-row scales
  const int bits = coef_bits_of(D);
  const unsigned char* ck = static_cast<const unsigned char*>(p.C.coef_k) + bh * D.T_cap * (size_t)(r_k * bits / 8);
  const unsigned char* cv = static_cast<const unsigned char*>(p.C.coef_v) + bh * D.T_cap * (size_t)(r_v * bits / 8);
  auto coef_at = [&](const unsigned char* rows, int t, int j, int r) -> float {
    if (bits == 16) return bf2f(reinterpret_cast<const uint16_t*>(rows)[(size_t)t * r + j]);
    if (bits == 8) return (float)(int8_t)rows[(size_t)t * r + j];
    const int byte = rows[(size_t)t * (r / 2) + (j >> 1)];
    const int nib = (j & 1) ? (byte >> 4) : (byte & 0xf);
    return (float)(nib >= 8 ? nib - 16 : nib);
  };
  for (int t = c0 + warp; t < c1; t += kDecWarps) {
    if ((mask[t >> 5] >> (t & 31)) & 1u) continue;
    float kv[4], vv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j = lane + 32 * k;
      kv[k] = j < r_k ? coef_at(ck, t, j, r_k) : 0.f;
      vv[k] = j < r_v ? coef_at(cv, t, j, r_v) : 0.f;
    }
    const float sk = bits < 16 ? p.C.scale_k[bh * D.T_cap + t] : 1.f;   // code scales
    const float sv = bits < 16 ? p.C.scale_v[bh * D.T_cap + t] : 1.f;
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int j = lane + 32 * k;
        if (j < r_k) s = fmaf(qt[gi * kD + j], kv[k], s);
      }
      s = fmaf(warp_sum(s), sk, s_bias[gi]);
      const float mn = fmaxf(m[gi], s);
      const float sc = exp2f(m[gi] - mn);
      const float pr = exp2f(s - mn);
      l[gi] = l[gi] * sc + pr;
      const float pv = pr * sv;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        accc[gi][k] = fmaf(pv, vv[k], accc[gi][k] * sc);
        accf[gi][k] *= sc;
      }
      m[gi] = mn;
    }
  }

  // full-rank tokens: this split's share of the list
  const int F = min(max(p.C.full_cnt[bh], 0), D.F_cap);
  const int share = (F + n_chunks - 1) / n_chunks;
  const int f0 = c * share, f1 = min(F, f0 + share);
  const lrkv_bf16* fk = p.C.full_k + bh * D.F_cap * kD;
  const lrkv_bf16* fv = p.C.full_v + bh * D.F_cap * kD;
  for (int f = f0 + warp; f < f1; f += kDecWarps) {
    float kv[4], vv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      kv[k] = bf2f(fk[(size_t)f * kD + lane + 32 * k]);
      vv[k] = bf2f(fv[(size_t)f * kD + lane + 32 * k]);
    }
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) s = fmaf(qs[gi * kD + lane + 32 * k], kv[k], s);
      s = warp_sum(s);
      const float mn = fmaxf(m[gi], s);
      const float sc = exp2f(m[gi] - mn);
      const float pr = exp2f(s - mn);
      l[gi] = l[gi] * sc + pr;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        accf[gi][k] = fmaf(pr, vv[k], accf[gi][k] * sc);
        accc[gi][k] *= sc;
      }
      m[gi] = mn;
    }
  }

  // combine the warps of this CTA
  const int stride = 2 + 2 * kD;
#pragma unroll
  for (int gi = 0; gi < G; ++gi) {
    float* w = ws + (warp * G + gi) * stride;
    if (lane == 0) {
      w[0] = m[gi];
      w[1] = l[gi];
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      w[2 + lane + 32 * k] = accc[gi][k];
      w[2 + kD + lane + 32 * k] = accf[gi][k];
    }
  }
  __syncthreads();
  for (int o = tid; o < G * (2 + r_v + kD); o += kDecThreads) {
    const int gi = o / (2 + r_v + kD), e = o % (2 + r_v + kD);
    float M = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, ws[(w * G + gi) * stride]);
    float v = 0.f;
    if (e == 0) {
      v = M;
    } else {
      for (int w = 0; w < kDecWarps; ++w) {
        const float* ww = ws + (w * G + gi) * stride;
        const float wm = ww[0];
        if (wm == -INFINITY) continue;
        const float f = exp2f(wm - M);
        float x;
        if (e == 1) x = ww[1];
        else if (e < 2 + r_v) x = ww[e];
        else x = ww[2 + kD + (e - 2 - r_v)];
        v += f * x;
      }
    }
    partial_ptr(p, b, h, c, gi, G)[e] = v;
  }

  // the last split of this (b, kv head) merges all splits and lifts by U_v
  __shared__ bool s_last;
  __threadfence();               // every thread's partial writes are visible device-wide
  __syncthreads();
  if (tid == 0) {
    const int done = atomicAdd(p.tickets + bh, 1);
    s_last = (done == n_chunks - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  float* Mg = wts + p.n_chunk_max * G;      // [G] global max, then [G] 1/L
  if (tid < G) {
    float M = -INFINITY;
    for (int cc = 0; cc < n_chunks; ++cc) M = fmaxf(M, __ldcg(partial_ptr(p, b, h, cc, tid, G)));
    float L = 0.f;
    for (int cc = 0; cc < n_chunks; ++cc) {
      const float* pp = partial_ptr(p, b, h, cc, tid, G);
      const float m_c = __ldcg(pp);
      const float wgt = m_c == -INFINITY ? 0.f : exp2f(m_c - M);
      wts[cc * G + tid] = wgt;
      L += wgt * __ldcg(pp + 1);
    }
    Mg[tid] = L > 0.f ? 1.f / L : 0.f;
  }
  __syncthreads();
  // merged acc_c and acc_f into the (now free) per-warp area: [G][r_v + d]
  float* A = ws;
  for (int o = tid; o < G * (r_v + kD); o += kDecThreads) {
    const int gi = o / (r_v + kD), e = o % (r_v + kD);
    float v = 0.f;
    for (int cc = 0; cc < n_chunks; ++cc)
      v = fmaf(wts[cc * G + gi], __ldcg(partial_ptr(p, b, h, cc, gi, G) + 2 + e), v);
    A[o] = v;
  }
  __syncthreads();
  const lrkv_bf16* Uv = p.C.U_v + (size_t)h * kD * r_v;
  for (int o = tid; o < G * kD; o += kDecThreads) {
    const int gi = o / kD, i = o % kD;
    const float* a = A + gi * (r_v + kD);
    float v = a[r_v + i];
    for (int j = 0; j < r_v; ++j) v = fmaf(bf2f(Uv[i * r_v + j]), a[j], v);
    p.out[((size_t)b * D.Hq + h * G + gi) * kD + i] = v * Mg[gi];
  }
  if (tid == 0) p.tickets[bh] = 0;
}

}  // namespace lrkv
