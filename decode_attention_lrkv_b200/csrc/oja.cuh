// OjaKV's online basis update on the GPU (OjaKV repository README, "Method
// Summary > OjaKV": the low-rank subspace follows the context with Oja's
// algorithm, during prefill and during decoding).  The page gives no rule,
// step size or normalisation; the update is Oja's subspace rule (reading R23):
//   y_n = U^T x_n,   U <- U + eta (1/N) sum_n (x_n - U y_n) y_n^T
// over a batch of N rows (one row per decode step), then re-orthonormalised
// by a QR factorisation whose R has a positive diagonal.
//
// With Y = X U the sum is A - U Bm, A = X^T Y (d x r), Bm = Y^T Y (r x r).
//
// Kernel 1, oja_accum_kernel: grid (splits, Hkv), 256 threads.  A CTA streams
// its rows in 64-row tiles (bf16 -> fp32 in shared memory), forms the tile's
// Y = X U, and accumulates A and Bm in registers (fp32); the partial sums go
// to the workspace.
//
// Kernel 2, oja_finish_kernel: one CTA per kv head sums the partials in fp64,
// forms V = U + eta (A - U Bm) / N in fp64 and orthonormalises V's columns by
// Gram-Schmidt with a second orthogonalisation pass (fp64; the diagonal of R
// is the norm, positive), then writes the fp32 basis and its bf16 rounding.
#pragma once

#include "lrkv_common.cuh"

namespace lrkv {
namespace oja {

constexpr int kThreads = 256;
constexpr int kTile = 64;             // rows per tile
constexpr int kFinishThreads = 512;

struct AccumParams {
  const lrkv_bf16* X;   // [n_rows][Hkv][d]
  const float* U;       // [Hkv][d][r] fp32
  int n_rows, Hkv, r;
  int rows_per_split;   // a multiple of kTile
  float* partials;      // [Hkv][splits][d * r + r * r]
};

// Shared memory: U [d][r], X tile [64][d], Y tile [64][r] (fp32).
inline size_t accum_smem_bytes(int r) { return sizeof(float) * ((size_t)kD * r + kTile * kD + kTile * r); }

// RB = r / 16 column blocks.  Thread (ty, tx) = (tid / 16, tid % 16) owns
// A rows ty + 16a (a < 8) x columns tx + 16b (b < RB), Y rows ty + 16a (a < 4)
// x the same columns, and Bm rows tx + 16c x columns ty + 16b.
template <int RB>
__global__ void __launch_bounds__(kThreads) oja_accum_kernel(AccumParams p) {
  extern __shared__ float sm_oja[];
  constexpr int R = RB * 16;
  const int s = blockIdx.x, h = blockIdx.y;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float* Us = sm_oja;                  // [d][R]
  float* Xs = Us + kD * R;             // [64][d]
  float* Ys = Xs + kTile * kD;         // [64][R]
  const float* Ug = p.U + (size_t)h * kD * R;
  for (int e = tid; e < kD * R; e += kThreads) Us[e] = Ug[e];
  float acc_a[8][RB], acc_b[RB][RB];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < RB; ++b) acc_a[a][b] = 0.f;
#pragma unroll
  for (int c = 0; c < RB; ++c)
#pragma unroll
    for (int b = 0; b < RB; ++b) acc_b[c][b] = 0.f;
  const int r0 = s * p.rows_per_split;
  const int r1 = min(p.n_rows, r0 + p.rows_per_split);
  for (int t0 = r0; t0 < r1; t0 += kTile) {
    __syncthreads();   // the previous tile's X and Y are consumed (and U is in)
    // X tile: 16-byte pieces of bf16, widened; rows past the end are zero
    for (int q = tid; q < kTile * kD / 8; q += kThreads) {
      const int n = q / (kD / 8), c8 = (q - n * (kD / 8)) * 8;
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (t0 + n < r1)
        w = *reinterpret_cast<const uint4*>(p.X + ((size_t)(t0 + n) * p.Hkv + h) * kD + c8);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        Xs[n * kD + c8 + 2 * k] = bf_lo(ws[k]);
        Xs[n * kD + c8 + 2 * k + 1] = bf_hi(ws[k]);
      }
    }
    __syncthreads();
    // Y = X U for this tile
    {
      float y[4][RB];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < RB; ++b) y[a][b] = 0.f;
#pragma unroll 4
      for (int i = 0; i < kD; ++i) {
        float xv[4], uv[RB];
#pragma unroll
        for (int a = 0; a < 4; ++a) xv[a] = Xs[(ty + 16 * a) * kD + i];
#pragma unroll
        for (int b = 0; b < RB; ++b) uv[b] = Us[i * R + tx + 16 * b];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < RB; ++b) y[a][b] = fmaf(xv[a], uv[b], y[a][b]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < RB; ++b) Ys[(ty + 16 * a) * R + tx + 16 * b] = y[a][b];
    }
    __syncthreads();
    // A += X^T Y, Bm += Y^T Y over the tile's rows (zero rows add nothing)
#pragma unroll 2
    for (int n = 0; n < kTile; ++n) {
      float xv[8], yv[RB], yc[RB];
#pragma unroll
      for (int a = 0; a < 8; ++a) xv[a] = Xs[n * kD + ty + 16 * a];
#pragma unroll
      for (int b = 0; b < RB; ++b) yv[b] = Ys[n * R + tx + 16 * b];
#pragma unroll
      for (int b = 0; b < RB; ++b) yc[b] = Ys[n * R + ty + 16 * b];
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < RB; ++b) acc_a[a][b] = fmaf(xv[a], yv[b], acc_a[a][b]);
#pragma unroll
      for (int c = 0; c < RB; ++c)
#pragma unroll
        for (int b = 0; b < RB; ++b) acc_b[c][b] = fmaf(yv[c], yc[b], acc_b[c][b]);
    }
  }
  float* out = p.partials + ((size_t)h * gridDim.x + s) * ((size_t)kD * R + R * R);
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < RB; ++b) out[(ty + 16 * a) * R + tx + 16 * b] = acc_a[a][b];
  // Bm[j][k]: thread holds j = tx + 16c, k = ty + 16b
#pragma unroll
  for (int c = 0; c < RB; ++c)
#pragma unroll
    for (int b = 0; b < RB; ++b) out[kD * R + (tx + 16 * c) * R + ty + 16 * b] = acc_b[c][b];
}

struct FinishParams {
  const float* partials;   // [Hkv][splits][d * r + r * r]
  int splits, r, n_rows;
  float eta;
  float* U;                // [Hkv][d][r] fp32, in and out
  lrkv_bf16* U_bf16;       // nullable [Hkv][d][r]
};

// Shared memory: V [d][r] fp64, dots [r] fp64, norm, Bm [r][r] (summed in fp64, kept as fp32).
inline size_t finish_smem_bytes(int r) {
  return sizeof(double) * ((size_t)kD * r + r + 8) + sizeof(float) * (size_t)r * r;
}

__global__ void __launch_bounds__(kFinishThreads) oja_finish_kernel(FinishParams p) {
  extern __shared__ double sm_fin[];
  const int h = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kWarps = kFinishThreads / 32;
  const int R = p.r;
  double* V = sm_fin;               // [d][R]
  double* dots = V + kD * R;        // [R]
  double* nrm = dots + R;           // [1], padded to 8
  float* Bm = reinterpret_cast<float*>(nrm + 8);   // [R][R]
  const size_t stride = (size_t)kD * R + (size_t)R * R;
  const float* part = p.partials + (size_t)h * p.splits * stride;
  float* Ug = p.U + (size_t)h * kD * R;
  // the partial sums, in fp64: V = A for now, Bm
  for (int e = tid; e < kD * R; e += kFinishThreads) {
    double a = 0.0;
    for (int s = 0; s < p.splits; ++s) a += (double)part[s * stride + e];
    V[e] = a;
  }
  for (int e = tid; e < R * R; e += kFinishThreads) {
    double a = 0.0;
    for (int s = 0; s < p.splits; ++s) a += (double)part[s * stride + kD * R + e];
    Bm[e] = (float)a;
  }
  __syncthreads();
  // V = U + eta (A - U Bm) / N
  const double step = (double)p.eta / (double)p.n_rows;
  for (int e = tid; e < kD * R; e += kFinishThreads) {
    const int i = e / R, j = e - i * R;
    double ub = 0.0;
    for (int k = 0; k < R; ++k) ub += (double)Ug[i * R + k] * (double)Bm[k * R + j];
    V[e] = (double)Ug[e] + step * (V[e] - ub);   // this thread's own element
  }
  __syncthreads();
  // Gram-Schmidt, each column orthogonalised twice against the earlier ones
  for (int j = 0; j < R; ++j) {
    for (int pass = 0; pass < 2; ++pass) {
      for (int k = warp; k < j; k += kWarps) {
        double sdot = 0.0;
        for (int i = lane; i < kD; i += 32) sdot += V[i * R + k] * V[i * R + j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, o);
        if (lane == 0) dots[k] = sdot;
      }
      __syncthreads();
      if (tid < kD) {
        double v = V[tid * R + j];
        for (int k = 0; k < j; ++k) v -= dots[k] * V[tid * R + k];
        V[tid * R + j] = v;
      }
      __syncthreads();
    }
    if (warp == 0) {
      double ss = 0.0;
      for (int i = lane; i < kD; i += 32) ss += V[i * R + j] * V[i * R + j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) nrm[0] = ss > 0.0 ? 1.0 / sqrt(ss) : 0.0;
    }
    __syncthreads();
    if (tid < kD) V[tid * R + j] *= nrm[0];
    __syncthreads();
  }
  for (int e = tid; e < kD * R; e += kFinishThreads) {
    Ug[e] = (float)V[e];
    if (p.U_bf16) p.U_bf16[(size_t)h * kD * R + e] = __bfloat16_as_ushort(__double2bfloat16(V[e]));
  }
}

}  // namespace oja
}  // namespace lrkv
