// StaticPCA's offline basis on the GPU: per kv head, the top-r eigenvectors of
// the scatter matrix G = X^T X of calibration rows (OjaKV repository README,
// "Method Summary > StaticPCA": an offline low-rank basis computed from a
// calibration corpus; KV-CoRE page, abstract: the optimal low-rank
// approximation under the Frobenius norm, which by Eckart-Young is the span of
// G's leading eigenvectors).  No mean-centring (c = U^T x).
//
// Kernel 1, gram_kernel: grid (splits, Hkv).  A CTA accumulates its rows' share
// of G in fp32 on the tensor cores (mma.sync m16n8k16, bf16 inputs are exact
// products): warp w owns rows [16w, 16w + 16) of G, all 128 columns; rows of X
// stream through a two-stage cp.async ring of 64-token tiles, and both MMA
// operands are X^T slices loaded with ldmatrix.trans.  Partial Gram matrices go
// to the workspace.
//
// Kernel 2, eig_kernel: one CTA per kv head sums the partials in fp64 and runs
// cyclic Jacobi on the 128 x 128 symmetric matrix (Golub & Van Loan's
// two-by-two symmetric Schur rotation), 64 disjoint pairs per round in the
// round-robin order, fp64 matrix and fp32 eigenvectors in shared memory, until
// the off-diagonal mass falls below 1e-26 of the diagonal's or 16 sweeps.
// Eigenvalues are sorted descending; each of the first r eigenvectors is
// signed so that its largest-magnitude entry is positive (lowest index on a
// tie) and stored as bf16 (round to nearest even) into U[h][d][r].
#pragma once

#include "lrkv_common.cuh"
#include "ptx.cuh"

namespace lrkv {
namespace fit {

constexpr int kThreads = 256;            // gram_kernel: 8 warps
constexpr int kTileRows = 64;            // tokens per ring stage
constexpr int kRowStride = 2 * kD + 16;  // padded smem row (bytes): conflict-free ldmatrix
constexpr int kStageBytes = kTileRows * kRowStride;
constexpr int kEigThreads = 512;
constexpr int kMaxSweeps = 16;

struct GramParams {
  const lrkv_bf16* X;   // [n_rows][Hkv][d]
  int n_rows;
  int Hkv;
  int rows_per_split;   // a multiple of kTileRows
  float* partials;      // [Hkv][splits][d][d]
};

__global__ void __launch_bounds__(kThreads, 1) gram_kernel(GramParams p) {
  extern __shared__ __align__(128) unsigned char sm_fit[];
  const int s = blockIdx.x, h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3, lm = lane >> 3, lr = lane & 7;
  const int r0 = s * p.rows_per_split;
  const int r1 = min(p.n_rows, r0 + p.rows_per_split);
  const int n_tiles = r1 > r0 ? (r1 - r0 + kTileRows - 1) / kTileRows : 0;
  const size_t row_pitch = (size_t)p.Hkv * kD;   // elements between two tokens' rows

  // one 64 x 128 tile into stage st: 16-byte pieces, rows past r1 zero-filled
  auto load = [&](int tile, int st) {
    unsigned char* dst = sm_fit + st * kStageBytes;
    const int base = r0 + tile * kTileRows;
    for (int q = tid; q < kTileRows * 16; q += kThreads) {
      const int row = q >> 4, piece = q & 15;
      const int tok = base + row;
      const bool on = tok < r1;
      const lrkv_bf16* src = p.X + ((size_t)(on ? tok : r0) * row_pitch + (size_t)h * kD) + piece * 8;
      cp_async16_zfill(dst + row * kRowStride + piece * 16, src, on ? 16u : 0u);
    }
    cp_async_commit();
  };

  float acc[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  if (n_tiles > 0) load(0, 0);
  for (int i = 0; i < n_tiles; ++i) {
    if (i + 1 < n_tiles) load(i + 1, (i + 1) & 1);
    else cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const unsigned char* tile = sm_fit + (i & 1) * kStageBytes;
#pragma unroll
    for (int kk = 0; kk < kTileRows; kk += 16) {
      // A (rows = G rows 16w.., k = tokens) = X^T: 8x8 blocks of X (rows tokens) transposed
      uint32_t a0, a1, a2, a3;
      ldsm_x4_t(a0, a1, a2, a3,
                tile + (kk + (lm >> 1) * 8 + lr) * kRowStride + (16 * warp + (lm & 1) * 8) * 2);
#pragma unroll
      for (int n2 = 0; n2 < 8; ++n2) {   // G columns [16 n2, 16 n2 + 16): two n-tiles
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(b0, b1, b2, b3,
                  tile + (kk + (lm & 1) * 8 + lr) * kRowStride + (16 * n2 + (lm >> 1) * 8) * 2);
        mma_16816(acc[2 * n2], a0, a1, a2, a3, b0, b1);
        mma_16816(acc[2 * n2 + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();   // the stage is refilled two steps later
  }
  cp_async_wait<0>();
  float* out = p.partials + ((size_t)h * gridDim.x + s) * kD * kD;
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    const int row = 16 * warp + g, col = 8 * n + 2 * t;
    out[row * kD + col] = acc[n][0];
    out[row * kD + col + 1] = acc[n][1];
    out[(row + 8) * kD + col] = acc[n][2];
    out[(row + 8) * kD + col + 1] = acc[n][3];
  }
}

struct EigParams {
  const float* partials;   // [Hkv][splits][d][d]
  int splits;
  int r;
  lrkv_bf16* U;            // [Hkv][d][r]
  float* eigvals;          // [Hkv][d] descending, nullable
};

// shared memory: A fp64 [d][d + 1], V fp32 [d][d + 1] (padded rows: the column
// updates of a warp hit distinct banks), rotations [64][2] fp64, scratch
constexpr int kAS = kD + 1;
inline size_t eig_smem_bytes() {
  return sizeof(double) * kD * kAS + sizeof(float) * kD * (kD + 1) + sizeof(double) * 2 * (kD / 2) +
         sizeof(double) * 2 * kEigThreads + sizeof(int) * kD + 64;
}

__global__ void __launch_bounds__(kEigThreads, 1) eig_kernel(EigParams p) {
  extern __shared__ __align__(16) unsigned char sm_eig[];
  double* A = reinterpret_cast<double*>(sm_eig);                  // [d][kAS]
  float* V = reinterpret_cast<float*>(A + kD * kAS);              // [d][d + 1]
  double* cs = reinterpret_cast<double*>(V + kD * (kD + 1));      // [64][2]
  double* red = cs + kD;                                          // [2][kEigThreads]
  int* rank = reinterpret_cast<int*>(red + 2 * kEigThreads);      // [d]
  constexpr int VS = kD + 1;
  const int h = blockIdx.x, tid = threadIdx.x;

  // G = sum of the partials (fp64), made exactly symmetric; V = I
  const float* part = p.partials + (size_t)h * p.splits * kD * kD;
  for (int e = tid; e < kD * kD; e += kEigThreads) {
    const int i = e / kD, j = e % kD;
    double x = 0.0, y = 0.0;
    for (int s = 0; s < p.splits; ++s) {
      x += (double)part[(size_t)s * kD * kD + i * kD + j];
      y += (double)part[(size_t)s * kD * kD + j * kD + i];
    }
    A[i * kAS + j] = 0.5 * (x + y);
    V[i * VS + j] = i == j ? 1.f : 0.f;
  }
  __syncthreads();

  for (int sweep = 0; sweep < kMaxSweeps; ++sweep) {
    // off-diagonal and diagonal mass: stop when the former is negligible
    double off = 0.0, dia = 0.0;
    for (int e = tid; e < kD * kD; e += kEigThreads) {
      const double a = A[(e / kD) * kAS + e % kD];
      if (e / kD == e % kD) dia += a * a;
      else off += a * a;
    }
    red[tid] = off;
    red[kEigThreads + tid] = dia;
    __syncthreads();
    for (int w = kEigThreads / 2; w > 0; w >>= 1) {
      if (tid < w) {
        red[tid] += red[tid + w];
        red[kEigThreads + tid] += red[kEigThreads + tid + w];
      }
      __syncthreads();
    }
    const bool done = red[0] <= 1e-26 * red[kEigThreads];
    __syncthreads();
    if (done) break;
    for (int rd = 0; rd < kD - 1; ++rd) {
      // round-robin pairing: index 0 fixed, 1..127 rotated by rd; pair i = (pos i, pos 127 - i)
      auto pos = [&](int i) { return i == 0 ? 0 : 1 + (i - 1 + rd) % (kD - 1); };
      if (tid < kD / 2) {   // the two-by-two symmetric Schur rotation of each pair
        const int pp = pos(tid), qq = pos(kD - 1 - tid);
        const double apq = A[pp * kAS + qq];
        double c = 1.0, sn = 0.0;
        if (apq != 0.0) {
          const double tau = (A[qq * kAS + qq] - A[pp * kAS + pp]) / (2.0 * apq);
          const double tt = tau >= 0.0 ? 1.0 / (tau + sqrt(1.0 + tau * tau))
                                       : -1.0 / (-tau + sqrt(1.0 + tau * tau));
          c = 1.0 / sqrt(1.0 + tt * tt);
          sn = tt * c;
        }
        cs[2 * tid] = c;
        cs[2 * tid + 1] = sn;
      }
      __syncthreads();
      // rows p, q of J^T A
      for (int e = tid; e < (kD / 2) * kD; e += kEigThreads) {
        const int pi = e / kD, j = e % kD;
        const int pp = pos(pi), qq = pos(kD - 1 - pi);
        const double c = cs[2 * pi], sn = cs[2 * pi + 1];
        const double ap = A[pp * kAS + j], aq = A[qq * kAS + j];
        A[pp * kAS + j] = c * ap - sn * aq;
        A[qq * kAS + j] = sn * ap + c * aq;
      }
      __syncthreads();
      // columns p, q of (J^T A) J, and of V J
      for (int e = tid; e < (kD / 2) * kD; e += kEigThreads) {
        const int pi = e / kD, i = e % kD;
        const int pp = pos(pi), qq = pos(kD - 1 - pi);
        const double c = cs[2 * pi], sn = cs[2 * pi + 1];
        const double ap = A[i * kAS + pp], aq = A[i * kAS + qq];
        A[i * kAS + pp] = c * ap - sn * aq;
        A[i * kAS + qq] = sn * ap + c * aq;
        const float vp = V[i * VS + pp], vq = V[i * VS + qq];
        V[i * VS + pp] = (float)c * vp - (float)sn * vq;
        V[i * VS + qq] = (float)sn * vp + (float)c * vq;
      }
      __syncthreads();
    }
  }

  // eigenvalues on the diagonal; rank descending (lower index first on a tie)
  if (tid < kD) {
    const double li = A[tid * kAS + tid];
    int rk = 0;
    for (int j = 0; j < kD; ++j) {
      const double lj = A[j * kAS + j];
      rk += (lj > li) || (lj == li && j < tid);
    }
    rank[tid] = rk;
    if (p.eigvals) p.eigvals[(size_t)h * kD + rk] = (float)li;
  }
  __syncthreads();
  // the first r eigenvectors: warp w takes columns i with rank < r, w, w + 16, ...
  const int warp = tid >> 5, lane = tid & 31;
  for (int i = warp; i < kD; i += kEigThreads / 32) {
    const int k = rank[i];
    if (k >= p.r) continue;
    // entry of largest magnitude, the lowest index on a tie
    float best = -1.f;
    int bi = kD;
    for (int row = lane; row < kD; row += 32) {
      const float a = fabsf(V[row * VS + i]);
      if (a > best || (a == best && row < bi)) best = a, bi = row;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob > best || (ob == best && oi < bi)) best = ob, bi = oi;
    }
    const float sg = V[bi * VS + i] < 0.f ? -1.f : 1.f;
    for (int row = lane; row < kD; row += 32)
      p.U[((size_t)h * kD + row) * p.r + k] = f2bf(sg * V[row * VS + i]);
  }
}

}  // namespace fit
}  // namespace lrkv
