// Read path, B200 version: split-K decode attention over the compressed
// cache, logits and value sums on the tensor cores.
//
// Coefficient-space form of the StaticPCA read path (OjaKV repository
// README, "Method Summary > StaticPCA": keys and values reconstructed on the
// fly for standard attention).  With q~ = U_k^T q, a compressed token's logit
// is q~ . c_k / sqrt(d) and its value contribution is accumulated in r_v
// space, lifted by U_v once per split; full-rank tokens ("Method Summary >
// OjaKV", hybrid storage) use their stored rows.  One softmax covers both.
//
// Why mma.sync: per kv head the work is [tokens x r] x [r x g] and
// [r x tokens] x [tokens x g] with g <= 4 query heads.  On CUDA cores that is
// tens of instructions per token and the kernel is issue-bound far below the
// HBM roof; as m16n8k16 MMAs it is a handful.  Tokens are the M dimension and
// the query heads the N dimension: q~ and the probabilities p are fp32, so
// each is split into a bf16 high part (columns 0..3) and low part (columns
// 4..7) and the two columns of a head are summed afterwards -- fp32-level
// accuracy.  tcgen05 wants M >= 64 per instruction and a single issuing
// thread; here N is 8 and the contraction per tile is tiny, so the
// warp-level MMA keeps the whole per-token chain inside one warp.
//
// Work split.  Grid (splits, Hkv, B), one CTA of 8 warps per SM (255
// registers per thread).  A CTA takes positions [c*chunk, (c+1)*chunk) of one
// (batch row, kv head) and an equal share of its full-rank list.  Each warp
// streams its own tiles through a 2-stage cp.async ring:
//   - a compressed tile is 32 consecutive positions, copied in place with
//     16-byte pieces, consecutive lanes on consecutive bytes; a routed
//     position (mask bit set) or one past the end is zero-filled instead of
//     read, and its logit is -inf;
//   - a full-rank tile is 16 list rows (keys, then values).
// Rows land in padded shared-memory rows (stride 2r+16 bytes) so ldmatrix is
// conflict-free.  Three ring stages where shared memory allows, else two.
// At the end each warp leaves its partial softmax state in its own slot, the
// CTA merges its warps, lifts its value sum on the tensor cores
// (U_v acc_c + acc_f) and writes one record (m, l, o[d]) per query head; the
// last CTA of the (batch row, kv head) (atomic ticket, no waiting) merges the
// records in registers, straight from L2: o = sum_c w_c o_c / sum_c w_c l_c.
//
// Programmatic dependent launch: the bases U_k and U_v are loaded before
// waiting on the preceding kernel of the stream (they are not written by the
// kernels around a decode); the query, produced upstream, and every piece of
// cache state (an append to the same cache may precede) are read after it.
// Every CTA lets the next kernel launch right after its own base loads.
#pragma once

#include <type_traits>

#include "decode_simple.cuh"
#include "lrkv_common.cuh"
#include "ptx.cuh"

namespace lrkv {
namespace ds {

constexpr int kTileC = 32;                       // positions per compressed tile (one mask word)
constexpr int kTileF = 16;                       // rows per full-rank tile
constexpr int kMaxChunk = kMaxDecodeChunk;       // positions per split (mask words in smem)
constexpr unsigned kFull = 0xffffffffu;

constexpr int al16(int x) { return (x + 15) & ~15; }
constexpr int al128(int x) { return (x + 127) & ~127; }
constexpr int imax(int a, int b) { return a > b ? a : b; }

// W warps per CTA and NS ring stages per warp: per shape, as many warps as
// shared memory allows with U_v resident beside the ring.
// x (a multiple of 16) raised to an odd multiple of 16: rows that far apart
// put the 8 rows an ldmatrix reads in distinct shared-memory banks
constexpr int odd16(int x) { return (x / 16) % 2 ? x : x + 16; }

// CB: bits of a stored coefficient, 16 (bf16), 8 or 4 (int8 / int4 codes
// with per-row fp32 scales).
template <int G, int RK, int RV, int W, int NS, int CB = 16>
struct Shape {
  static_assert(G == 1 || G == 2 || G == 4, "1, 2 or 4 query heads per kv head");
  static_assert(RK % 16 == 0 && RV % 16 == 0 && RK <= kD && RV <= kD, "ranks");
  static_assert(W >= 8 && NS >= 2, "at least 8 warps and 2 ring stages");
  static_assert(CB == 16 || CB == 8 || CB == 4, "bf16 coefficients or int8 / int4 codes");
  static constexpr int kWarps = W;
  static constexpr int kThreads = W * 32;
  // the bases in shared memory: bf16 rows, padded
  static constexpr int UKP = RK / 8, UVP = RV / 8;  // 16-byte pieces per basis row
  static constexpr int KS = 2 * RK + 16;           // padded basis row strides (bytes)
  static constexpr int VS = 2 * RV + 16;
  // a compressed tile: 32 stored rows of keys, then of values, then (codes
  // only) their 32 + 32 fp32 scales
  static constexpr int TKB = RK * CB / 8, TVB = RV * CB / 8;   // bytes per stored row
  // bf16 and int8 rows are copied piece by piece into padded rows (16-byte
  // pieces per row; routed rows zero-filled); int4 rows (8 bytes per 16 codes)
  // are copied as the tile's flat block (16-byte pieces per tile) and read
  // with plain shared loads, rows TKB apart
  static constexpr int KP = CB == 4 ? 2 * TKB : TKB / 16;     // pieces per row, or per tile / 16
  static constexpr int VP = CB == 4 ? 2 * TVB : TVB / 16;
  static constexpr int TKS = CB == 4 ? TKB : odd16(TKB);      // tile row strides
  static constexpr int TVS = CB == 4 ? TVB : odd16(TVB);
  static constexpr int T_SC = kTileC * (TKS + TVS);           // scales: [2][32] fp32
  static constexpr int FS = 2 * kD + 16;
  static constexpr int SLOT_C = T_SC + (CB < 16 ? 2 * kTileC * 4 : 0);
  static constexpr int SLOT_F = kTileF * 2 * FS;
  static constexpr int SLOT = al128(imax(SLOT_C, SLOT_F));
  static constexpr int MASK_BYTES = (kMaxChunk / 32) * 4;          // mask words
  static constexpr int SMEM_MAX = 227 * 1024 - 2048;               // static shared memory aside
  static constexpr int STAGES = NS;
  static constexpr int RING = W * NS * SLOT;                      // [stage][warp][SLOT]
  static constexpr int OFF_MASK = RING;
  // U_v rows [d][VS], resident beside the ring (loaded in the prologue) for
  // the per-warp lift
  static constexpr int OFF_UV = RING + MASK_BYTES;
  static constexpr int SMEM = OFF_UV + kD * VS;
  static_assert(SMEM <= SMEM_MAX, "shared memory of one CTA");
  // U_k rows [d][KS] (the query-side basis U_kq when the cache has one) live in
  // the last stage until every warp has its q~; with an attention-aware key
  // basis the fused append also needs the key-side U_k: second copy behind it
  static constexpr int OFF_UK = (NS - 1) * W * SLOT;
  static constexpr int OFF_UK2 = OFF_UK + al16(kD * KS);
  static_assert(kD * KS <= W * SLOT, "U_k fits in one stage");
  // per-warp partial state in the warp's stage-0 slot (floats)
  static constexpr int W_PF = 0;                    // [G][d]
  static constexpr int W_M = W_PF + G * kD;         // [G]
  static constexpr int W_L = W_M + G;               // [G]
  static_assert((W_L + G) * 4 <= SLOT, "partials fit in a slot");
  // record of one split per query head: m, l, flag, pad, o[d] = U_v acc_c + acc_f
  // (flag, head 0 only: the split appended a full-rank row, fused append)
  static constexpr int REC = 4 + kD;
  // fused append scratch behind the two key bases in the last stage (untouched
  // until the stream's first refill), floats: c_k [RK], c_v [RV], q~ (scaled)
  // [G][RK], x [2][d] (key, value), the key minus its mean [d], sums [24]
  static constexpr int OFF_APP = OFF_UK2 + al16(kD * KS);
  static constexpr int A_CK = 0, A_CV = RK, A_QT = RK + RV, A_X = A_QT + G * RK,
                       A_XC = A_X + 2 * kD, A_RED = A_XC + kD, A_QR = A_RED + 24,
                       A_FLOATS = A_QR + 8;
  static_assert(2 * al16(kD * KS) + A_FLOATS * 4 <= W * SLOT,
                "both key bases and the append scratch fit in a stage");
};

// The append CTA's work in a fused decode-time append: one new token of row b,
// kv head h, at position pos, with every thread of the CTA (the StaticPCA
// write path and the OjaKV hybrid policy, as in the append kernel):
//   c_k = U_k^T k and c_v = U_v^T v on the tensor cores (x as an A row,
//   exact in bf16, fp32 accumulation); e = max(||k - U_k c_k|| / ||k||,
//   ||v - U_v c_v|| / ||v||) by direct reconstruction from the unrounded c;
//   routed iff e > tau: the rows go to list slot F when there is room (the
//   mask bit set), else the token stays compressed (FULL_OVERFLOW).  bf16(c),
//   or its per-row codes and scale (CB 8 or 4), is stored at pos either way.
//   Then the token's base-2 logit per head and its value row (v, or c_v as
//   stored) for the fold after the stream.
template <typename S, int G, int RK, int RV, int CB>
__device__ __forceinline__ void append_token(const DecodeParams& p, float* app,
                                             const unsigned char* uk, const unsigned char* ukq,
                                             const unsigned char* uv, const float* s_bias,
                                             int b, int h, size_t bh, int pos, int F, float scale,
                                             uint16_t xe, float* s_new, float* s_vals, int* s_keep) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3, lm = lane >> 3, lr = lane & 7;
  const lrkv_dims& D = p.D;
  constexpr int KST = RK / 16, MVT = RV / 16;
  app[S::A_X + tid] = bf2f(xe);   // new key (threads < d) and value (threads >= d) rows
  // the key as projected: minus the key mean of an attention-aware basis
  if (tid < kD) app[S::A_XC + tid] = bf2f(xe) - (p.C.mu_k ? p.C.mu_k[(size_t)h * kD + tid] : 0.f);
  __syncthreads();                // x and q~ in; the bases in since the prologue
  // c = U^T (x - mu) on the tensor cores: x (bf16, exact) is row 8 of the A
  // operand; a key mean (fp32) enters as its bf16 high and low parts in rows 9
  // and 10, so U^T mu is fp32-accurate and c = row 8 - (row 9 + row 10).  Warp
  // w forms columns [16w, 16w + 16) of c_k (w < r_k / 16) and of c_v (w < r_v / 16),
  // the two products interleaved and the even and odd k-steps in separate
  // accumulators (short chains of dependent MMAs).
  const float* mu_h = p.C.mu_k ? p.C.mu_k + (size_t)h * kD : nullptr;
  {
    const bool do_k = warp < KST, do_v = warp < MVT;
    float ak[2][2][4], av[2][2][4];   // [k-step parity][column half][fragment]
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) ak[q][u][e] = av[q][u][e] = 0.f;
    const float* xk = app + S::A_X;
    const float* xv = app + S::A_X + kD;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int i0 = ks * 16 + 2 * t, i1 = i0 + 8;
      if (do_k) {
        uint32_t x0 = 0u, x1 = 0u;
        if (g == 0) {
          x0 = pack_bf16(xk[i0], xk[i0 + 1]);
          x1 = pack_bf16(xk[i1], xk[i1 + 1]);
        } else if (mu_h && g <= 2) {
          const bool lo = g == 2;
          x0 = pack_bf16(bf16_part(mu_h[i0], lo), bf16_part(mu_h[i0 + 1], lo));
          x1 = pack_bf16(bf16_part(mu_h[i1], lo), bf16_part(mu_h[i1 + 1], lo));
        }
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(b0, b1, b2, b3, uk + (ks * 16 + (lm & 1) * 8 + lr) * S::KS + (16 * warp + (lm >> 1) * 8) * 2);
        mma_16816(ak[ks & 1][0], 0u, x0, 0u, x1, b0, b1);
        mma_16816(ak[ks & 1][1], 0u, x0, 0u, x1, b2, b3);
      }
      if (do_v) {
        const uint32_t x0 = g == 0 ? pack_bf16(xv[i0], xv[i0 + 1]) : 0u;
        const uint32_t x1 = g == 0 ? pack_bf16(xv[i1], xv[i1 + 1]) : 0u;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(b0, b1, b2, b3, uv + (ks * 16 + (lm & 1) * 8 + lr) * S::VS + (16 * warp + (lm >> 1) * 8) * 2);
        mma_16816(av[ks & 1][0], 0u, x0, 0u, x1, b0, b1);
        mma_16816(av[ks & 1][1], 0u, x0, 0u, x1, b2, b3);
      }
    }
    if (do_k) {
      float m[4] = {0.f, 0.f, 0.f, 0.f};   // U^T mu: rows 9 and 10, from lanes 4 + t and 8 + t
      const float v[4] = {ak[0][0][2] + ak[1][0][2], ak[0][0][3] + ak[1][0][3],
                          ak[0][1][2] + ak[1][1][2], ak[0][1][3] + ak[1][1][3]};
      if (mu_h) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          m[e] = __shfl_sync(kFull, v[e], (lane + 4) & 31) + __shfl_sync(kFull, v[e], (lane + 8) & 31);
      }
      if (g == 0) {
        float* cdst = app + S::A_CK;
        cdst[16 * warp + 2 * t] = v[0] - m[0];
        cdst[16 * warp + 2 * t + 1] = v[1] - m[1];
        cdst[16 * warp + 8 + 2 * t] = v[2] - m[2];
        cdst[16 * warp + 8 + 2 * t + 1] = v[3] - m[3];
      }
    }
    if (do_v && g == 0) {
      float* cdst = app + S::A_CV;
      cdst[16 * warp + 2 * t] = av[0][0][2] + av[1][0][2];
      cdst[16 * warp + 2 * t + 1] = av[0][0][3] + av[1][0][3];
      cdst[16 * warp + 8 + 2 * t] = av[0][1][2] + av[1][1][2];
      cdst[16 * warp + 8 + 2 * t + 1] = av[0][1][3] + av[1][1][3];
    }
  }
  __syncthreads();
  // direct reconstruction x_hat = U c on the tensor cores: A = U's rows
  // [16w, 16w + 16) (warp w), B = c split into bf16 high (column 0) and low
  // (column 1) parts; lane (g, t = 0) gets x_hat of rows 16w + g and 16w + g + 8
  // as the sum of its two columns.  Keys and values interleaved, even and odd
  // k-steps in separate accumulators.
  {
    float rk_acc[2][4], rv_acc[2][4];
#pragma unroll
    for (int q = 0; q < 2; ++q)
#pragma unroll
      for (int e = 0; e < 4; ++e) rk_acc[q][e] = rv_acc[q][e] = 0.f;
    const bool lo = g & 1;
    auto bfrag = [&](const float* c2, uint32_t& b0, uint32_t& b1) {
      b0 = g < 2 ? pack_bf16(bf16_part(c2[0], lo), bf16_part(c2[1], lo)) : 0u;
      b1 = g < 2 ? pack_bf16(bf16_part(c2[8], lo), bf16_part(c2[9], lo)) : 0u;
    };
    constexpr int KS_MAX = KST > MVT ? KST : MVT;
#pragma unroll
    for (int ks = 0; ks < KS_MAX; ++ks) {
      if (ks < KST) {
        uint32_t a0, a1, a2, a3, b0, b1;
        ldsm_x4(a0, a1, a2, a3, ukq + (16 * warp + (lm & 1) * 8 + lr) * S::KS + (ks * 16 + (lm >> 1) * 8) * 2);
        bfrag(app + S::A_CK + ks * 16 + 2 * t, b0, b1);
        mma_16816(rk_acc[ks & 1], a0, a1, a2, a3, b0, b1);
      }
      if (ks < MVT) {
        uint32_t a0, a1, a2, a3, b0, b1;
        ldsm_x4(a0, a1, a2, a3, uv + (16 * warp + (lm & 1) * 8 + lr) * S::VS + (ks * 16 + (lm >> 1) * 8) * 2);
        bfrag(app + S::A_CV + ks * 16 + 2 * t, b0, b1);
        mma_16816(rv_acc[ks & 1], a0, a1, a2, a3, b0, b1);
      }
    }
    float rk = 0.f, rv = 0.f;
    if (t == 0) {
      const float* xk = app + S::A_XC;
      const float* xv = app + S::A_X + kD;
      const float k0 = xk[16 * warp + g] - ((rk_acc[0][0] + rk_acc[1][0]) + (rk_acc[0][1] + rk_acc[1][1]));
      const float k1 = xk[16 * warp + g + 8] - ((rk_acc[0][2] + rk_acc[1][2]) + (rk_acc[0][3] + rk_acc[1][3]));
      const float v0 = xv[16 * warp + g] - ((rv_acc[0][0] + rv_acc[1][0]) + (rv_acc[0][1] + rv_acc[1][1]));
      const float v1 = xv[16 * warp + g + 8] - ((rv_acc[0][2] + rv_acc[1][2]) + (rv_acc[0][3] + rv_acc[1][3]));
      rk = k0 * k0 + k1 * k1;
      rv = v0 * v0 + v1 * v1;
    }
    const float x = app[S::A_X + tid];
    float ns = x * x;   // warps < 4: the key's squares, else the value's
    // the three warp sums together (independent shuffles)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      rk += __shfl_xor_sync(kFull, rk, o);
      rv += __shfl_xor_sync(kFull, rv, o);
      ns += __shfl_xor_sync(kFull, ns, o);
    }
    if (lane == 0) {
      app[S::A_RED + warp] = rk;
      app[S::A_RED + 8 + warp] = rv;
      app[S::A_RED + 16 + warp] = ns;
    }
  }
  __syncthreads();
  const float* red = app + S::A_RED;   // [3][8]: key residual, value residual, squares per warp
  float rk = 0.f, rv = 0.f, nk = 0.f, nv = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) rk += red[w], rv += red[8 + w];
#pragma unroll
  for (int w = 0; w < 4; ++w) nk += red[16 + w], nv += red[20 + w];
  const float e = fmaxf(nk > 0.f ? sqrtf(rk / nk) : 0.f, nv > 0.f ? sqrtf(rv / nv) : 0.f);
  const bool routed = e > p.tau;
  const bool keep = routed && F < D.F_cap;
  {  // the stored rows: thread j of each half owns column j of its tensor's row
    const bool kside = tid < kD;
    const int j = tid & (kD - 1), r = kside ? RK : RV;
    float* cval = app + (kside ? S::A_CK : S::A_CV) + j;
    const size_t row = bh * D.T_cap + pos;
    const float cb = j < r ? bf16_round(*cval) : 0.f;
    if constexpr (CB == 16) {
      if (j < r) reinterpret_cast<uint16_t*>(kside ? p.C.coef_k : p.C.coef_v)[row * r + j] = f2bf(cb);
      if (j < r) *cval = cb;
    } else {   // per-row codes: the row's amax over its half's warps, one code per column
      const float wm = warp_max(fabsf(cb));
      if (lane == 0) app[S::A_QR + warp] = wm;
      __syncthreads();
      const float* qr = app + S::A_QR + (kside ? 0 : 4);
      const float s = quant_scale(fmaxf(fmaxf(qr[0], qr[1]), fmaxf(qr[2], qr[3])), CB);
      const int qv = quant_code(cb, s, CB);
      const int qn = __shfl_down_sync(kFull, qv, 1);   // the odd neighbour's code (4-bit pairs)
      unsigned char* codes = static_cast<unsigned char*>(kside ? p.C.coef_k : p.C.coef_v) +
                             row * (size_t)(r * CB / 8);
      if (j < r) {
        if (CB == 8) codes[j] = (unsigned char)(qv & 0xff);
        else if ((j & 1) == 0) codes[j >> 1] = (unsigned char)((qv & 0xf) | ((qn & 0xf) << 4));
        *cval = s * (float)qv;   // the coefficient as the decode reads it
      }
      if (j == 0) (kside ? p.C.scale_k : p.C.scale_v)[row] = s;
    }
  }
  __syncthreads();   // every stored coefficient in, for the token's logit and value row
  if (keep) {
    if (tid < kD) reinterpret_cast<uint16_t*>(p.C.full_k)[(bh * D.F_cap + F) * kD + tid] = xe;
    else reinterpret_cast<uint16_t*>(p.C.full_v)[(bh * D.F_cap + F) * kD + tid - kD] = xe;
  }
  if (tid == 0) {
    uint32_t* mword = p.C.route_mask + bh * (D.T_cap / 32) + (pos >> 5);
    const uint32_t bit = 1u << (pos & 31);
    if (keep) {
      red_or_u32(mword, bit);
      p.C.full_idx[bh * D.F_cap + F] = pos;
    } else {
      red_and_u32(mword, ~bit);
    }
    if (routed && !keep) atomicOr(p.C.dev_status, LRKV_DEV_FULL_OVERFLOW);
    if (p.err_out) p.err_out[bh] = e;
    *s_keep = keep;
  }
  if (warp < G && warp < p.g_all - p.g_off) {   // the token's logit for query head `warp`, base 2
    float sd = 0.f;
    if (keep) {     // full rank: q . k / sqrt(d)
      const uint16_t* qrow = reinterpret_cast<const uint16_t*>(p.q) +
                             ((size_t)b * D.Hq + (size_t)h * p.g_all + p.g_off + warp) * kD;
      for (int i = lane; i < kD; i += 32) sd = fmaf(bf2f(qrow[i]), app[S::A_X + i], sd);
      sd = warp_sum(sd) * scale;
    } else {        // compressed: q . mu_k + q~ . c_k as stored, both already scaled
      for (int j = lane; j < RK; j += 32) sd = fmaf(app[S::A_QT + warp * RK + j], app[S::A_CK + j], sd);
      sd = warp_sum(sd) + s_bias[warp];
    }
    if (lane == 0) s_new[warp] = sd;
  } else if (warp < G && lane == 0) {
    s_new[warp] = -INFINITY;   // no such query head in this pass
  }
  // the token's value row in d-space: v itself when it went to the list, else
  // U_v c_v as stored, on the tensor cores (warp w: rows [16w, 16w + 16), c_v
  // as bf16 high and low parts in columns 0 and 1, even and odd k-steps apart)
  if (keep) {
    if (tid < kD) s_vals[tid] = app[S::A_X + kD + tid];
  } else {
    float acc[2][4];
#pragma unroll
    for (int q = 0; q < 2; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.f;
    const bool lo = g & 1;
#pragma unroll
    for (int ks = 0; ks < MVT; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(a0, a1, a2, a3, uv + (16 * warp + (lm & 1) * 8 + lr) * S::VS + (ks * 16 + (lm >> 1) * 8) * 2);
      const float* c2 = app + S::A_CV + ks * 16 + 2 * t;
      const uint32_t b0 = g < 2 ? pack_bf16(bf16_part(c2[0], lo), bf16_part(c2[1], lo)) : 0u;
      const uint32_t b1 = g < 2 ? pack_bf16(bf16_part(c2[8], lo), bf16_part(c2[9], lo)) : 0u;
      mma_16816(acc[ks & 1], a0, a1, a2, a3, b0, b1);
    }
    if (t == 0) {
      s_vals[16 * warp + g] = (acc[0][0] + acc[1][0]) + (acc[0][1] + acc[1][1]);
      s_vals[16 * warp + g + 8] = (acc[0][2] + acc[1][2]) + (acc[0][3] + acc[1][3]);
    }
  }
}

template <int G, int RK, int RV, int W, int NS, bool APP, int CB>
__global__ void __launch_bounds__(W * 32, 1) decode_stream_kernel(DecodeParams p) {
  using S = Shape<G, RK, RV, W, NS, CB>;
  static_assert(!APP || W * 32 == 2 * kD, "the fused append maps one row element to a thread");
  constexpr int kWarps = S::kWarps, kThreads = S::kThreads;
  constexpr int KST = RK / 16;                   // k-steps of the compressed logits
  constexpr int MVT = RV / 16;                   // m-tiles of the compressed value sum
  // int4 value rows that are whole 16-byte pieces (r_v a multiple of 32) are
  // read with transposing ldmatrix (value columns in the order noted there)
  constexpr bool kInt4Ldsm = CB == 4 && RV % 32 == 0;
  constexpr int KP = S::KP, VP = S::VP;          // 16-byte pieces per stored row
  constexpr int UKP = S::UKP, UVP = S::UVP;      // 16-byte pieces per basis row
  constexpr int NST = S::STAGES;
  extern __shared__ __align__(128) unsigned char sm[];
  const lrkv_dims& D = p.D;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;         // MMA fragment coordinates
  // N columns of the token-side MMAs: column 2h = bf16 high part of query head
  // h, column 2h + 1 = its low part.  A lane's accumulator fragment (columns
  // 2t, 2t + 1) therefore holds both parts of head t: one head per lane.
  // query heads of this pass: q_head(x) is the x-th of the kv head's group;
  // heads x >= g_live of the template's G do not exist in this pass
  const int g_live = min(G, p.g_all - p.g_off);
  auto q_head = [&](int x) { return (size_t)b * D.Hq + (size_t)h * p.g_all + p.g_off + x; };
  const bool live_t = t < g_live;                // this lane's head exists
  const int lm = lane >> 3, lr = lane & 7;       // ldmatrix address roles
  const size_t bh = (size_t)b * D.Hkv + h;

  unsigned char* uk = sm + S::OFF_UK;
  uint32_t* maskw = reinterpret_cast<uint32_t*>(sm + S::OFF_MASK);
  auto slot_of = [&](int stage, int w) { return sm + (size_t)(stage * kWarps + w) * S::SLOT; };
  __shared__ int s_last;

  // ---- prologue, independent of the preceding kernel: the bases ------------------
  {  // U_k into padded rows, 16-byte pieces over every thread: the query-side
     // basis for q~ (U_kq when given), and the key-side basis for the fused
     // append when it differs
    auto load_uk = [&](const lrkv_bf16* src, unsigned char* dst) {
      const unsigned char* Uk = reinterpret_cast<const unsigned char*>(src + (size_t)h * kD * RK);
      for (int q = tid; q < kD * UKP; q += kThreads) {
        const int r = q / UKP, sg = q - r * UKP;
        cp_async16(dst + r * S::KS + sg * 16, Uk + q * 16);
      }
    };
    load_uk(p.C.U_kq ? p.C.U_kq : p.C.U_k, uk);
    if (APP && p.C.U_kq && blockIdx.x == gridDim.x - 1) load_uk(p.C.U_k, sm + S::OFF_UK2);   // the append CTA
    cp_async_commit();
  }
  auto load_uv = [&]() {   // U_v into padded rows, 16-byte pieces over every thread
    const unsigned char* Uv = reinterpret_cast<const unsigned char*>(p.C.U_v + (size_t)h * kD * RV);
    for (int q = tid; q < kD * UVP; q += kThreads) {
      const int r = q / UVP, sg = q - r * UVP;
      cp_async16(sm + S::OFF_UV + r * S::VS + sg * 16, Uv + q * 16);
    }
    cp_async_commit();
  };
  load_uv();
  // The next kernel of the stream may be launched now: its CTAs take SMs as
  // this grid's CTAs leave and load their bases, and its wait still covers all
  // of this grid (every CTA of it has started once all have passed here).
  griddep_launch_dependents();

  // ---- after the preceding kernel of the stream: the query (produced upstream)
  // and the cache state (an append may precede), all loaded in one batch ----------
  griddep_wait();
  // q as fragments over k = d: the B operand of the full-rank logits (column
  // n = 2h holds head h; q is bf16, hence exact, so the low-part columns are 0)
  // and the A operand (rows = heads) of q~ = U_k^T q
  uint32_t qf0[8], qf1[8];
  {
    const int hq = g >> 1;                                    // B column g: head g / 2
    const bool on = (g & 1) == 0 && hq < g_live;
    const lrkv_bf16* qrow = p.q + q_head(hq < g_live ? hq : 0) * kD;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qf0[ks] = on ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * t) : 0u;
      qf1[ks] = on ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 8 + 2 * t) : 0u;
    }
  }
  uint32_t qa0[8], qa1[8];   // q as the A operand: row m = head m < G
  {
    const lrkv_bf16* qrow = p.q + q_head(g < g_live ? g : 0) * kD;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qa0[ks] = g < g_live ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * t) : 0u;
      qa1[ks] = g < g_live ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 8 + 2 * t) : 0u;
    }
  }
  // fused append: does row b have a new token; one element of its new key
  // (threads < d) or value (threads >= d) row per thread, for the append CTA
  int n_b = 0;
  uint32_t st_new = 0;
  uint16_t xe = 0;
  if constexpr (APP) {
    n_b = new_tokens(p.t_new_b, b, 1, &st_new);
    xe = (tid < kD ? p.k_new : p.v_new)[bh * kD + (tid & (kD - 1))];   // [B][1][Hkv][d]
  }
  // the sequence length and the list length; the split's mask words follow
  // once the live length has fixed the split
  int T = p.C.seq_len[b];
  const int F_raw = p.C.full_cnt[bh];
  T = T < 0 ? 0 : (T > D.T_cap ? D.T_cap : T);
  // fused append: the new token (if the row has one and there is room) takes
  // position T_old
  int n_eff = 0;
  if constexpr (APP) {
    n_eff = n_b > 0 && T < D.T_cap ? 1 : 0;
    if (n_b > 0 && T >= D.T_cap) st_new |= LRKV_DEV_SEQ_OVERFLOW;
  }
  const int T_old = T;
  T += n_eff;
  // splits from the live length (every CTA of the (b, kv head) finds the same).
  // With a fused append the grid's last CTA does the append and nothing else
  // (its record joins the merge), so the stream never waits for it: the other
  // CTAs split the T_old cached positions among the remaining n_chunk_max - 1
  // (at least the ceil(T_cap / kMaxDecodeChunk) splits any cached length needs).
  int chunk;
  const int n_chunks = APP ? decode_split(T_old, p.n_chunk_max - 1, (long long)D.B * D.Hkv, p.num_sms, &chunk)
                           : decode_split(T, p.n_split, (long long)D.B * D.Hkv, p.num_sms, &chunk);
  const bool is_app = APP && c == (int)gridDim.x - 1;   // the append CTA
  const bool streams = !is_app && c < n_chunks;
  const bool active = streams || is_app;
  const int n_rec = n_chunks + (APP ? 1 : 0);            // records merged: the splits', then the append's
  const int c0 = c * chunk;
  // this split's mask words (words past the sequence end are never used): the
  // loads go out now and land while q~ is formed
  constexpr int kMW = (kMaxChunk / 32 + kThreads - 1) / kThreads;   // mask words per thread
  uint32_t mw[kMW];
#pragma unroll
  for (int u = 0; u < kMW; ++u) {
    const int wl = tid + u * kThreads, wi = c0 / 32 + wl;
    mw[u] = streams && wl < chunk / 32 && wi < D.T_cap / 32 ? p.C.route_mask[bh * (D.T_cap / 32) + wi] : 0u;
  }

  // ---- this warp's tiles; the first ones are issued before the mask words and
  // the query projection, so their copies overlap both ------------------------------
  const int c1 = min(T_old, c0 + chunk);   // the new position is not read from the cache
  const int n_pos = streams && c1 > c0 ? c1 - c0 : 0;
  // this split's share of the full-rank list
  const int F = min(max(F_raw, 0), D.F_cap);
  const int share = (F + n_chunks - 1) / n_chunks;
  const int f0 = min(F, c * share), f1 = min(F, f0 + share);
  const int n_full = streams ? f1 - f0 : 0;
  const unsigned char* ck = static_cast<const unsigned char*>(p.C.coef_k) + (bh * D.T_cap + c0) * S::TKB;
  const unsigned char* cv = static_cast<const unsigned char*>(p.C.coef_v) + (bh * D.T_cap + c0) * S::TVB;
  const float* sck = CB < 16 ? p.C.scale_k + bh * D.T_cap + c0 : nullptr;   // code scales
  const float* scv = CB < 16 ? p.C.scale_v + bh * D.T_cap + c0 : nullptr;
  const lrkv_bf16* fk = p.C.full_k + (bh * D.F_cap + f0) * kD;
  const lrkv_bf16* fv = p.C.full_v + (bh * D.F_cap + f0) * kD;

  // this warp's tiles: every kWarps-th compressed tile and every kWarps-th full-rank tile
  const int n_ct = (n_pos + kTileC - 1) / kTileC;
  const int n_ft = (n_full + kTileF - 1) / kTileF;
  const int nct_w = n_ct > warp ? (n_ct - warp + kWarps - 1) / kWarps : 0;
  const int nft_w = n_ft > warp ? (n_ft - warp + kWarps - 1) / kWarps : 0;
  const int n_tiles = nct_w + nft_w;
  // The warp's sequence interleaves its compressed and full-rank tiles evenly
  // (a Bresenham walk: step i is compressed when floor((i+1) nct_w / n_tiles)
  // grows), so the bytes in flight stay near their mean even when a high routed
  // fraction leaves compressed tiles nearly empty.  `Walk` yields, step by
  // step, whether the tile is compressed and its index among the warp's tiles
  // of that kind; the copy side and the compute side each keep one.
  struct Walk {
    int err, ic, jf;
    __device__ __forceinline__ bool next(int nc, int n, int& k) {
      err += nc;
      if (err >= n) {
        err -= n;
        k = ic++;
        return true;
      }
      k = jf++;
      return false;
    }
  };
  Walk wi_copy{0, 0, 0}, wi_comp{0, 0, 0};

  // positions of compressed tile k before the end, and those of them that are
  // read: unmasked (compressed) too
  auto valid_bits = [&](int k) -> uint32_t {
    const int nv = n_pos - k * kTileC;
    return nv >= 32 ? kFull : ((1u << nv) - 1u);
  };
  auto tile_bits = [&](int k) -> uint32_t { return ~maskw[k] & valid_bits(k); };
  // masked: skip routed positions (zero-filled, not read).  The prologue's tiles
  // go out before the mask words have arrived and copy every valid row: the
  // routed ones hold finite coefficients too and their logits are -inf.
  auto issue = [&](int i, bool masked) {
    unsigned char* slot = slot_of(i % NST, warp);
    int kw;
    if (wi_copy.next(nct_w, n_tiles, kw)) {
      const int k = warp + kWarps * kw;
      const uint32_t bits = masked ? tile_bits(k) : valid_bits(k);
      const unsigned char* src_k = ck + (size_t)k * kTileC * S::TKB;
      const unsigned char* src_v = cv + (size_t)k * kTileC * S::TVB;
      unsigned char* vslot = slot + kTileC * S::TKS;
      if constexpr (CB == 4) {
        // the tile's rows are one block of 32 * TKB (32 * TVB) bytes: 16-byte
        // pieces, no per-row zero-fill (routed and past-the-end rows hold
        // finite codes; their logits are -inf and their weights 0)
        for (int q = lane; q < kTileC * S::TKB / 16; q += 32) cp_async16(slot + q * 16, src_k + q * 16);
        for (int q = lane; q < kTileC * S::TVB / 16; q += 32) cp_async16(vslot + q * 16, src_v + q * 16);
        (void)bits;
      } else {
#pragma unroll
        for (int j = 0; j < KP; ++j) {   // piece q = lane + 32 j of the tile's key rows
          const int q = lane + 32 * j, r = q / KP, sg = q - r * KP;
          const bool on = (bits >> r) & 1u;
          cp_async16_zfill(slot + r * S::TKS + sg * 16, on ? src_k + q * 16 : src_k, on ? 16u : 0u);
        }
#pragma unroll
        for (int j = 0; j < VP; ++j) {
          const int q = lane + 32 * j, r = q / VP, sg = q - r * VP;
          const bool on = (bits >> r) & 1u;
          cp_async16_zfill(vslot + r * S::TVS + sg * 16, on ? src_v + q * 16 : src_v, on ? 16u : 0u);
        }
      }
      if constexpr (CB < 16) {   // the tile's 32 key and 32 value scales: 16 pieces
        if (lane < 16) {
          const float* src = (lane < 8 ? sck : scv) + (size_t)k * kTileC + (lane & 7) * 4;
          cp_async16(slot + S::T_SC + lane * 16, src);
        }
      }
    } else {
      const int k = warp + kWarps * kw;
      const int r0 = k * kTileF;
      const int n = min(kTileF, n_full - r0);
      const unsigned char* src_k = reinterpret_cast<const unsigned char*>(fk + (size_t)r0 * kD);
      const unsigned char* src_v = reinterpret_cast<const unsigned char*>(fv + (size_t)r0 * kD);
      const int sg = lane & 15;
#pragma unroll
      for (int j = 0; j < kTileF / 2; ++j) {
        const int r = (lane >> 4) + 2 * j;
        const bool on = r < n;
        const int off = r * kD * 2 + sg * 16;
        cp_async16_zfill(slot + r * S::FS + sg * 16, on ? src_k + off : src_k, on ? 16u : 0u);
        cp_async16_zfill(slot + (kTileF + r) * S::FS + sg * 16, on ? src_v + off : src_v,
                         on ? 16u : 0u);
      }
    }
  };
#pragma unroll
  for (int s = 0; s < NST - 1; ++s) {
    if (streams && s < n_tiles) issue(s, false);
    cp_async_commit();
  }

  const float scale = kLog2e * rsqrtf((float)kD);
  // q~ = U_k^T q as B fragments over k = r_k (column n = 2h + part: the bf16
  // high or low part of head h), on the tensor cores: warp w < r_k / 16 forms
  // columns [16w, 16w + 16) and leaves its fragments in shared memory for all
  static_assert(KST <= kWarps, "one block of q~ columns per warp");
  __shared__ uint32_t s_qb[KST][2][32];
  float* app = reinterpret_cast<float*>(sm + S::OFF_APP);   // fused append scratch
  cp_async_wait<NST>();   // U_k in (U_v and the prologue's tiles may still be in flight)
  __syncthreads();
  if (active && warp < KST) {
    const int ks2 = warp;                      // columns [16 ks2, 16 ks2 + 16) of q~
    float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(b0, b1, b2, b3, uk + (ks * 16 + (lm & 1) * 8 + lr) * S::KS + (16 * ks2 + (lm >> 1) * 8) * 2);
      mma_16816(a0, qa0[ks], 0u, qa1[ks], 0u, b0, b1);
      mma_16816(a1, qa0[ks], 0u, qa1[ks], 0u, b2, b3);
    }
    if constexpr (APP) {
      if (g < G) {    // q~ rows (scaled), for the new token's logit if it stays compressed
        float* qt = app + S::A_QT + g * RK + 16 * ks2;
        qt[2 * t] = a0[0] * scale;
        qt[2 * t + 1] = a0[1] * scale;
        qt[8 + 2 * t] = a1[0] * scale;
        qt[8 + 2 * t + 1] = a1[1] * scale;
      }
    }
    // lane (m, t) holds q~[head m][16 ks2 + 2t (+1)] in a0 and [+8] in a1 (rows m < 4).
    // B column g = 2h + part takes head h from lane 4h + t'.  The B fragment of
    // k = 2t, 2t+1 (b0) and 2t+8, 2t+9 (b1) is the q~ columns of those k in the
    // tiles' contraction order: the same columns for bf16 rows; for int8 codes a
    // thread's four bytes 4t..4t+3 are k = 2t, 2t+1, 2t+8, 2t+9, so b0 holds
    // columns 4t, 4t+1 and b1 columns 4t+2, 4t+3.
    const int hq4 = (g >> 1) << 2;
    const int sa = hq4 | (CB == 16 ? t : (t < 2 ? 2 * t : 2 * t - 4));
    const int sb = hq4 | (CB == 16 ? t : (t < 2 ? 2 * t + 1 : 2 * t - 3));
    const bool from_a1 = CB == 16 ? false : t >= 2;   // columns 8..15 of the block
    const float pa0 = __shfl_sync(kFull, a0[0], sa), pa1 = __shfl_sync(kFull, a0[1], sa);
    const float qa0_ = __shfl_sync(kFull, a1[0], sa), qa1_ = __shfl_sync(kFull, a1[1], sa);
    const float pb0 = __shfl_sync(kFull, a0[0], sb), pb1 = __shfl_sync(kFull, a0[1], sb);
    const float qb0_ = __shfl_sync(kFull, a1[0], sb), qb1_ = __shfl_sync(kFull, a1[1], sb);
    float x0, x1, y0, y1;   // b0's and b1's two columns
    if (CB == 16) {
      x0 = pa0, x1 = pa1, y0 = qb0_, y1 = qb1_;
    } else {
      x0 = from_a1 ? qa0_ : pa0, x1 = from_a1 ? qa1_ : pa1;
      y0 = from_a1 ? qb0_ : pb0, y1 = from_a1 ? qb1_ : pb1;
    }
    const bool lo_n = g & 1;
    const bool live = (g >> 1) < g_live;
    if constexpr (CB == 8) {
      // int8 codes meet q~ as f16 (high and low parts): a code widens to f16
      // in half the instructions it takes to reach bf16
      s_qb[ks2][0][lane] = live ? f16_part_bits(x0 * scale, lo_n) | (f16_part_bits(x1 * scale, lo_n) << 16) : 0u;
      s_qb[ks2][1][lane] = live ? f16_part_bits(y0 * scale, lo_n) | (f16_part_bits(y1 * scale, lo_n) << 16) : 0u;
    } else {
      s_qb[ks2][0][lane] = live ? pack_bf16(bf16_part(x0 * scale, lo_n), bf16_part(x1 * scale, lo_n)) : 0u;
      s_qb[ks2][1][lane] = live ? pack_bf16(bf16_part(y0 * scale, lo_n), bf16_part(y1 * scale, lo_n)) : 0u;
    }
  }
  // q . mu_k per query head (scaled), added to every compressed logit: 0 unless
  // the cache has an attention-aware key basis with a mean
  __shared__ float s_bias[G];
  if (warp >= kWarps - G) {
    const int gi = warp - (kWarps - G);
    float sb = 0.f;
    if (p.C.mu_k && gi < g_live) {
      const lrkv_bf16* qrow = p.q + q_head(gi) * kD;
      for (int i = lane; i < kD; i += 32) sb = fmaf(bf2f(qrow[i]), p.C.mu_k[(size_t)h * kD + i], sb);
    }
    sb = warp_sum(sb);
    if (lane == 0) s_bias[gi] = sb * scale;
  }
  const bool owner = is_app && n_eff > 0;   // the append CTA has a token to append
  // Every thread of this CTA has read seq_len[b] (the barrier above): each CTA
  // takes the row's ticket once (release only) and looks at it later; the last
  // CTA of the grid for row b advances its length.
  int seq_ticket = 0;
  auto advance_len = [&]() {
    if (seq_ticket == D.Hkv * (int)gridDim.x - 1) {
      fence_acq_rel_gpu();
      p.C.seq_len[b] = T;
      p.seq_tickets[b] = 0;
    }
  };
  const int tk = kThreads - 32;   // the thread that takes it: lane 0 of the last warp
  if constexpr (APP) {
    if (tid == 0 && h == 0 && c == 0 && st_new) atomicOr(p.C.dev_status, st_new);
  }
  if (!active) {
    cp_async_wait<0>();   // U_v (in flight since the prologue): none left behind on exit
    if (APP && tid == tk) {
      seq_ticket = atom_add_release_gpu(p.seq_tickets + b, 1);
      advance_len();
    }
    return;
  }
#pragma unroll
  for (int u = 0; u < kMW; ++u)
    if (tid + u * kThreads < kMaxChunk / 32) maskw[tid + u * kThreads] = mw[u];
  cp_async_wait<NST - 1>();   // U_v in (only the prologue's tiles may be in flight)
  // the append CTA's new token: its logit per head, whether it went to the
  // full-rank list, and its value row (v, or c_v as stored)
  __shared__ float s_new[G];
  __shared__ float s_vals[kD];
  __shared__ int s_keep;
  __syncthreads();   // mask words, U_v and q~ in; every warp is done with U_k (the last stage is free)
  uint32_t qb0[KST], qb1[KST];
#pragma unroll
  for (int ks2 = 0; ks2 < KST; ++ks2) qb0[ks2] = s_qb[ks2][0][lane], qb1[ks2] = s_qb[ks2][1][lane];
  const float bias = live_t ? s_bias[t] : 0.f;   // this lane's head
  // ---- the append CTA: the new token's compress and its record ------------------------
  // (its U_k copy and scratch sit in the last stage; it streams no tiles)
  if constexpr (APP) {
    if (is_app) {
      if (owner)
        append_token<S, G, RK, RV, CB>(p, app, p.C.U_kq ? sm + S::OFF_UK2 : uk, uk, sm + S::OFF_UV, s_bias,
                                       b, h, bh, T_old, F, scale, xe, s_new, s_vals, &s_keep);
      __syncthreads();   // the token's logits and value row in
      // record n_chunks: per query head m = the token's logit, l = 1 and o = its
      // value row in d-space (v, or U_v c_v as stored); an empty record
      // (m = -inf) when the row has no token
      float* recA = p.partials + (bh * p.n_chunk_max + n_chunks) * G * (size_t)S::REC;
      for (int o = tid; o < G * kD; o += kThreads) {
        const int gi = o / kD, i = o - gi * kD;
        recA[gi * S::REC + 4 + i] = owner ? s_vals[i] : 0.f;
      }
      if (tid < G) {
        recA[tid * S::REC] = owner ? s_new[tid] : -INFINITY;
        recA[tid * S::REC + 1] = owner ? 1.f : 0.f;
        if (tid == 0) recA[2] = owner && s_keep ? 1.f : 0.f;
      }
      if (tid == tk) seq_ticket = atom_add_release_gpu(p.seq_tickets + b, 1);
    }
  }

  if (!is_app) {
    // ---- stream the tiles ------------------------------------------------------------
    // lane state: running max and sum of head t; accumulators O^T (rows = value
    // columns, columns = head parts: all four fragment entries are head t) for
    // the compressed and full-rank sums
    float m_run = -INFINITY, l_run = 0.f;
    float oc[MVT][4], of[8][4];
  #pragma unroll
    for (int mt = 0; mt < MVT; ++mt) oc[mt][0] = oc[mt][1] = oc[mt][2] = oc[mt][3] = 0.f;
  #pragma unroll
    for (int mt = 0; mt < 8; ++mt) of[mt][0] = of[mt][1] = of[mt][2] = of[mt][3] = 0.f;

    // int8 codes: the value sums run on f16 operands, p * w (w the row's code
    // scale) times 2^e_v, so the largest row scale seen sits near 2^9..2^10:
    // far from f16 overflow, and the smallest weights that matter stay normal.
    // e_v is set by the first tile with a code row and only lowered when a
    // later tile would come within 2^15; the accumulators then scale by the
    // power of two (exact).  The lift divides them by 2^e_v.
    int e_v = 0;
    bool e_set = false;
    float v_scale = 1.f;

    // Online softmax over NB 16-row blocks: s[nb] = {row g, row g + 8} of head t
    // (-inf = no token).  Rescales this lane's accumulators when the max grows,
    // and returns the probabilities packed as the P^T B fragments of each block
    // (column 2t = high part, 2t + 1 = low part; bf16, or f16 with F16); with
    // value weights wv (the rows' code scales) the packed entries are p * wv,
    // the sum l takes p.
    auto softmax_pack_w = [&](auto& s, auto& pb0, auto& pb1, auto nb_tag, const float (*wv)[2],
                              auto f16_tag) {
      constexpr int NB = decltype(nb_tag)::value;
      constexpr bool F16 = decltype(f16_tag)::value;
      float x = -INFINITY;
  #pragma unroll
      for (int nb = 0; nb < NB; ++nb) x = fmaxf(x, fmaxf(s[nb][0], s[nb][1]));
      // the running max only grows: the reduction over the rows is needed only
      // when some lane holds a score above it (rare after the first tiles)
      if (__any_sync(kFull, x > m_run)) {
  #pragma unroll
        for (int o = 4; o < 32; o <<= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, o));
        if (x > m_run) {
          const float sc = m_run == -INFINITY ? 0.f : exp2f(m_run - x);
          l_run *= sc;
  #pragma unroll
          for (int mt = 0; mt < MVT; ++mt) oc[mt][0] *= sc, oc[mt][1] *= sc, oc[mt][2] *= sc, oc[mt][3] *= sc;
  #pragma unroll
          for (int mt = 0; mt < 8; ++mt) of[mt][0] *= sc, of[mt][1] *= sc, of[mt][2] *= sc, of[mt][3] *= sc;
          m_run = x;
        }
      }
      __syncwarp();
  #pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        float p0 = s[nb][0] == -INFINITY ? 0.f : exp2f(s[nb][0] - m_run);
        float p1 = s[nb][1] == -INFINITY ? 0.f : exp2f(s[nb][1] - m_run);
        l_run += p0 + p1;
        if (wv) p0 *= wv[nb][0], p1 *= wv[nb][1];
        if constexpr (F16) {   // (high part, low part): f16(p) and f16(p - f16(p))
          const float h0 = __half2float(__float2half_rn(p0));
          const float h1 = __half2float(__float2half_rn(p1));
          pb0[nb] = movmatrix_t(cvt_f16x2(p0, p0 - h0));
          pb1[nb] = movmatrix_t(cvt_f16x2(p1, p1 - h1));
          continue;
        }
        // (high part, low part) of p: bf16(p) and bf16(p - bf16(p))
        const float h0 = __uint_as_float(cvt_bf16x2(p0, p0) << 16);
        const float h1 = __uint_as_float(cvt_bf16x2(p1, p1) << 16);
        pb0[nb] = movmatrix_t(cvt_bf16x2(p0, p0 - h0));
        pb1[nb] = movmatrix_t(cvt_bf16x2(p1, p1 - h1));
      }
    };
    auto softmax_pack = [&](auto& s, auto& pb0, auto& pb1, auto nb_tag) {
      softmax_pack_w(s, pb0, pb1, nb_tag, static_cast<const float (*)[2]>(nullptr), std::false_type{});
    };

    for (int i = 0; i < n_tiles; ++i) {
      if (i + NST - 1 < n_tiles) issue(i + NST - 1, true);
      cp_async_commit();
      cp_async_wait<NST - 1>();
      __syncwarp();
      const unsigned char* slot = slot_of(i % NST, warp);
      int kw;
      if (wi_comp.next(nct_w, n_tiles, kw)) {
        // compressed tile: S^T[token][head part] = C_k q~^T, then O^T += C_v^T P^T
        const uint32_t bits = tile_bits(warp + kWarps * kw);
        float st[2][4];
        if constexpr (CB == 16) {
          // even and odd k-steps into separate accumulators: shorter chains of
          // dependent MMAs
          float so[2][4];
  #pragma unroll
          for (int nb = 0; nb < 2; ++nb) {
            st[nb][0] = st[nb][1] = st[nb][2] = st[nb][3] = 0.f;
            so[nb][0] = so[nb][1] = so[nb][2] = so[nb][3] = 0.f;
  #pragma unroll
            for (int ks = 0; ks < KST; ++ks) {
              uint32_t a0, a1, a2, a3;
              ldsm_x4(a0, a1, a2, a3,
                      slot + (16 * nb + (lm & 1) * 8 + lr) * S::TKS + (ks * 16 + (lm >> 1) * 8) * 2);
              mma_16816(ks & 1 ? so[nb] : st[nb], a0, a1, a2, a3, qb0[ks], qb1[ks]);
            }
  #pragma unroll
            for (int e = 0; e < 4; ++e) st[nb][e] += so[nb][e];
          }
          float s[2][2];
  #pragma unroll
          for (int nb = 0; nb < 2; ++nb)
  #pragma unroll
            for (int x = 0; x < 2; ++x) {   // rows g, g + 8: high + low part of head t
              const float v = st[nb][2 * x] + st[nb][2 * x + 1] + bias;
              s[nb][x] = live_t && ((bits >> (16 * nb + g + x * 8)) & 1u) ? v : -INFINITY;
            }
          uint32_t pb0[2], pb1[2];
          softmax_pack(s, pb0, pb1, std::integral_constant<int, 2>{});
          const unsigned char* vrows = slot + kTileC * S::TKS;
  #pragma unroll
          for (int mt = 0; mt < MVT; ++mt)
  #pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
              uint32_t a0, a1, a2, a3;
              ldsm_x4_t(a0, a1, a2, a3,
                        vrows + (16 * nb + (lm >> 1) * 8 + lr) * S::TVS + (mt * 16 + (lm & 1) * 8) * 2);
              mma_16816(oc[mt], a0, a1, a2, a3, pb0[nb], pb1[nb]);
            }
        } else if constexpr (CB == 4) {
          // int4 codes, converted to bf16 in registers (exact): a nibble n with
          // its sign bit flipped is u = n + 8, the bf16 0x4300 | u is 128 + u, and
          // subtracting 136 gives n.  Logits: a 16-bit load of a row gives a
          // thread the k-step's codes 4t..4t+3 (k = 2t, 2t+1 | 2t+8, 2t+9, the
          // order of q~'s B fragments, as for int8).  Values: a byte of a row holds
          // columns 2g, 2g+1 of a 16-column block (accumulator rows g, g + 8).
          const float* scl = reinterpret_cast<const float*>(slot + S::T_SC);   // [2][32]
          const uint32_t k136 = 0xC308C308u, k1 = 0x3F803F80u;                 // bf16x2 (-136, -136), (1, 1)
          // nibble i (bits 4i..4i+3) of both 16-bit halves of u (sign bits
          // already flipped) -> bf16x2 of the two codes
          auto nib_col = [&](uint32_t u, int i) {
            uint32_t x = ((u >> (4 * i)) & 0x000F000Fu) | 0x43004300u;
            asm("fma.rn.bf16x2 %0, %0, %1, %2;" : "+r"(x) : "r"(k1), "r"(k136));
            return x;
          };
          auto nib_pairs = [&](uint32_t x16, uint32_t& lo01, uint32_t& lo23) {
            // x16: four nibbles (codes c0..c3 from the low end) -> bf16x2 (c0, c1), (c2, c3)
            const uint32_t u = x16 ^ 0x8888u;
            lo01 = 0x43004300u | (u & 0xFu) | ((u & 0xF0u) << 12);
            lo23 = 0x43004300u | ((u >> 8) & 0xFu) | ((u & 0xF000u) << 4);
            asm("fma.rn.bf16x2 %0, %0, %1, %2;" : "+r"(lo01) : "r"(k1), "r"(k136));
            asm("fma.rn.bf16x2 %0, %0, %1, %2;" : "+r"(lo23) : "r"(k1), "r"(k136));
          };
  #pragma unroll
          for (int nb = 0; nb < 2; ++nb) {
            st[nb][0] = st[nb][1] = st[nb][2] = st[nb][3] = 0.f;
            const unsigned char* r_lo = slot + (16 * nb + g) * S::TKS + 2 * t;
            const unsigned char* r_hi = r_lo + 8 * S::TKS;
  #pragma unroll
            for (int ks = 0; ks < KST; ++ks) {
              uint32_t a0, a1, a2, a3;
              nib_pairs(*reinterpret_cast<const uint16_t*>(r_lo + 8 * ks), a0, a2);
              nib_pairs(*reinterpret_cast<const uint16_t*>(r_hi + 8 * ks), a1, a3);
              mma_16816(st[nb], a0, a1, a2, a3, qb0[ks], qb1[ks]);
            }
          }
          float s[2][2], wv[2][2];
  #pragma unroll
          for (int nb = 0; nb < 2; ++nb)
  #pragma unroll
            for (int x = 0; x < 2; ++x) {
              const int row = 16 * nb + g + x * 8;
              const bool on = live_t && ((bits >> row) & 1u);
              const float v = st[nb][2 * x] + st[nb][2 * x + 1];
              s[nb][x] = on ? fmaf(v, scl[row], bias) : -INFINITY;
              wv[nb][x] = on ? scl[kTileC + row] : 0.f;
            }
          uint32_t pb0[2], pb1[2];
          softmax_pack_w(s, pb0, pb1, std::integral_constant<int, 2>{}, wv, std::false_type{});
          const unsigned char* vrows = slot + kTileC * S::TKS;
          if constexpr (kInt4Ldsm) {
            // value rows of 16-byte multiples: one transposing ldmatrix per 32
            // value columns (16 bytes of 8 token rows per matrix; matrices =
            // tokens 0-7, 8-15, 16-23, 24-31) gives thread (g, t) the 16-bit
            // element g (columns 4g..4g+3, one nibble each) of tokens 2t, 2t+1.
            // Accumulator block 2 qc + sb: row g is value column 32 qc + 4g + 2 sb,
            // row g + 8 the next one; nibble 2 sb (2 sb + 1) of both tokens makes a
            // bf16 pair through 0x4300 | u and one packed fma.
  #pragma unroll
            for (int qc = 0; qc < RV / 32; ++qc) {
              uint32_t r[4];
              ldsm_x4_t(r[0], r[1], r[2], r[3], vrows + (8 * lm + lr) * S::TVS + qc * 16);
  #pragma unroll
              for (int nb = 0; nb < 2; ++nb) {
                const uint32_t lo = r[2 * nb] ^ 0x88888888u, hi = r[2 * nb + 1] ^ 0x88888888u;
  #pragma unroll
                for (int sb = 0; sb < 2; ++sb)
                  mma_16816(oc[2 * qc + sb], nib_col(lo, 2 * sb), nib_col(lo, 2 * sb + 1), nib_col(hi, 2 * sb),
                            nib_col(hi, 2 * sb + 1), pb0[nb], pb1[nb]);
              }
            }
          } else {
  #pragma unroll
          for (int mt = 0; mt < MVT; ++mt)
  #pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
              // tokens 16 nb + 2t, 2t+1 (a0, a1) and 2t+8, 2t+9 (a2, a3), byte g of the block
              const unsigned char* c0p = vrows + (16 * nb + 2 * t) * S::TVS + 8 * mt + g;
              const uint32_t x01 = (uint32_t)c0p[0] | ((uint32_t)c0p[S::TVS] << 8);
              const uint32_t x89 = (uint32_t)c0p[8 * S::TVS] | ((uint32_t)c0p[9 * S::TVS] << 8);
              // nibbles of x01: (token 2t: col 2g, 2g+1), (token 2t+1: col 2g, 2g+1)
              uint32_t a0, a1, a2, a3, e, o;
              nib_pairs(x01, e, o);   // e = (2t:2g, 2t:2g+1), o = (2t+1:2g, 2t+1:2g+1)
              a0 = __byte_perm(e, o, 0x5410);   // (2t:2g, 2t+1:2g)
              a1 = __byte_perm(e, o, 0x7632);   // (2t:2g+1, 2t+1:2g+1)
              nib_pairs(x89, e, o);
              a2 = __byte_perm(e, o, 0x5410);
              a3 = __byte_perm(e, o, 0x7632);
              mma_16816(oc[mt], a0, a1, a2, a3, pb0[nb], pb1[nb]);
            }
          }
        } else {
          // int8 codes, converted in registers (exact): to f16 for the logits
          // (against q~'s f16 high and low parts), to bf16 for the value sums.
          // Logits: an ldmatrix of a k-step's 16 code bytes gives a thread bytes
          // 4t..4t+3 of its row, k = 2t, 2t+1 (a0/a1) and 2t+8, 2t+9 (a2/a3) in
          // the order q~'s B fragments were built in; the row's key scale
          // multiplies the logit.
          const float* scl = reinterpret_cast<const float*>(slot + S::T_SC);   // [2][32]
          float so8[2][4];
  #pragma unroll
          for (int nb = 0; nb < 2; ++nb) {
            st[nb][0] = st[nb][1] = st[nb][2] = st[nb][3] = 0.f;
            so8[nb][0] = so8[nb][1] = so8[nb][2] = so8[nb][3] = 0.f;
            const unsigned char* rows = slot + (16 * nb + (lm & 1) * 8 + lr) * S::TKS;
  #pragma unroll
            for (int kp = 0; kp < KST; kp += 2) {
              uint32_t r0, r1, r2 = 0u, r3 = 0u, e0, e1, f0, f1;
              if (kp + 1 < KST) ldsm_x4(r0, r1, r2, r3, rows + kp * 16 + (lm >> 1) * 16);
              else ldsm_x2(r0, r1, rows + kp * 16);
              s8x4_f16pairs(r0, e0, f0);
              s8x4_f16pairs(r1, e1, f1);
              mma_16816_f16(st[nb], e0, e1, f0, f1, qb0[kp], qb1[kp]);
              if (kp + 1 < KST) {   // odd k-steps in their own accumulator
                s8x4_f16pairs(r2, e0, f0);
                s8x4_f16pairs(r3, e1, f1);
                mma_16816_f16(so8[nb], e0, e1, f0, f1, qb0[kp + 1], qb1[kp + 1]);
              }
            }
  #pragma unroll
            for (int e = 0; e < 4; ++e) st[nb][e] += so8[nb][e];
          }
          float s[2][2], wv[2][2];
          float wmax = 0.f;   // the largest code scale of the tile's read rows
  #pragma unroll
          for (int nb = 0; nb < 2; ++nb)
  #pragma unroll
            for (int x = 0; x < 2; ++x) {   // rows g, g + 8: high + low part of head t
              const int row = 16 * nb + g + x * 8;
              const bool read = (bits >> row) & 1u;
              const bool on = live_t && read;
              const float v = st[nb][2 * x] + st[nb][2 * x + 1];
              s[nb][x] = on ? fmaf(v, scl[row], bias) : -INFINITY;
              const float w = read ? scl[kTileC + row] : 0.f;   // scales of unread rows are never used
              wmax = fmaxf(wmax, w);
              wv[nb][x] = on ? w : 0.f;
            }
  #pragma unroll
          for (int o = 4; o < 32; o <<= 1) wmax = fmaxf(wmax, __shfl_xor_sync(kFull, wmax, o));
          if (wmax > 0.f) {   // warp-uniform
            const int ew = (int)((__float_as_uint(wmax) >> 23) & 0xff) - 127;   // wmax in [2^ew, 2^(ew+1))
            if (!e_set || ew + e_v >= 15) {
              const int e_new = min(max(9 - ew, -126), 126);
              if (e_set) {   // lower the scale of what is summed so far (e_new < e_v)
                const int d = e_new - e_v;
                const float f = d < -126 ? 0.f : __uint_as_float((uint32_t)(d + 127) << 23);
  #pragma unroll
                for (int mt = 0; mt < MVT; ++mt) oc[mt][0] *= f, oc[mt][1] *= f, oc[mt][2] *= f, oc[mt][3] *= f;
              }
              e_v = e_new;
              e_set = true;
              v_scale = __uint_as_float((uint32_t)(e_v + 127) << 23);
            }
          }
  #pragma unroll
          for (int nb = 0; nb < 2; ++nb) wv[nb][0] *= v_scale, wv[nb][1] *= v_scale;
          uint32_t pb0[2], pb1[2];
          softmax_pack_w(s, pb0, pb1, std::integral_constant<int, 2>{}, wv, std::true_type{});
          // values: one transposing ldmatrix per 16 value columns covers the 32
          // tokens; a thread's bytes are (token 2t | 2t+1) x (column 2g | 2g+1), so
          // accumulator row g is column 2g of the block and row g + 8 column 2g + 1
          const unsigned char* vrows = slot + kTileC * S::TKS;
  #pragma unroll
          for (int mt = 0; mt < MVT; ++mt) {
            uint32_t r0, r1, r2, r3, a0, a1, a2, a3;
            ldsm_x4_t(r0, r1, r2, r3, vrows + (8 * lm + lr) * S::TVS + mt * 16);
            s8x4_f16evenodd(r0, a0, a1);
            s8x4_f16evenodd(r1, a2, a3);
            mma_16816_f16(oc[mt], a0, a1, a2, a3, pb0[0], pb1[0]);
            s8x4_f16evenodd(r2, a0, a1);
            s8x4_f16evenodd(r3, a2, a3);
            mma_16816_f16(oc[mt], a0, a1, a2, a3, pb0[1], pb1[1]);
          }
        }
      } else {
        // full-rank tile: 16 list rows
        const int k = warp + kWarps * kw;
        const int nrows = min(kTileF, n_full - k * kTileF);
        // the 8 k-steps into 4 accumulators: chains of 2 dependent MMAs, not 8
        // (a dependent mma.sync waits for the previous one's result)
        float sq[4][4];
  #pragma unroll
        for (int u = 0; u < 4; ++u) sq[u][0] = sq[u][1] = sq[u][2] = sq[u][3] = 0.f;
  #pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(a0, a1, a2, a3, slot + ((lm & 1) * 8 + lr) * S::FS + (ks * 16 + (lm >> 1) * 8) * 2);
          mma_16816(sq[ks & 3], a0, a1, a2, a3, qf0[ks], qf1[ks]);
        }
        float st[4];
  #pragma unroll
        for (int e = 0; e < 4; ++e) st[e] = (sq[0][e] + sq[1][e]) + (sq[2][e] + sq[3][e]);
        float s[1][2];
  #pragma unroll
        for (int x = 0; x < 2; ++x) {   // rows g, g + 8 (the low-part column is 0 for q)
          const float v = (st[2 * x] + st[2 * x + 1]) * scale;
          s[0][x] = live_t && g + x * 8 < nrows ? v : -INFINITY;
        }
        uint32_t pb0[1], pb1[1];
        softmax_pack(s, pb0, pb1, std::integral_constant<int, 1>{});
        const unsigned char* vrows = slot + kTileF * S::FS;
  #pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(a0, a1, a2, a3, vrows + ((lm >> 1) * 8 + lr) * S::FS + (mt * 16 + (lm & 1) * 8) * 2);
          mma_16816(of[mt], a0, a1, a2, a3, pb0[0], pb1[0]);
        }
      }
      __syncwarp();
    }
    cp_async_wait<0>();
    // the row's length ticket: release-only, taken now that this thread has no
    // copy in flight (a release waits for them); looked at after the record
    if (APP && tid == tk) seq_ticket = atom_add_release_gpu(p.seq_tickets + b, 1);
    __syncwarp();

    // ---- lift: of += U_v acc_c^T on the tensor cores --------------------------------
    // acc_c^T (rows = r_v, columns = head parts) becomes the B operand: lane
    // (g, t) holds acc_c[head t][16 mt + g (+8)] (high + low part columns), packs
    // it as bf16 high and low parts (columns 2t, 2t + 1 of an 8x8 tile) and one
    // transpose gives the fragment (k = 2t, 2t + 1; n = g).  The product lands in
    // the full-rank accumulators, whose layout is the same: o = both parts summed.
    {
      const unsigned char* uv = sm + S::OFF_UV;
      uint32_t lb0[MVT], lb1[MVT];
  #pragma unroll
      for (int mt = 0; mt < MVT; ++mt) {
        float x0 = oc[mt][0] + oc[mt][1], x1 = oc[mt][2] + oc[mt][3];
        if constexpr (CB == 8) {   // back from the 2^e_v scale of the value sums (exact)
          const float inv = __uint_as_float((uint32_t)(127 - e_v) << 23);
          x0 *= inv, x1 *= inv;
        }
        const float h0 = __uint_as_float(cvt_bf16x2(x0, x0) << 16);
        const float h1 = __uint_as_float(cvt_bf16x2(x1, x1) << 16);
        lb0[mt] = movmatrix_t(cvt_bf16x2(x0, x0 - h0));
        lb1[mt] = movmatrix_t(cvt_bf16x2(x1, x1 - h1));
      }
  #pragma unroll
      for (int mi = 0; mi < 8; ++mi)
  #pragma unroll
        for (int mt = 0; mt < MVT; ++mt) {
          uint32_t a0, a1, a2, a3;
          if constexpr (CB == 16) {
            ldsm_x4(a0, a1, a2, a3, uv + (16 * mi + (lm & 1) * 8 + lr) * S::VS + (mt * 16 + (lm >> 1) * 8) * 2);
          } else if constexpr (kInt4Ldsm) {
            // block mt = 2 qc + sb: accumulator row k < 8 is value column 32 qc +
            // 4k + 2 sb, row k >= 8 the one after 32 qc + 4(k - 8) + 2 sb; a
            // thread's k = 2t, 2t+1 are columns 8t + 2 sb, 8t + 4 + 2 sb of the
            // 32 and k = 2t+8, 2t+9 the next ones: columns 8t..8t+7 in one load
            const int qc = mt >> 1, sb = mt & 1;
            const uint4 w0 = *reinterpret_cast<const uint4*>(uv + (16 * mi + g) * S::VS + (32 * qc + 8 * t) * 2);
            const uint4 w1 = *reinterpret_cast<const uint4*>(uv + (16 * mi + g + 8) * S::VS + (32 * qc + 8 * t) * 2);
            const uint32_t p0 = sb ? w0.y : w0.x, q0 = sb ? w0.w : w0.z;
            const uint32_t p1 = sb ? w1.y : w1.x, q1 = sb ? w1.w : w1.z;
            a0 = __byte_perm(p0, q0, 0x5410);
            a2 = __byte_perm(p0, q0, 0x7632);
            a1 = __byte_perm(p1, q1, 0x5410);
            a3 = __byte_perm(p1, q1, 0x7632);
          } else {
            // accumulator row k of the block is value column 2k (k < 8) or
            // 2(k - 8) + 1: A[i][k] = U_v[i][that column], so a thread's k = 2t,
            // 2t+1 are columns 4t, 4t+2 and k = 2t+8, 2t+9 columns 4t+1, 4t+3
            const uint2 w0 = *reinterpret_cast<const uint2*>(uv + (16 * mi + g) * S::VS + (mt * 16 + 4 * t) * 2);
            const uint2 w1 = *reinterpret_cast<const uint2*>(uv + (16 * mi + g + 8) * S::VS + (mt * 16 + 4 * t) * 2);
            a0 = __byte_perm(w0.x, w0.y, 0x5410);
            a2 = __byte_perm(w0.x, w0.y, 0x7632);
            a1 = __byte_perm(w1.x, w1.y, 0x5410);
            a3 = __byte_perm(w1.x, w1.y, 0x7632);
          }
          mma_16816(of[mi], a0, a1, a2, a3, lb0[mt], lb1[mt]);
        }
    }

    // ---- this warp's partial state into its stage-0 slot -------------------------------
  #pragma unroll
    for (int o = 4; o < 32; o <<= 1) l_run += __shfl_xor_sync(kFull, l_run, o);
    {
      float* Wp = reinterpret_cast<float*>(slot_of(0, warp));
      if (live_t) {
        // lane (g, t): head t, output rows mi*16 + g and mi*16 + g + 8, high + low part
        float* pf = Wp + S::W_PF + t * kD;
  #pragma unroll
        for (int mi = 0; mi < 8; ++mi) {
          pf[mi * 16 + g] = of[mi][0] + of[mi][1];
          pf[mi * 16 + g + 8] = of[mi][2] + of[mi][3];
        }
        if (g == 0) {
          Wp[S::W_M + t] = m_run;
          Wp[S::W_L + t] = l_run;
        }
      }
    }
    __syncthreads();

    // ---- merge the warps into this split's record ---------------------------------
    auto wpart = [&](int w) { return reinterpret_cast<const float*>(slot_of(0, w)); };
    __shared__ float s_we[kWarps][G];
    float* rec0 = p.partials + (bh * p.n_chunk_max + c) * G * (size_t)S::REC;
    if (tid < G) {
      float M = -INFINITY;
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wpart(w)[S::W_M + tid]);
      float Ls = 0.f;
      for (int w = 0; w < kWarps; ++w) {
        const float mw = wpart(w)[S::W_M + tid];
        const float e = mw == -INFINITY ? 0.f : exp2f(mw - M);
        s_we[w][tid] = e;
        Ls = fmaf(wpart(w)[S::W_L + tid], e, Ls);
      }
      rec0[tid * S::REC] = M;
      rec0[tid * S::REC + 1] = Ls;
      if (APP && tid == 0) rec0[2] = 0.f;
    }
    __syncthreads();
    for (int o = tid; o < G * kD; o += kThreads) {
      const int gi = o / kD, i = o - gi * kD;
      float x = 0.f;
  #pragma unroll
      for (int w = 0; w < kWarps; ++w) x = fmaf(wpart(w)[S::W_PF + o], s_we[w][gi], x);
      rec0[gi * S::REC + 4 + i] = x;
    }
  }

  if (APP && tid == tk) advance_len();

  // ---- the last split of this (batch row, kv head) merges every record ------------
  __syncthreads();
  if (tid == 0) s_last = atom_add_acq_rel_gpu(p.tickets + bh, 1) == n_rec - 1;
  __syncthreads();
  if (!s_last) return;
  // Warp w < 8 serves query head w / (8 / G) and a block of its columns; each
  // lane finds the head's global max and sum itself (lanes over records), then
  // accumulates its columns over the records with the weights passed by
  // shuffle.  Records come from L2 (ld.global.cg): other CTAs wrote them.
  if (warp < 8) {
    constexpr int WPH = 8 / G;                   // warps per head (the first 8 warps)
    constexpr int CPW = kD / WPH;                // columns per warp: 16, 32, 64
    constexpr int CPL = CPW >= 32 ? CPW / 32 : 1;
    const int gi = warp / WPH;
    const int col = (warp - gi * WPH) * CPW + lane * CPL;
    const bool on = lane * CPL < CPW;
    const float* recs = p.partials + bh * p.n_chunk_max * G * (size_t)S::REC + gi * S::REC;
    constexpr size_t kStride = (size_t)G * S::REC;   // floats between two records of a head
    float acc[CPL];
#pragma unroll
    for (int u = 0; u < CPL; ++u) acc[u] = 0.f;
    float Lsum = 0.f;
    // one batch of up to 32 records: every load is issued before the first use
    auto batch = [&](int k0, float M) {
      const int k = k0 + lane;
      const int nk = min(32, n_rec - k0);
      float vals[32][CPL];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float* v = recs + (size_t)(k0 + j) * kStride + 4 + col;
        if constexpr (CPL == 2) {
          const float2 x = j < nk && on ? __ldcg(reinterpret_cast<const float2*>(v)) : make_float2(0.f, 0.f);
          vals[j][0] = x.x;
          vals[j][CPL - 1] = x.y;
        } else {
          vals[j][0] = j < nk && on ? __ldcg(v) : 0.f;
        }
      }
      const float m = k < n_rec ? __ldcg(recs + (size_t)k * kStride) : -INFINITY;
      const float l = k < n_rec ? __ldcg(recs + (size_t)k * kStride + 1) : 0.f;
      if (M == -INFINITY) M = warp_max(m);      // a single batch: its own max is the max
      const float w = m == -INFINITY ? 0.f : exp2f(m - M);
      Lsum = fmaf(w, l, Lsum);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float wj = __shfl_sync(kFull, w, j);
#pragma unroll
        for (int u = 0; u < CPL; ++u) acc[u] = fmaf(wj, vals[j][u], acc[u]);
      }
    };
    if (n_rec <= 32) {
      batch(0, -INFINITY);
    } else {
      float M = -INFINITY;
      for (int k = lane; k < n_rec; k += 32) M = fmaxf(M, __ldcg(recs + (size_t)k * kStride));
      M = warp_max(M);
      for (int k0 = 0; k0 < n_rec; k0 += 32) batch(k0, M);
    }
    Lsum = warp_sum(Lsum);
    if (on && gi < g_live) {
      float* out = p.out + q_head(gi) * kD + col;
#pragma unroll
      for (int u = 0; u < CPL; ++u) out[u] = Lsum > 0.f ? acc[u] / Lsum : 0.f;
    }
  }
  if (tid == 0) {
    p.tickets[bh] = 0;
    // fused append: every CTA of this (b, kv head) has read the list length;
    // the new full-rank row (if the append CTA added one) now counts
    if (APP && __ldcg(p.partials + (bh * p.n_chunk_max + n_chunks) * G * (size_t)S::REC + 2) != 0.f)
      p.C.full_cnt[bh] = F + 1;
  }
}

}  // namespace ds
}  // namespace lrkv
