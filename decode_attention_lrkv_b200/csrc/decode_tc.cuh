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
// [r x tokens] x [tokens x g] with g <= 4 query heads, over rows gathered from
// a sparse position set.  On CUDA cores that is ~60 instructions per token and
// the kernel is issue-bound far below the HBM roof; as m16n8k16 MMAs it is a
// handful.  Tokens are the M dimension (16 per tile) and the query heads the
// N dimension: q~ and the probabilities p are fp32, so each is split into a
// bf16 high part (columns 0..3) and low part (columns 4..7) and the two
// columns of a head are summed afterwards -- the products keep ~16 bits more
// than bf16, fp32-level accuracy.  tcgen05 needs M >= 64 and canonical
// shared-memory layouts that rows gathered one by one do not have; the tensor
// work here is tiny either way.
//
// Work split.  Grid (splits, Hkv, B), one CTA of 16 warps per SM.  A CTA takes
// positions [c*chunk, (c+1)*chunk) of one (batch row, kv head) and an equal
// share of its full-rank list.  Each warp streams its own tiles through a
// 2-stage cp.async ring: a compressed tile is the unmasked rows of 16
// positions (routed positions are never read), a full-rank tile is 8 rows.
// Rows land in padded shared-memory rows so ldmatrix is conflict-free.  At
// the end the CTA merges its warps, lifts by U_v (MMA), writes one record
// (m, l, o[d]) per query head, and the last CTA of the (batch row, kv head)
// merges all records (atomic ticket, no waiting).
#pragma once

#include "decode_simple.cuh"
#include "lrkv_common.cuh"
#include "ptx.cuh"

namespace lrkv {
namespace tc {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 2;
constexpr int kTileC = 16;                       // positions per compressed tile
constexpr int kTileF = 8;                        // rows per full-rank tile
constexpr int kMaxChunk = kMaxDecodeChunk;                // positions per split (mask words in smem)
constexpr int kRecFloats = 4 + kD;               // m, l, (pad), o[d]: 16-byte multiple
constexpr uint32_t kWaitIters = 1u << 24;        // bounded mbarrier polls (seconds)
constexpr unsigned kFull = 0xffffffffu;

constexpr int al16(int x) { return (x + 15) & ~15; }
constexpr int al128(int x) { return (x + 127) & ~127; }

template <int G, int RK, int RV>
struct Shape {
  static_assert(G == 1 || G == 2 || G == 4, "1, 2 or 4 query heads per kv head");
  static_assert(RK % 16 == 0 && RV % 16 == 0 && RK <= kD && RV <= kD, "ranks");
  static constexpr int KS = 2 * RK + 16;         // padded row strides (bytes): odd multiples of 16
  static constexpr int VS = 2 * RV + 16;
  static constexpr int FS = 2 * kD + 16;
  static constexpr int SLOT_C = kTileC * (KS + VS);
  static constexpr int SLOT_F = kTileF * 2 * FS;
  static constexpr int SLOT = al128(SLOT_C > SLOT_F ? SLOT_C : SLOT_F);
  static constexpr int OFF_UK = kWarps * kStages * SLOT;      // U_k rows [d][KS]
  static constexpr int OFF_UV = al128(OFF_UK + kD * KS);      // U_v rows [d][VS]
  static constexpr int OFF_MASK = al128(OFF_UV + kD * VS);
  static constexpr int OFF_ROWS = al16(OFF_MASK + (kMaxChunk / 32) * 4);  // [warps][16] row -> offset
  static constexpr int OFF_BAR = al16(OFF_ROWS + kWarps * 16);           // merge, bases mbarriers
  static constexpr int SMEM = OFF_BAR + 16;
  static_assert(SMEM <= 227 * 1024, "shared memory of one CTA");
  // end-of-kernel reuse of the slot area (floats)
  static constexpr int R_PC = 0;                                  // [warps][G][RV]
  static constexpr int R_PF = R_PC + kWarps * G * RV;             // [warps][G][d]
  static constexpr int R_WM = R_PF + kWarps * G * kD;             // [warps][G]
  static constexpr int R_WL = R_WM + kWarps * G;                  // [warps][G]
  static constexpr int R_WE = R_WL + kWarps * G;                  // [warps][G] weights
  static constexpr int R_CC = R_WE + kWarps * G;                  // [G][RV] merged acc_c
  static constexpr int R_CF = R_CC + G * RV;                      // [G][d] merged acc_f
  static constexpr int R_M = R_CF + G * kD;                       // [G] max, [G] sum
  static constexpr int R_END = (R_M + 2 * G + 3) & ~3;            // 16-byte aligned staging after it
  static_assert(R_END * 4 <= kWarps * kStages * SLOT, "epilogue scratch fits in the slots");
};

template <int G, int RK, int RV>
__global__ void __launch_bounds__(kThreads, 1) decode_tc_kernel(DecodeParams p) {
  using S = Shape<G, RK, RV>;
  constexpr int KST = RK / 16;                   // k-steps of the compressed logits
  constexpr int MVT = RV / 16;                   // m-tiles of the compressed value sum
  extern __shared__ __align__(128) unsigned char sm[];
  const lrkv_dims& D = p.D;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;         // MMA fragment coordinates
  const bool lo_col = t >= 2;                    // columns 4..7 hold the bf16 low parts
  const int ha = 2 * (t & 1);                    // heads ha, ha + 1 of this lane's two columns
  int T = p.C.seq_len[b];
  T = T < 0 ? 0 : (T > D.T_cap ? D.T_cap : T);
  const int n_chunks = T > 0 ? (T + p.chunk - 1) / p.chunk : 1;
  if (c >= n_chunks) return;
  const size_t bh = (size_t)b * D.Hkv + h;

  unsigned char* uk = sm + S::OFF_UK;
  unsigned char* uv = sm + S::OFF_UV;
  uint32_t* maskw = reinterpret_cast<uint32_t*>(sm + S::OFF_MASK);
  unsigned char* rowtab = sm + S::OFF_ROWS + warp * 16;   // compressed tile: row -> position offset
  uint64_t* merge_bar = reinterpret_cast<uint64_t*>(sm + S::OFF_BAR);
  uint64_t* base_bar = merge_bar + 1;
  float* R = reinterpret_cast<float*>(sm);       // epilogue scratch (slot area)
  __shared__ int s_last;

  const int c0 = c * p.chunk;
  const int c1 = min(T, c0 + p.chunk);
  const int n_pos = c1 > c0 ? c1 - c0 : 0;
  const int F = min(max(p.C.full_cnt[bh], 0), D.F_cap);
  const int share = (F + n_chunks - 1) / n_chunks;
  const int f0 = min(F, c * share), f1 = min(F, f0 + share);
  const int n_full = f1 - f0;
  const lrkv_bf16* ck = p.C.coef_k + bh * D.T_cap * RK;
  const lrkv_bf16* cv = p.C.coef_v + bh * D.T_cap * RV;
  const lrkv_bf16* fk = p.C.full_k + bh * D.F_cap * kD;
  const lrkv_bf16* fv = p.C.full_v + bh * D.F_cap * kD;

  // ---- prologue -------------------------------------------------------------------
  {  // zero the slots once: rows past a tile's count must hold finite values
    uint4* z = reinterpret_cast<uint4*>(sm);
    for (int i = tid; i < kWarps * kStages * S::SLOT / 16; i += kThreads) z[i] = make_uint4(0, 0, 0, 0);
  }
  const int n_words = (n_pos + 31) / 32;
  const uint32_t* mask_g = p.C.route_mask + bh * (D.T_cap / 32) + c0 / 32;
  for (int i = tid; i < n_words; i += kThreads) maskw[i] = mask_g[i];
  if (tid == 0) {
    mbar_init(merge_bar, 1);
    mbar_init(base_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0) {  // both bases into padded rows, one bulk copy per row
    const lrkv_bf16* Uk = p.C.U_k + (size_t)h * kD * RK;
    const lrkv_bf16* Uv = p.C.U_v + (size_t)h * kD * RV;
    if (lane == 0) mbar_arrive_expect_tx(base_bar, kD * 2u * (RK + RV));
    __syncwarp();
#pragma unroll
    for (int r = lane; r < kD; r += 32) {
      bulk_g2s(uk + r * S::KS, Uk + (size_t)r * RK, 2u * RK, base_bar);
      bulk_g2s(uv + r * S::VS, Uv + (size_t)r * RV, 2u * RV, base_bar);
    }
  }

  // this warp's tiles: full-rank ones first (they need only q), then compressed ones
  const int n_ct = (n_pos + kTileC - 1) / kTileC;
  const int n_ft = (n_full + kTileF - 1) / kTileF;
  const int nct_w = n_ct > warp ? (n_ct - warp + kWarps - 1) / kWarps : 0;
  const int nft_w = n_ft > warp ? (n_ft - warp + kWarps - 1) / kWarps : 0;
  const int n_tiles = nct_w + nft_w;
  unsigned char* ring = sm + (size_t)warp * kStages * S::SLOT;
  // tile i of this warp: i < nft_w -> full-rank tile warp + kWarps*i, else
  // compressed tile warp + kWarps*(i - nft_w)

  auto tile_bits = [&](int k) -> uint32_t {  // unmasked positions of compressed tile k
    const int rel = k * kTileC;
    const int nv = min(kTileC, n_pos - rel);
    const uint32_t valid = nv >= 16 ? 0xffffu : ((1u << nv) - 1u);
    return (~maskw[rel >> 5] >> (rel & 31)) & valid;
  };
  // one tile into its ring slot; consecutive lanes take consecutive 16-byte pieces
  auto issue = [&](int i) {
    unsigned char* slot = ring + (i % kStages) * S::SLOT;
    if (i >= nft_w) {
      constexpr int KP = RK / 8, VP = RV / 8;
      const int k = warp + kWarps * (i - nft_w);
      const uint32_t bits = tile_bits(k);
      const int nrows = __popc(bits);
      if (lane < kTileC && ((bits >> lane) & 1u))
        rowtab[__popc(bits & ((1u << lane) - 1u))] = (unsigned char)lane;
      __syncwarp();
      const lrkv_bf16* ckt = ck + (size_t)(c0 + k * kTileC) * RK;
      const lrkv_bf16* cvt = cv + (size_t)(c0 + k * kTileC) * RV;
      for (int q = lane; q < nrows * KP; q += 32) {
        const int r = q / KP, sg = q - r * KP;
        cp_async16(slot + r * S::KS + sg * 16, ckt + rowtab[r] * RK + sg * 8);
      }
      unsigned char* vslot = slot + kTileC * S::KS;
      for (int q = lane; q < nrows * VP; q += 32) {
        const int r = q / VP, sg = q - r * VP;
        cp_async16(vslot + r * S::VS + sg * 16, cvt + rowtab[r] * RV + sg * 8);
      }
      __syncwarp();
    } else {
      const int k = warp + kWarps * i;
      const int r0 = f0 + k * kTileF;
      const int n = min(kTileF, f1 - r0);
      const lrkv_bf16* fkt = fk + (size_t)r0 * kD;
      const lrkv_bf16* fvt = fv + (size_t)r0 * kD;
#pragma unroll
      for (int u = 0; u < kTileF * 16 / 32; ++u) {
        const int q = u * 32 + lane, r = q >> 4, sg = q & 15;
        if (r < n) {
          cp_async16(slot + r * S::FS + sg * 16, fkt + r * kD + sg * 8);
          cp_async16(slot + kTileF * S::FS + r * S::FS + sg * 16, fvt + r * kD + sg * 8);
        }
      }
    }
  };
  // the first tiles go out first; q in registers
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < n_tiles) issue(s);
    cp_async_commit();
  }
  // q as fragments over k = d: as the B operand of the full-rank logits (column
  // n = head n < G; q is bf16, hence exact, so no low-part columns) and, the same
  // bytes, as the A operand (rows = heads) of q~ = U_k^T q
  uint32_t qf0[8], qf1[8];
  {
    const lrkv_bf16* qrow = p.q + ((size_t)b * D.Hq + (size_t)h * G + (g < G ? g : 0)) * kD;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qf0[ks] = g < G ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * t) : 0u;
      qf1[ks] = g < G ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 8 + 2 * t) : 0u;
    }
  }
  const float scale = kLog2e * rsqrtf((float)kD);
  bool bases_ok = true;
  // q~ = U_k^T q as this warp's B fragments over k = r_k (column n < 4 = bf16 high
  // part of head n, n >= 4 = low part of head n - 4).  Each warp with compressed
  // tiles computes its own copy on the tensor cores once the bases have landed,
  // while its first tiles are in flight: no block barrier.
  uint32_t qb0[KST], qb1[KST];
  auto make_qtilde = [&]() {
    bases_ok = mbar_wait_bounded(base_bar, 0, kWaitIters);
    const int m = lane >> 3, rr = lane & 7;
#pragma unroll
    for (int ks2 = 0; ks2 < KST; ++ks2) {      // columns [16 ks2, 16 ks2 + 16) of q~
      float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(b0, b1, b2, b3, uk + (ks * 16 + (m & 1) * 8 + rr) * S::KS + (16 * ks2 + (m >> 1) * 8) * 2);
        mma_16816(a0, qf0[ks], 0u, qf1[ks], 0u, b0, b1);
        mma_16816(a1, qf0[ks], 0u, qf1[ks], 0u, b2, b3);
      }
      // lane (g, t) holds q~[head g][16 ks2 + 2t (+1)] in a0 and [+8] in a1 (rows g < 4);
      // the low-part columns n = g >= 4 take head g - 4 from lane ^ 16
      float x0 = __shfl_xor_sync(kFull, a0[0], 16), x1 = __shfl_xor_sync(kFull, a0[1], 16);
      float y0 = __shfl_xor_sync(kFull, a1[0], 16), y1 = __shfl_xor_sync(kFull, a1[1], 16);
      const bool lo_n = g >= 4;
      if (!lo_n) x0 = a0[0], x1 = a0[1], y0 = a1[0], y1 = a1[1];
      const bool live = (g & 3) < G;
      qb0[ks2] = live ? pack_bf16(bf16_part(x0 * scale, lo_n), bf16_part(x1 * scale, lo_n)) : 0u;
      qb1[ks2] = live ? pack_bf16(bf16_part(y0 * scale, lo_n), bf16_part(y1 * scale, lo_n)) : 0u;
    }
  };
  if (nct_w > 0) make_qtilde();     // overlaps the first tiles' flight

  // ---- stream the tiles ------------------------------------------------------------
  // lane state: running max and sum of heads ha, hb; accumulators O^T (rows =
  // value columns, columns = head parts) for the compressed and full-rank sums
  float ma = -INFINITY, mb = -INFINITY, la = 0.f, lb = 0.f;
  float oc[MVT][4], of[8][4];
#pragma unroll
  for (int mt = 0; mt < MVT; ++mt) oc[mt][0] = oc[mt][1] = oc[mt][2] = oc[mt][3] = 0.f;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) of[mt][0] = of[mt][1] = of[mt][2] = of[mt][3] = 0.f;

  // Online softmax over one tile: s = {head ha at token g, hb at g, ha at g+8,
  // hb at g+8} (-inf = no token).  Rescales this lane's accumulator columns when
  // a max grows and returns the probabilities.
  auto softmax = [&](const float (&s)[4], float (&pr)[4]) {
    float xa = fmaxf(s[0], s[2]), xb = fmaxf(s[1], s[3]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      xa = fmaxf(xa, __shfl_xor_sync(kFull, xa, o));
      xb = fmaxf(xb, __shfl_xor_sync(kFull, xb, o));
    }
    if (xa > ma || xb > mb) {
      const float na = fmaxf(ma, xa), nb = fmaxf(mb, xb);
      const float sa = ma == -INFINITY ? 0.f : exp2f(ma - na);
      const float sb = mb == -INFINITY ? 0.f : exp2f(mb - nb);
      la *= sa;
      lb *= sb;
#pragma unroll
      for (int mt = 0; mt < MVT; ++mt) oc[mt][0] *= sa, oc[mt][2] *= sa, oc[mt][1] *= sb, oc[mt][3] *= sb;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) of[mt][0] *= sa, of[mt][2] *= sa, of[mt][1] *= sb, of[mt][3] *= sb;
      ma = na;
      mb = nb;
    }
    __syncwarp();
    pr[0] = s[0] == -INFINITY ? 0.f : exp2f(s[0] - ma);
    pr[1] = s[1] == -INFINITY ? 0.f : exp2f(s[1] - mb);
    pr[2] = s[2] == -INFINITY ? 0.f : exp2f(s[2] - ma);
    pr[3] = s[3] == -INFINITY ? 0.f : exp2f(s[3] - mb);
    la += pr[0] + pr[2];
    lb += pr[1] + pr[3];
  };

  const int lm = lane >> 3, lr = lane & 7;       // ldmatrix address roles
  for (int i = 0; i < n_tiles; ++i) {
    if (i + kStages - 1 < n_tiles) issue(i + kStages - 1);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    __syncwarp();
    const unsigned char* slot = ring + (i % kStages) * S::SLOT;
    if (i >= nft_w) {
      // compressed tile: S^T[token][head part] = C_k q~^T, then O^T += C_v^T P^T
      const int nrows = __popc(tile_bits(warp + kWarps * (i - nft_w)));
      float st[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < KST; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(a0, a1, a2, a3, slot + ((lm & 1) * 8 + lr) * S::KS + (ks * 16 + (lm >> 1) * 8) * 2);
        mma_16816(st, a0, a1, a2, a3, qb0[ks], qb1[ks]);
      }
      float s[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        s[x] = st[x] + __shfl_xor_sync(kFull, st[x], 2);      // high part + low part
        if (g + (x >> 1) * 8 >= nrows) s[x] = -INFINITY;
      }
      float pr[4];
      softmax(s, pr);
      const uint32_t top = pack_bf16(bf16_part(pr[0], lo_col), bf16_part(pr[1], lo_col));
      const uint32_t bot = pack_bf16(bf16_part(pr[2], lo_col), bf16_part(pr[3], lo_col));
      const uint32_t pb0 = movmatrix_t(top), pb1 = movmatrix_t(bot);
      const unsigned char* vrows = slot + kTileC * S::KS;
#pragma unroll
      for (int mt = 0; mt < MVT; ++mt) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(a0, a1, a2, a3, vrows + ((lm >> 1) * 8 + lr) * S::VS + (mt * 16 + (lm & 1) * 8) * 2);
        mma_16816(oc[mt], a0, a1, a2, a3, pb0, pb1);
      }
    } else {
      // full-rank tile: 8 tokens (the MMA's rows 8..15 repeat them and are masked)
      const int k = warp + kWarps * i;
      const int nrows = min(kTileF, f1 - (f0 + k * kTileF));
      float st[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kp = 0; kp < 4; ++kp) {
        uint32_t r0, r1, r2, r3;
        ldsm_x4(r0, r1, r2, r3, slot + lr * S::FS + ((2 * kp + (lm >> 1)) * 16 + (lm & 1) * 8) * 2);
        mma_16816(st, r0, r0, r1, r1, qf0[2 * kp], qf1[2 * kp]);
        mma_16816(st, r2, r2, r3, r3, qf0[2 * kp + 1], qf1[2 * kp + 1]);
      }
      float s[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        s[x] = (st[x] + __shfl_xor_sync(kFull, st[x], 2)) * scale;   // low-part columns are 0 here
        if (x >= 2 || g >= nrows) s[x] = -INFINITY;
      }
      float pr[4];
      softmax(s, pr);
      const uint32_t top = pack_bf16(bf16_part(pr[0], lo_col), bf16_part(pr[1], lo_col));
      const uint32_t pb0 = movmatrix_t(top);
      const unsigned char* vrows = slot + kTileF * S::FS;
#pragma unroll
      for (int mp = 0; mp < 4; ++mp) {
        uint32_t r0, r1, r2, r3;
        ldsm_x4_t(r0, r1, r2, r3, vrows + lr * S::FS + (mp * 32 + lm * 8) * 2);
        mma_16816(of[2 * mp], r0, r1, r0, r1, pb0, 0u);
        mma_16816(of[2 * mp + 1], r2, r3, r2, r3, pb0, 0u);
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  __syncthreads();                                 // every warp is done with the slots

  // ---- per-warp results into the slot area ----------------------------------------
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    la += __shfl_xor_sync(kFull, la, o);
    lb += __shfl_xor_sync(kFull, lb, o);
  }
#pragma unroll
  for (int mt = 0; mt < MVT; ++mt)
#pragma unroll
    for (int x = 0; x < 4; ++x) oc[mt][x] += __shfl_xor_sync(kFull, oc[mt][x], 2);
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int x = 0; x < 4; ++x) of[mt][x] += __shfl_xor_sync(kFull, of[mt][x], 2);
  if (t < 2) {
    // lane (g, t<2): heads ha, hb; value columns mt*16 + g and mt*16 + g + 8
#pragma unroll
    for (int hx = 0; hx < 2; ++hx) {
      const int hd = ha + hx;
      if (hd < G) {
        float* pc = R + S::R_PC + (warp * G + hd) * RV;
        float* pf = R + S::R_PF + (warp * G + hd) * kD;
#pragma unroll
        for (int mt = 0; mt < MVT; ++mt) pc[mt * 16 + g] = oc[mt][hx], pc[mt * 16 + g + 8] = oc[mt][2 + hx];
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) pf[mt * 16 + g] = of[mt][hx], pf[mt * 16 + g + 8] = of[mt][2 + hx];
        if (g == 0) {
          R[S::R_WM + warp * G + hd] = hx == 0 ? ma : mb;
          R[S::R_WL + warp * G + hd] = hx == 0 ? la : lb;
        }
      }
    }
  }
  __syncthreads();

  // ---- merge the warps -------------------------------------------------------------
  if (tid < G) {
    float M = -INFINITY;
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, R[S::R_WM + w * G + tid]);
    float Ls = 0.f;
    for (int w = 0; w < kWarps; ++w) {
      const float mw = R[S::R_WM + w * G + tid];
      const float e = mw == -INFINITY ? 0.f : exp2f(mw - M);
      R[S::R_WE + w * G + tid] = e;
      Ls = fmaf(R[S::R_WL + w * G + tid], e, Ls);
    }
    R[S::R_M + tid] = M;
    R[S::R_M + G + tid] = Ls;
  }
  __syncthreads();
  for (int o = tid; o < G * RV; o += kThreads) {
    const int gi = o / RV;
    float x = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) x = fmaf(R[S::R_PC + w * G * RV + o], R[S::R_WE + w * G + gi], x);
    R[S::R_CC + o] = x;
  }
  for (int o = tid; o < G * kD; o += kThreads) {
    const int gi = o / kD;
    float x = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) x = fmaf(R[S::R_PF + w * G * kD + o], R[S::R_WE + w * G + gi], x);
    R[S::R_CF + o] = x;
  }
  __syncthreads();

  // ---- lift by U_v on the tensor cores, write this split's record ------------------
  if (!mbar_wait_bounded(base_bar, 0, kWaitIters)) bases_ok = false;
  if (!bases_ok && lane == 0) atomicOr(p.C.dev_status, LRKV_DEV_WAIT_TIMEOUT);
  {
    // A = merged acc_c split into hi (rows 0..3) / lo (rows 4..7) parts over
    // k = r_v; B = U_v rows (n = output column); warp w owns columns 8w..8w+7
    const int hh = g & 3;
    const bool lo_row = g >= 4;
    float l0[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < RV / 16; ++ks) {
      uint32_t a0 = 0u, a2 = 0u;
      if (hh < G) {
        const float* row = R + S::R_CC + hh * RV + ks * 16 + 2 * t;
        a0 = pack_bf16(bf16_part(row[0], lo_row), bf16_part(row[1], lo_row));
        a2 = pack_bf16(bf16_part(row[8], lo_row), bf16_part(row[9], lo_row));
      }
      uint32_t b0, b1, b2, b3;   // (cols 8w.., k lo), (cols 8w.., k hi), repeated
      ldsm_x4(b0, b1, b2, b3, uv + (8 * warp + lr) * S::VS + (ks * 16 + (lm & 1) * 8) * 2);
      mma_16816(l0, a0, 0u, a2, 0u, b0, b1);
    }
#pragma unroll
    for (int x = 0; x < 2; ++x) l0[x] += __shfl_xor_sync(kFull, l0[x], 16);
    float* rec0 = p.partials + (bh * p.n_chunk_max + c) * G * (size_t)kRecFloats;
    if (g < G) {
      const int i0 = 8 * warp + 2 * t;
      const float* cf = R + S::R_CF + g * kD;
      float* o = rec0 + g * kRecFloats + 4;
      o[i0] = l0[0] + cf[i0];
      o[i0 + 1] = l0[1] + cf[i0 + 1];
    }
    if (tid < G) {
      rec0[tid * kRecFloats] = R[S::R_M + tid];
      rec0[tid * kRecFloats + 1] = R[S::R_M + G + tid];
    }
  }

  // ---- the last split of this (batch row, kv head) merges every record ------------
  __syncthreads();
  if (tid == 0) s_last = atom_add_acq_rel_gpu(p.tickets + bh, 1) == n_chunks - 1;
  __syncthreads();
  if (!s_last) return;
  // one pass: records streamed by bulk copy into the (idle) slot area, merged
  // with a running max per head
  const float* recs = p.partials + bh * p.n_chunk_max * G * (size_t)kRecFloats;
  constexpr int kRecBytes = G * kRecFloats * 4;
  constexpr int kStageFloats = (kWarps * kStages * S::SLOT) / 4;
  constexpr int per_batch = (kStageFloats - S::R_END) * 4 / kRecBytes;
  float* stage = R + S::R_END;                    // 16-byte aligned
  constexpr int NO = (G * kD + kThreads - 1) / kThreads;
  float acc_o[NO], m_o[NO], l_o[NO];
#pragma unroll
  for (int u = 0; u < NO; ++u) acc_o[u] = 0.f, m_o[u] = -INFINITY, l_o[u] = 0.f;
  int batch = 0;
  for (int cb = 0; cb < n_chunks; cb += per_batch, ++batch) {
    const int nb = min(per_batch, n_chunks - cb);
    if (tid == 0) {
      fence_proxy_async_smem();
      fence_proxy_async_global();
      mbar_arrive_expect_tx(merge_bar, nb * kRecBytes);
      bulk_g2s(stage, recs + (size_t)cb * G * kRecFloats, nb * kRecBytes, merge_bar);
    }
    const bool timed_out = !mbar_wait_bounded(merge_bar, batch & 1, kWaitIters);
    if (__syncthreads_or(timed_out)) {
      if (tid == 0) atomicOr(p.C.dev_status, LRKV_DEV_WAIT_TIMEOUT);
      break;
    }
#pragma unroll
    for (int u = 0; u < NO; ++u) {
      const int o = tid + u * kThreads;
      if (o < G * kD) {
        const int gi = o / kD, ii = o % kD;
        float mx = m_o[u];
        for (int k2 = 0; k2 < nb; ++k2) mx = fmaxf(mx, stage[(k2 * G + gi) * kRecFloats]);
        const float sc = m_o[u] == -INFINITY ? 0.f : exp2f(m_o[u] - mx);
        float x = acc_o[u] * sc, l = l_o[u] * sc;
        for (int k2 = 0; k2 < nb; ++k2) {
          const float* rc = stage + (k2 * G + gi) * kRecFloats;
          const float w = rc[0] == -INFINITY ? 0.f : exp2f(rc[0] - mx);
          x = fmaf(w, rc[4 + ii], x);
          l = fmaf(w, rc[1], l);
        }
        acc_o[u] = x, l_o[u] = l, m_o[u] = mx;
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < NO; ++u) {
    const int o = tid + u * kThreads;
    if (o < G * kD) {
      const int gi = o / kD, ii = o % kD;
      p.out[((size_t)b * D.Hq + (size_t)h * G + gi) * kD + ii] = l_o[u] > 0.f ? acc_o[u] / l_o[u] : 0.f;
    }
  }
  if (tid == 0) p.tickets[bh] = 0;
}

}  // namespace tc
}  // namespace lrkv
