// Write path for prefill-sized appends on the 5th-generation tensor cores.
//
// OjaKV repository README, "Method Summary": a fixed per-head basis U
// (StaticPCA) and the hybrid policy that keeps tokens whose reconstruction
// error is high in full rank (OjaKV).  For every new row x (a key with U_k, a
// value with U_v):
//   c = U^T x                       (fp32 accumulation, stored as bf16 RNE)
//   e = ||x - U c|| / ||x||         (0 when x = 0)
// Since c = U^T x, the residual is x - U U^T x = P x with P = I - U U^T, the
// same quantity computed in one product; U is bf16 and not exactly
// orthonormal, so P is not a projector and no norm identity is used.
//
// Kernel 1, project_tc_kernel: each CTA works on a contiguous run of the
// 128-token tiles of one (kv head, K or V) group.  Per CTA, P is formed once
// on the tensor cores (U U^T) and split into bf16 high and low parts (P =
// P_hi + P_lo to 2^-17).
// Per tile, TMA brings the 128 x 128 input rows (128-byte swizzle); one
// thread issues
//     [D2 | D1] = X [P_hi | U]   (M 128, N 128 + r, K 128)
//     D2       += X P_lo^T       (M 128, N 128)
// into tensor memory (double-buffered): D1 = X U holds the coefficients and
// D2 = X P^T the residual vectors.  P_hi and U^T sit back to back in shared
// memory as one B operand, so each K slice of X is read twice per tile, not
// three times: the MMAs read their operands from shared memory at close to
// its bandwidth, and every byte saved there also speeds up the loads and the
// epilogue, which share it.  Eight epilogue warps (two per token row) store
// bf16(c), sum the squared residual and the squared input, and write e.  Up
// to four input stages and two accumulator buffers let the loads, the MMAs
// and the epilogue of consecutive tiles overlap.
//
// Kernel 2, route_count_kernel: e_t = max(e_k, e_v); routed iff e_t > tau.
// Per 128-token tile: err_out, the routed bits (warp ballots) and their count.
//
// Kernel 3, route_scatter_kernel: the list slot of a routed token is the
// list length before the call + routed tokens of earlier tiles (a block sum
// over the tile counts) + earlier routed tokens of its tile (ballot prefix),
// so the list stays in position order.  A CTA takes a run of up to 8 tiles of
// one (b, kv head) when the grid is large (fewer CTAs, fewer same-address
// tickets); their kept rows are listed in shared memory and copied
// warp-cooperatively, 8 rows per warp with every load before the first store.
// Mask words are updated with atomics where tiles share a word.  The last CTA
// of each (b, kv head) sets full_cnt; the last CTA of the grid advances seq_len.
#pragma once

#include <cuda.h>

#include "compress_params.cuh"
#include "lrkv_common.cuh"
#include "ptx.cuh"
#include "tc_ptx.cuh"

namespace lrkv {
namespace ptc {

constexpr int kTile = 128;                 // tokens per tile (MMA M)
constexpr int kMaxStages = 4;              // input stages (fewer when shared memory is short)
constexpr int kThreads = 320;              // warps 0-7 epilogue, 8 TMA, 9 MMA + TMEM
constexpr int kEpi = 256;                  // epilogue threads: two per token row
constexpr int kTmaWarp = 8, kMmaWarp = 9;
constexpr int kStageBytes = kTile * kD * 2;          // two 64-column boxes
constexpr int kBoxBytes = kStageBytes / 2;
constexpr uint32_t kTmemCols = 512;                  // two buffers of [D1 | D2]
constexpr uint32_t kWaitIters = 1u << 22;
constexpr size_t kSmemLimit = 227 * 1024;
constexpr int kMaxRanges = 256;                      // tile ranges of the end-to-end split

// Shared memory (bytes) for rank rm (the larger rank of the launch: both
// tensors share one layout) and ns input stages; operand regions 1024-aligned.
//   X stages [ns][128][128] (128-byte swizzle), P_hi [128][128] directly
//   followed by U^T [rm][128] (rows 128.. of the merged B operand),
//   P_lo [128][128], mbarriers, group B's per-row sums [2][128], the key
//   mean's constants [2][128] (U^T mu and P mu, attention-aware keys only).
// U [128][rm] for U U^T is needed only before the first tile: it borrows the
// last input stage; the query-side key basis U_q of an attention-aware key
// basis (P = I - U_q U^T) borrows the one before.
struct Layout {
  int x, phi, plo, ut, u, uq, bar, part, mu, amx;
  size_t bytes;
  __host__ __device__ Layout(int rm, int ns) {
    x = 0;
    phi = ns * kStageBytes;
    ut = phi + kD * kD * 2;
    plo = ut + rm * kD * 2;
    u = (ns - 1) * kStageBytes;
    uq = (ns - 2) * kStageBytes;
    bar = plo + kD * kD * 2;
    part = bar + 128;
    mu = part + 2 * kTile * 8;
    amx = mu + 2 * kD * 4;                   // [2][2][128] u32: the two groups' row amax halves
    bytes = (size_t)amx + 2 * 2 * kTile * 4 + 1024;   // + slack to align the base to 1024
  }
};
static_assert(kD * 128 * 2 <= kStageBytes, "U fits in one input stage");
inline int stages_for(int rm) {
  int ns = kMaxStages;
  while (ns > 2 && Layout(rm, ns).bytes > kSmemLimit) --ns;
  return ns;
}

struct Params {
  CUtensorMap map_k;     // k_new viewed as [B*t_new][Hkv][d], box {64, 1, 128}
  CUtensorMap map_v;
  lrkv_dims D;
  lrkv_cache C;
  int t_new;
  const int32_t* t_new_b;
  float* errs;           // [2][B][Hkv][T_cap]
  int tiles_per_b;       // ceil(min(t_new, T_cap) / 128)
  int r_max;             // max(r_k, r_v): the shared-memory layout
  int n_stages;          // input stages: stages_for(r_max)
  uint32_t wait_iters;   // limit of the MMA issuer's wait for each input tile (kWaitIters)
  // Which tiles a CTA takes.  per_group > 0: that many CTAs per group, CTA x
  // on group x / per_group.  per_group = 0: the groups' tiles laid end to end
  // are cut into n_ranges equal ranges (one per SM, each within two groups);
  // CTA x < n_ranges takes range x up to its group's end, and CTA n_ranges + k
  // the rest of range second[k] (those rests in decreasing length, so that the
  // SM that finishes its first part soonest picks up the longest rest).
  int per_group;
  int n_ranges;
  uint16_t second[kMaxRanges];
};

// This CTA's group and tiles [u_begin, u_end) of it (Params: per_group).
__device__ __forceinline__ int cta_tiles(const Params& p, int n_units, int* u_begin, int* u_end) {
  const int x = (int)blockIdx.x;
  if (p.per_group > 0) {
    const int grp = x / p.per_group, sub = x - grp * p.per_group;
    const int q = n_units / p.per_group, r = n_units - q * p.per_group;
    *u_begin = sub * q + min(sub, r);
    *u_end = *u_begin + q + (sub < r ? 1 : 0);
    return grp;
  }
  const int total = 2 * p.D.Hkv * n_units;
  const int q = total / p.n_ranges, r = total - q * p.n_ranges;
  const bool first = x < p.n_ranges;
  const int rg = first ? x : p.second[x - p.n_ranges];
  const int l0 = rg * q + min(rg, r), l1 = l0 + q + (rg < r ? 1 : 0);
  const int grp = l0 / n_units + (first ? 0 : 1);
  *u_begin = first ? l0 - grp * n_units : 0;
  *u_end = min(l1 - grp * n_units, n_units);
  return grp;
}

// Byte offset of element (row n, column k) in a no-swizzle K-major operand:
// 8x8 core matrices of 128 contiguous bytes, K-adjacent ones 128 B apart and
// 8-row groups `sbo` bytes apart.
__device__ __forceinline__ int core_off(int n, int k, int sbo) {
  return (n >> 3) * sbo + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2;
}

// Tokens of row b in this call, and the position of the first one.
__device__ __forceinline__ int eff_tokens(const Params& p, int b, int* start) {
  uint32_t st = 0;
  const int n = new_tokens(p.t_new_b, b, p.t_new, &st);
  const int s0 = min(max(p.C.seq_len[b], 0), p.D.T_cap);
  int ne = p.D.T_cap - s0;
  if (ne > n) ne = n;
  if (ne < 0) ne = 0;
  *start = s0;
  return ne;
}

// eff_tokens of the last row asked for: a CTA's units are a contiguous range
// of (row, tile), so the row changes rarely and its length is loaded once.
struct RowLen {
  int b = -1, ne = 0, start = 0;
  __device__ __forceinline__ int get(const Params& p, int bb, int* st) {
    if (bb != b) {
      b = bb;
      ne = eff_tokens(p, bb, &start);
    }
    *st = start;
    return ne;
  }
};

// Bounded wait that also gives up once another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag,
                                              uint32_t max_iters = kWaitIters) {
  for (uint32_t i = 0; i < max_iters; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 63 && *abort_flag) return false;
    if (i > 64) __nanosleep(32);
  }
  *abort_flag = 1;
  return false;
}

// 1-d grid (Params: per_group); group = 2 h + tensor (0 keys, 1 values).
// CB: stored coefficient format, 16 (bf16) or 8, 4 (codes with per-row scales).
template <int CB>
__global__ void __launch_bounds__(kThreads, 1) project_tc_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the dynamic window is only guaranteed 16-byte aligned: round up to 1024
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const lrkv_dims& D = p.D;
  // the routing passes may launch now: they wait for this grid to finish
  griddep_launch_dependents();
  const int n_units = D.B * p.tiles_per_b;
  int u_begin, u_end;
  const int group = cta_tiles(p, n_units, &u_begin, &u_end), tensor = group & 1, h = group >> 1;
  const CUtensorMap* map = tensor == 0 ? &p.map_k : &p.map_v;
  const int R = tensor == 0 ? D.r_k : D.r_v;
  const int NS = p.n_stages;
  const Layout Lo(p.r_max, NS);
  const lrkv_bf16* Ug = (tensor == 0 ? p.C.U_k : p.C.U_v) + (size_t)h * kD * R;
  // attention-aware keys: the query-side basis reconstructs, the mean is subtracted
  const lrkv_bf16* Uqg = tensor == 0 && p.C.U_kq ? p.C.U_kq + (size_t)h * kD * R : nullptr;
  const float* mug = tensor == 0 && p.C.mu_k ? p.C.mu_k + (size_t)h * kD : nullptr;
  unsigned char* coef = static_cast<unsigned char*>(tensor == 0 ? p.C.coef_k : p.C.coef_v);
  const bool coef32 = (reinterpret_cast<uintptr_t>(coef) & 31u) == 0;   // 32-byte stores allowed
  float* scales = tensor == 0 ? p.C.scale_k : p.C.scale_v;
  float* errs = p.errs + (size_t)tensor * D.B * D.Hkv * D.T_cap;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lo.bar);
  uint64_t* full = bars;                 // [NS] TMA -> MMA
  uint64_t* empty = bars + kMaxStages;   // [NS] epilogue -> TMA (kEpi arrivals)
  uint64_t* dready = bars + 2 * kMaxStages;  // [2] MMA -> epilogue
  uint64_t* tfree = dready + 2;          // [2] epilogue -> MMA (128 arrivals)
  uint64_t* pready = tfree + 2;          // U U^T done
  uint64_t* drain = pready + 1;          // final MMA drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kEpi);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&dready[b], 1);
      mbar_init(&tfree[b], kEpi);
    }
    mbar_init(pready, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tc5::tmem_alloc(tmem_slot, kTmemCols);
    tc5::tmem_relinquish();
  }
  if (warp == kTmaWarp && lane == 0) tc5::prefetch_tensormap(map);
  // U into two K-major no-swizzle operand layouts:
  //   U   as [m = i][k = j]   (A and B of U U^T), 8-row groups 16 r bytes apart
  //   U^T as [n = j][k = i]   (B of X U),         8-row groups 2048 bytes apart
  // Every 16-byte piece of U (8 columns of one row, r a multiple of 16) is
  // loaded before the first store, so the loads share one memory latency.
  {
    unsigned char* su = sm + Lo.u;
    unsigned char* sut = sm + Lo.ut;
    constexpr int kMaxPieces = (kD * kD / 8 + kThreads - 1) / kThreads;
    const int n_pieces = kD * R / 8;
    const uint4* ug = reinterpret_cast<const uint4*>(Ug);
    uint4 piece[kMaxPieces];
#pragma unroll
    for (int k = 0; k < kMaxPieces; ++k) {
      const int c = tid + k * kThreads;
      if (c < n_pieces) piece[k] = ug[c];
    }
#pragma unroll
    for (int k = 0; k < kMaxPieces; ++k) {
      const int c = tid + k * kThreads;
      if (c < n_pieces) {
        const int i = (c * 8) / R, j0 = c * 8 - i * R;
        *reinterpret_cast<uint4*>(su + core_off(i, j0, 16 * R)) = piece[k];
        const uint32_t w[4] = {piece[k].x, piece[k].y, piece[k].z, piece[k].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          *reinterpret_cast<uint16_t*>(sut + core_off(j0 + 2 * q, i, 2048)) = (uint16_t)(w[q] & 0xffffu);
          *reinterpret_cast<uint16_t*>(sut + core_off(j0 + 2 * q + 1, i, 2048)) = (uint16_t)(w[q] >> 16);
        }
      }
    }
    if (Uqg) {   // the query-side key basis, in U's layout (the A operand of U_q U^T)
      const uint4* uq = reinterpret_cast<const uint4*>(Uqg);
#pragma unroll
      for (int k = 0; k < kMaxPieces; ++k) {
        const int c = tid + k * kThreads;
        if (c < n_pieces) piece[k] = uq[c];
      }
#pragma unroll
      for (int k = 0; k < kMaxPieces; ++k) {
        const int c = tid + k * kThreads;
        if (c < n_pieces) {
          const int i = (c * 8) / R, j0 = c * 8 - i * R;
          *reinterpret_cast<uint4*>(sm + Lo.uq + core_off(i, j0, 16 * R)) = piece[k];
        }
      }
    }
  }
  fence_proxy_async_smem();
  tc5::fence_before_sync();
  __syncthreads();
  tc5::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // ---- P = I - U_q U^T (U_q = U unless an attention-aware key basis is given),
  // split into bf16 high and low parts -----------------------------------------------
  if (warp == kMmaWarp && lane == 0) {
    const uint32_t ub = smem_u32(sm + Lo.u);
    const uint32_t uqb = smem_u32(sm + (Uqg ? Lo.uq : Lo.u));
    for (int j = 0; j < R / 16; ++j) {
      const uint64_t db = tc5::smem_desc(ub + j * 256, 128, 16 * R, tc5::kSwizzleNone);
      const uint64_t da = tc5::smem_desc(uqb + j * 256, 128, 16 * R, tc5::kSwizzleNone);
      tc5::mma_bf16(tmem + 128, da, db, tc5::idesc_bf16_f32(128, 128), j > 0);
    }
    tc5::mma_commit(pready);
  }
  // attention-aware keys with a mean: the per-column constants U^T mu (from the
  // coefficients) and P mu = mu - U_q U^T mu (from the residual vectors)
  float* cmu = reinterpret_cast<float*>(sm + Lo.mu);   // [128]: U^T mu, columns < R
  float* rmu = cmu + kD;                               // [128]: P mu
  if (mug && warp < 8) {
    if (tid < R) {
      float a = 0.f;
      for (int i = 0; i < kD; ++i) a = fmaf(bf2f(Ug[i * R + tid]), mug[i], a);
      cmu[tid] = a;
    }
    tc5::named_bar_sync(1, kEpi);
    if (tid < kD) {
      const lrkv_bf16* uq = Uqg ? Uqg : Ug;
      float a = 0.f;
      for (int j = 0; j < R; ++j) a = fmaf(bf2f(uq[tid * R + j]), cmu[j], a);
      rmu[tid] = mug[tid] - a;
    }
  }
  if (warp < 8) {
    // row m of U U^T = TMEM lane m; warps w and w + 4 share the rows, columns split
    const int m = (warp & 3) * 32 + lane;
    const int cbeg = (warp >> 2) * 64;
    if (!wait_or_abort(pready, 0, abort_flag)) {
      atomicOr(p.C.dev_status, LRKV_DEV_WAIT_TIMEOUT);
    }
    tc5::fence_after_sync();
    unsigned char* phi = sm + Lo.phi;
    unsigned char* plo = sm + Lo.plo;
#pragma unroll 1
    for (int c0 = cbeg; c0 < cbeg + 64; c0 += 16) {
      float v[16];
      tc5::tmem_ld16(tmem + ((uint32_t)((warp & 3) * 32) << 16) + 128 + c0, v);
      tc5::tmem_wait_ld();
      uint32_t hi[8], lo[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float a = (m == c0 + 2 * q ? 1.f : 0.f) - v[2 * q];
        float b = (m == c0 + 2 * q + 1 ? 1.f : 0.f) - v[2 * q + 1];
        const float ah = __bfloat162float(__float2bfloat16_rn(a));
        const float bh = __bfloat162float(__float2bfloat16_rn(b));
        hi[q] = pack_bf16(ah, bh);
        lo[q] = pack_bf16(a - ah, b - bh);
      }
      // row m of P is row n = m of the B operand, columns c0..c0+15 = two core matrices
      *reinterpret_cast<uint4*>(phi + core_off(m, c0, 2048)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(phi + core_off(m, c0 + 8, 2048)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
      *reinterpret_cast<uint4*>(plo + core_off(m, c0, 2048)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint4*>(plo + core_off(m, c0 + 8, 2048)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
    }
  }
  fence_proxy_async_smem();
  tc5::fence_before_sync();
  __syncthreads();
  tc5::fence_after_sync();

  // ---- pipeline over this CTA's tiles -------------------------------------------------
  if (warp == kTmaWarp) {
    // TMA producer
    if (lane == 0) {
      int i = 0;
      RowLen rl;
      for (int u = u_begin; u < u_end && !*abort_flag; ++u) {
        const int b = u / p.tiles_per_b, t0 = (u - b * p.tiles_per_b) * kTile;
        int start;
        if (t0 >= rl.get(p, b, &start)) continue;
        const int s = i % NS;
        if (i >= NS && !wait_or_abort(&empty[s], ((i / NS) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        unsigned char* dst = sm + Lo.x + s * kStageBytes;
        const int z = b * p.t_new + t0;
        tc5::tma_load_3d(dst, map, 0, h, z, &full[s]);
        tc5::tma_load_3d(dst + kBoxBytes, map, 64, h, z, &full[s]);
        ++i;
      }
      // leave no copy in flight: wait for the last fill of every stage
      for (int k = (i > NS ? i - NS : 0); k < i; ++k)
        mbar_wait_bounded(&full[k % NS], (k / NS) & 1, kWaitIters);
    }
  } else if (warp == kMmaWarp) {
    // MMA issuer
    if (lane == 0) {
      const uint32_t idesc1 = tc5::idesc_bf16_f32(128, 128 + R);
      const uint32_t idesc2 = tc5::idesc_bf16_f32(128, 128);
      const uint32_t xbase = smem_u32(sm + Lo.x);
      const uint32_t phb = smem_u32(sm + Lo.phi);   // P_hi rows, then U^T rows
      const uint32_t plb = smem_u32(sm + Lo.plo);
      int i = 0;
      RowLen rl;
      for (int u = u_begin; u < u_end && !*abort_flag; ++u) {
        const int b = u / p.tiles_per_b, t0 = (u - b * p.tiles_per_b) * kTile;
        int start;
        if (t0 >= rl.get(p, b, &start)) continue;
        const int s = i % NS, buf = i & 1;
        if (!wait_or_abort(&full[s], (i / NS) & 1, abort_flag, p.wait_iters)) break;
        if (i >= 2 && !wait_or_abort(&tfree[buf], ((i >> 1) - 1) & 1, abort_flag)) break;
        tc5::fence_after_sync();
        const uint32_t d2 = tmem + buf * 256;   // D2 columns [0, 128), D1 [128, 128 + R)
        const uint32_t xs = xbase + s * kStageBytes;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint64_t a = tc5::smem_desc(xs + (j >> 2) * kBoxBytes + (j & 3) * 32, 16, 1024,
                                            tc5::kSwizzle128B);
          tc5::mma_bf16(d2, a, tc5::smem_desc(phb + j * 256, 128, 2048, tc5::kSwizzleNone), idesc1,
                        j > 0);
          tc5::mma_bf16(d2, a, tc5::smem_desc(plb + j * 256, 128, 2048, tc5::kSwizzleNone), idesc2,
                        1);
        }
        tc5::mma_commit(&dready[buf]);
        ++i;
      }
      // every MMA done before the epilogue leaves and TMEM is freed
      tc5::mma_commit(drain);
      mbar_wait_bounded(drain, 0, kWaitIters);
    }
  } else {
    // epilogue: two threads per token row m = TMEM lane m.  Group A (warps 0-3)
    // stores the coefficients and sums the squared residual of columns 0-63;
    // group B (warps 4-7) sums columns 64-127 and the squared input, and hands
    // its sums to A through shared memory (double-buffered by tile parity).
    const int m = (warp & 3) * 32 + lane;
    const bool grp_a = warp < 4;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    float2* part = reinterpret_cast<float2*>(sm + Lo.part);   // [2][128]
    int i = 0;
    RowLen rl;
    for (int u = u_begin; u < u_end; ++u) {
      const int b = u / p.tiles_per_b, t0 = (u - b * p.tiles_per_b) * kTile;
      int start;
      const int ne = rl.get(p, b, &start);
      if (t0 >= ne) continue;
      const int s = i % NS, buf = i & 1;
      // every epilogue thread stops together, so the named barriers below
      // always see all of them
      const bool ok = wait_or_abort(&dready[buf], (i >> 1) & 1, abort_flag);
      if (!tc5::named_bar_and(1, kEpi, ok)) break;
      tc5::fence_after_sync();
      const int t = t0 + m;
      const bool valid = t < ne;
      const size_t bh = (size_t)b * D.Hkv + h;
      const uint32_t d2 = lane_base + buf * 256, d1 = d2 + 128;
      float rs = 0.f, xs = 0.f;
      if (CB < 16) {
        // quantised rows: each group takes half of the coefficient columns (A
        // the first Rh, B the rest) in two TMEM passes, 32 columns per wait
        // (c = U^T x - U^T mu with a key mean): its part of the row's amax of
        // bf16(c), exchanged through shared memory, then its codes; A stores
        // the scale
        const size_t row = bh * D.T_cap + start + t;
        const int Rh = ((R / 16 + 1) / 2) * 16;
        const int cb0 = grp_a ? 0 : Rh, cb1 = grp_a ? Rh : R;
        // amax of the bf16 magnitudes, as a packed 16-bit unsigned max of their
        // bit patterns (the order of non-negative bf16 values)
        uint32_t am2 = 0u;
#pragma unroll 1
        for (int c0 = cb0; c0 < cb1; c0 += 32) {
          float v[2][16];
#pragma unroll
          for (int q = 0; q < 2; ++q)
            if (c0 + 16 * q < cb1) tc5::tmem_ld16(d1 + c0 + 16 * q, v[q]);
          tc5::tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 2; ++q)
            if (c0 + 16 * q < cb1)
#pragma unroll
              for (int k = 0; k < 16; k += 2) {
                const float m0 = mug ? cmu[(c0 + 16 * q + k) & (kD - 1)] : 0.f;
                const float m1 = mug ? cmu[(c0 + 16 * q + k + 1) & (kD - 1)] : 0.f;
                const uint32_t pr = cvt_bf16x2(v[q][k] - m0, v[q][k + 1] - m1);   // bf16 pair
                am2 = __vmaxu2(am2, pr & 0x7fff7fffu);
              }
        }
        uint32_t* amx = reinterpret_cast<uint32_t*>(sm + Lo.amx) + (i & 1) * 2 * kTile;
        amx[(grp_a ? 0 : kTile) + m] = max(am2 & 0xffffu, am2 >> 16);
        tc5::named_bar_sync(1, kEpi);   // both halves of every row's amax in
        const float amax = __uint_as_float(max(amx[m], amx[kTile + m]) << 16);
        const float qs = quant_scale(amax, CB);
        const float qinv = qs > 0.f ? 1.f / qs : 0.f;
        if (grp_a && valid) scales[row] = qs;
#pragma unroll 1
        for (int c0 = cb0; c0 < cb1; c0 += 32) {
          float v[2][16];
#pragma unroll
          for (int q = 0; q < 2; ++q)
            if (c0 + 16 * q < cb1) tc5::tmem_ld16(d1 + c0 + 16 * q, v[q]);
          tc5::tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            if (!valid || c0 + 16 * q >= cb1) continue;
            uint32_t bw[8];
#pragma unroll
            for (int k = 0; k < 16; k += 2) {
              const float m0 = mug ? cmu[(c0 + 16 * q + k) & (kD - 1)] : 0.f;
              const float m1 = mug ? cmu[(c0 + 16 * q + k + 1) & (kD - 1)] : 0.f;
              bw[k >> 1] = cvt_bf16x2(v[q][k] - m0, v[q][k + 1] - m1);
            }
            uint32_t cw[4];   // 16 codes: 16 bytes (8-bit) or 8 (4-bit)
            quant_pack16_bf(bw, qs, qinv, CB, cw);
            const int c = c0 + 16 * q;
            if (CB == 8)
              *reinterpret_cast<uint4*>(coef + row * R + c) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            else
              *reinterpret_cast<uint2*>(coef + row * (R / 2) + c / 2) = make_uint2(cw[0], cw[1]);
          }
        }
      }
      if (CB == 16 && grp_a) {
        // bf16 rows: group A stores the coefficients (c = U^T x - U^T mu with a
        // key mean), 64 columns per batch of TMEM loads (one wait per batch)
        const size_t row = bh * D.T_cap + start + t;
#pragma unroll 1
        for (int c0 = 0; c0 < R; c0 += 64) {
          float v[4][16];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (c0 + 16 * q < R) tc5::tmem_ld16(d1 + c0 + 16 * q, v[q]);
          tc5::tmem_wait_ld();
          if (mug) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int k = 0; k < 16; ++k) v[q][k] -= cmu[(c0 + 16 * q + k) & (kD - 1)];
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (!valid || c0 + 16 * q >= R) continue;
            const float* w = v[q];
            lrkv_bf16* crow = reinterpret_cast<lrkv_bf16*>(coef) + row * R;
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) pk[e] = pack_bf16(w[2 * e], w[2 * e + 1]);
            if (coef32) {   // 16 columns = 32 bytes in one store (rows are 32-byte multiples)
              asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                           ::"l"(crow + c0 + 16 * q), "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3]),
                           "r"(pk[4]), "r"(pk[5]), "r"(pk[6]), "r"(pk[7])
                           : "memory");
            } else {
              *reinterpret_cast<uint4*>(crow + c0 + 16 * q) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              *reinterpret_cast<uint4*>(crow + c0 + 16 * q + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
          }
        }
      }
      {  // squared residual of this group's 64 columns
        float v[4][16];
#pragma unroll
        for (int q = 0; q < 4; ++q) tc5::tmem_ld16(d2 + (grp_a ? 0 : 64) + 16 * q, v[q]);
        tc5::tmem_wait_ld();
        if (mug) {   // residual P (x - mu) = P x - P mu
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int k = 0; k < 16; ++k) v[q][k] -= rmu[(grp_a ? 0 : 64) + 16 * q + k];
        }
        float r0 = 0.f, r1 = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int k = 0; k < 16; k += 2) r0 = fmaf(v[q][k], v[q][k], r0), r1 = fmaf(v[q][k + 1], v[q][k + 1], r1);
        rs = r0 + r1;
      }
      if (!grp_a) {
        // squared input: row m of both 64-column boxes, every 16-byte chunk
        // (the swizzle only permutes chunks within the row)
        const unsigned char* xr = sm + Lo.x + s * kStageBytes + m * 128;
        float x0 = 0.f, x1 = 0.f;
#pragma unroll
        for (int box = 0; box < 2; ++box) {
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const uint4 w = *reinterpret_cast<const uint4*>(xr + box * kBoxBytes + (((cc + m) & 7) << 4));
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float a = bf_lo(ws[q]), c = bf_hi(ws[q]);
              x0 = fmaf(a, a, x0);
              x1 = fmaf(c, c, x1);
            }
          }
        }
        xs = x0 + x1;
        part[(i & 1) * kTile + m] = make_float2(rs, xs);
      }
      tc5::fence_before_sync();
      mbar_arrive(&tfree[buf]);
      mbar_arrive(&empty[s]);
      tc5::named_bar_sync(1, kEpi);   // group B's sums are in
      if (grp_a && valid) {
        const float2 pb = part[(i & 1) * kTile + m];
        const float rsum = rs + pb.x;
        errs[bh * D.T_cap + t] = pb.y > 0.f ? sqrtf(rsum / pb.y) : 0.f;
      }
      ++i;
    }
  }
  if (*abort_flag && tid == 0) atomicOr(p.C.dev_status, LRKV_DEV_WAIT_TIMEOUT);
  tc5::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc5::fence_after_sync();
    tc5::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- routing -------------------------------------------------------------------------

struct RouteParams {
  lrkv_dims D;
  lrkv_cache C;
  const lrkv_bf16* k_new;
  const lrkv_bf16* v_new;
  int t_new;
  const int32_t* t_new_b;
  float tau;
  float* err_out;          // nullable [B][Hkv][t_new]
  const float* errs;       // [2][B][Hkv][T_cap]
  int32_t* tile_cnt;       // [B][Hkv][n_tiles]
  uint32_t* tile_bits;     // [B][Hkv][n_tiles][4]
  int n_tiles;
  int tiles_per_cta;       // route_scatter_kernel: consecutive tiles per CTA, 1..kMaxScatterTiles
  int32_t* bh_tickets;     // [B][Hkv], zero between calls
  int32_t* ticket;         // [1], zero between calls
};

__device__ __forceinline__ int route_eff(const RouteParams& p, int b, int* start, uint32_t* st) {
  const int n = new_tokens(p.t_new_b, b, p.t_new, st);
  const int s0 = min(max(p.C.seq_len[b], 0), p.D.T_cap);
  int ne = p.D.T_cap - s0;
  if (ne > n) ne = n;
  if (ne < 0) ne = 0;
  *start = s0;
  return ne;
}

constexpr int kMaxScatterTiles = 8;

// grid (tiles_per_b, Hkv, B), 128 threads
__global__ void __launch_bounds__(128) route_count_kernel(RouteParams p) {
  // launched as a dependent of the projection: nothing is read before it is done
  griddep_wait();
  griddep_launch_dependents();
  const lrkv_dims& D = p.D;
  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __shared__ int s_cnt[4];
  uint32_t st = 0;
  int start;
  const int ne = route_eff(p, b, &start, &st);
  const size_t bh = (size_t)b * D.Hkv + h;
  const int t = tile * 128 + tid;
  const bool valid = t < ne;
  bool routed = false;
  if (valid) {
    const size_t i = bh * D.T_cap + t;
    const float e = fmaxf(p.errs[i], p.errs[(size_t)D.B * D.Hkv * D.T_cap + i]);
    routed = e > p.tau;
    if (p.err_out) p.err_out[bh * p.t_new + t] = e;
  }
  const uint32_t bits = __ballot_sync(0xffffffffu, routed);
  if (lane == 0) {
    p.tile_bits[(bh * p.n_tiles + tile) * 4 + warp] = bits;
    s_cnt[warp] = __popc(bits);
  }
  __syncthreads();
  if (tid == 0) p.tile_cnt[bh * p.n_tiles + tile] = (s_cnt[0] + s_cnt[1]) + (s_cnt[2] + s_cnt[3]);
}

// grid (ceil(tiles_per_b / tiles_per_cta), Hkv, B), 128 threads: tiles
// [x * tiles_per_cta, (x + 1) * tiles_per_cta) of one (b, kv head) per CTA
__global__ void __launch_bounds__(128) route_scatter_kernel(RouteParams p) {
  griddep_wait();   // a dependent of the count pass
  const lrkv_dims& D = p.D;
  const int h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __shared__ int s_red[4];
  __shared__ uint32_t s_bits[kMaxScatterTiles][4];
  __shared__ int2 s_rows[kMaxScatterTiles * 128];   // kept rows in list order: (slot, token)
  __shared__ bool s_last_bh, s_last;
  uint32_t st = 0;
  int start;
  const int ne = route_eff(p, b, &start, &st);
  const size_t bh = (size_t)b * D.Hkv + h;
  const int32_t* cnt = p.tile_cnt + bh * p.n_tiles;
  const int old = min(max(p.C.full_cnt[bh], 0), D.F_cap);
  const int tile_a = blockIdx.x * p.tiles_per_cta;
  const int n_tl = max(0, min(p.tiles_per_cta, (ne + 127) / 128 - tile_a));   // tiles with new tokens
  bool overflow = false;
  if (n_tl > 0) {
    // routed tokens of the earlier tiles of this (b, kv head)
    int before = 0;
    for (int i = tid; i < tile_a; i += 128) before += cnt[i];
    before = (int)warp_sum((float)before);   // counts < 2^24: exact in fp32
    if (lane == 0) s_red[warp] = before;
    if (tid < 4 * n_tl) s_bits[tid >> 2][tid & 3] = p.tile_bits[(bh * p.n_tiles + tile_a + (tid >> 2)) * 4 + (tid & 3)];
    __syncthreads();
    const int base = old + (s_red[0] + s_red[1]) + (s_red[2] + s_red[3]);   // this CTA's first slot
    int off = 0;   // routed tokens of this CTA's earlier tiles
    for (int j = 0; j < n_tl; ++j) {
      const int t0 = (tile_a + j) * 128;
      const uint32_t wbits = s_bits[j][warp];
      int wbefore = 0;
      for (int w = 0; w < warp; ++w) wbefore += __popc(s_bits[j][w]);
      const int t = t0 + tid;
      const bool valid = t < ne;
      const bool routed = (wbits >> lane) & 1u;
      const int idx = off + wbefore + __popc(wbits & ((1u << lane) - 1u));   // slot - base
      const int slot = base + idx;
      const bool keep = routed && slot < D.F_cap;
      overflow |= routed && !keep;
      if (keep) {
        p.C.full_idx[bh * D.F_cap + slot] = start + t;
        s_rows[idx] = make_int2(slot, t);
      }
      // mask words: this warp's 32 positions span at most two words
      const uint32_t keep_b = __ballot_sync(0xffffffffu, keep);
      const uint32_t valid_b = __ballot_sync(0xffffffffu, valid);
      if (lane == 0 && valid_b) {
        uint32_t* mrow = p.C.route_mask + bh * (D.T_cap / 32);
        const int p0 = start + t0 + warp * 32;
        const int w0 = p0 >> 5, sh = p0 & 31;
        const uint32_t r0 = valid_b << sh, k0 = keep_b << sh;
        if (r0) {
          if (r0 == 0xffffffffu) mrow[w0] = k0;
          else {
            atomicAnd(&mrow[w0], ~r0);
            if (k0) atomicOr(&mrow[w0], k0);
          }
        }
        if (sh) {
          const uint32_t r1 = valid_b >> (32 - sh), k1 = keep_b >> (32 - sh);
          if (r1) {
            atomicAnd(&mrow[w0 + 1], ~r1);
            if (k1) atomicOr(&mrow[w0 + 1], k1);
          }
        }
      }
      off += (__popc(s_bits[j][0]) + __popc(s_bits[j][1])) + (__popc(s_bits[j][2]) + __popc(s_bits[j][3]));
    }
    __syncthreads();   // the kept rows are listed
    // the kept rows are list entries [0, n_keep): slots are consecutive from base
    const int n_keep = max(0, min(off, D.F_cap - base));
    // copy them (32 lanes x 8 bytes per row): warp w takes rows [c0, c0 + 8)
    // for c0 = 8w, 8w + 32, ..., every load of a batch issued before its first store
    constexpr int kBatch = 8;
    for (int c0 = warp * kBatch; c0 < n_keep; c0 += 4 * kBatch) {
      uint2 kr[kBatch], vr[kBatch];
#pragma unroll
      for (int q = 0; q < kBatch; ++q) {
        if (c0 + q < n_keep) {
          const size_t x = (((size_t)b * p.t_new + s_rows[c0 + q].y) * D.Hkv + h) * kD;
          kr[q] = reinterpret_cast<const uint2*>(p.k_new + x)[lane];
          vr[q] = reinterpret_cast<const uint2*>(p.v_new + x)[lane];
        }
      }
#pragma unroll
      for (int q = 0; q < kBatch; ++q) {
        if (c0 + q < n_keep) {
          const size_t y = (bh * D.F_cap + s_rows[c0 + q].x) * kD;
          reinterpret_cast<uint2*>(p.C.full_k + y)[lane] = kr[q];
          reinterpret_cast<uint2*>(p.C.full_v + y)[lane] = vr[q];
        }
      }
    }
  }
  if (__syncthreads_or(overflow)) st |= LRKV_DEV_FULL_OVERFLOW;
  if (blockIdx.x == 0 && h == 0) {
    uint32_t dummy = 0;
    const int n = new_tokens(p.t_new_b, b, p.t_new, &dummy);
    if (ne < n) st |= LRKV_DEV_SEQ_OVERFLOW;
  } else {
    st &= LRKV_DEV_FULL_OVERFLOW;   // per-sequence conditions: reported once
  }
  if (tid == 0 && st) atomicOr(p.C.dev_status, st);
  // the last CTA of this (b, kv head) sets its list length
  __syncthreads();
  if (tid == 0) s_last_bh = atom_add_acq_rel_gpu(&p.bh_tickets[bh], 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (s_last_bh) {
    int tot = 0;
    const int nt = (ne + 127) / 128;
    for (int i = tid; i < nt; i += 128) tot += cnt[i];
    tot = (int)warp_sum((float)tot);
    if (lane == 0) s_red[warp] = tot;
    __syncthreads();
    if (tid == 0) {
      const int total = (s_red[0] + s_red[1]) + (s_red[2] + s_red[3]);
      p.C.full_cnt[bh] = min(old + total, D.F_cap);
      p.bh_tickets[bh] = 0;
      s_last = atom_add_acq_rel_gpu(p.ticket, 1) == (int)(gridDim.y * gridDim.z) - 1;
    }
    __syncthreads();
    if (s_last) {   // every (b, kv head) done: all seq_len reads are behind us
      for (int bb = tid; bb < D.B; bb += 128) {
        uint32_t dummy = 0;
        const int nb = new_tokens(p.t_new_b, bb, p.t_new, &dummy);
        const int sb = min(max(p.C.seq_len[bb], 0), D.T_cap);
        int e2 = D.T_cap - sb;
        if (e2 > nb) e2 = nb;
        if (e2 < 0) e2 = 0;
        p.C.seq_len[bb] = sb + e2;
      }
      if (tid == 0) *p.ticket = 0;
    }
  }
}

}  // namespace ptc
}  // namespace lrkv
