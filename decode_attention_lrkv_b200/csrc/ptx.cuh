// Thin wrappers over the sm_90+/sm_100 PTX this library uses: mbarriers and
// bulk (TMA) global->shared copies.  Every wait is bounded by the caller.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace lrkv {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Make mbarrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) writes to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Order generic-proxy global memory accesses (this thread's, and those it
// has observed through acquire) before its later async-proxy (bulk copy) reads.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Raise the barrier's expected transaction bytes without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Programmatic dependent launch: wait until the preceding kernel of the stream
// has completed and its memory is visible (a no-op without the launch
// attribute); let the next kernel of the stream start its prologue.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// One plain arrival.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One arrival that also raises the barrier's expected transaction bytes.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete, at most max_iter
// polls (each poll may suspend briefly in hardware).  Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint32_t max_iter) {
  for (uint32_t i = 0; i < max_iter; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (i > 64) __nanosleep(64);
  }
  return false;
}

// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) from
// global to this CTA's shared memory; completion is signalled on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

}  // namespace lrkv

namespace lrkv {

// 16-byte asynchronous global->shared copy (L2 only), grouped per thread.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// 16-byte async copy that reads `src_bytes` (16 or 0) and zero-fills the rest.
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ldmatrix: four 8x8 b16 matrices; lanes 8m..8m+7 give the row addresses of matrix m.
__device__ __forceinline__ void ldsm_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                        const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(row_addr)));
}
__device__ __forceinline__ void ldsm_x2(uint32_t& r0, uint32_t& r1, const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(smem_u32(row_addr)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                          const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(row_addr)));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// The same shape with f16 operands: D = A(16x16 f16, row) * B(16x8 f16, col) + D.
__device__ __forceinline__ void mma_16816_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// D = A(16x8 bf16, row) * B(8x8 bf16, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma_1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

// Ticket increment with acquire-release semantics at GPU scope.  Issued by one
// thread after a CTA barrier, it releases every write the CTA made before the
// barrier and, for the thread that sees the final count, acquires the others'.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int* addr, int v) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
  return old;
}

// Fire-and-forget bitwise OR / AND on a global word (no value returned, so the
// thread never waits for it).
__device__ __forceinline__ void red_or_u32(uint32_t* addr, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.or.b32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void red_and_u32(uint32_t* addr, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.and.b32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}

// Release-only add: later operations of the thread need not wait for it; a
// thread that acts on the returned count issues fence_acq_rel_gpu() first.
__device__ __forceinline__ int atom_add_release_gpu(int* addr, int v) {
  int old;
  asm volatile("atom.add.release.gpu.s32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Two floats -> bf16x2 (round to nearest even), the first in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return l | (h << 16);
}
// Two floats -> bf16x2 in one conversion (round to nearest even), `lo` in the low half.
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
// The bf16x2 high parts (lo_part false) or low parts (true) of the pair (a, b):
// x = hi + lo with hi = bf16(x), lo = bf16(x - hi); a in the low half.
__device__ __forceinline__ uint32_t split_bf16x2(float a, float b, bool lo_part) {
  const uint32_t h = cvt_bf16x2(a, b);
  const uint32_t l = cvt_bf16x2(a - __uint_as_float(h << 16), b - __uint_as_float(h & 0xffff0000u));
  return lo_part ? l : h;
}
// x = hi + lo with hi = bf16(x), lo = bf16(x - hi): the part selected by `lo_part`.
__device__ __forceinline__ float bf16_part(float x, bool lo_part) {
  const float h = __bfloat162float(__float2bfloat16_rn(x));
  return lo_part ? x - h : h;
}
// The f16 high part of x (round to nearest even), or the low part x - high,
// each as an f16 bit pattern.
__device__ __forceinline__ uint32_t f16_part_bits(float x, bool lo_part) {
  const __half h = __float2half_rn(x);
  return __half_as_ushort(lo_part ? __float2half_rn(x - __half2float(h)) : h);
}

}  // namespace lrkv

namespace lrkv {

// Transpose an 8x8 b16 matrix held in MMA fragment layout across the warp
// (thread holds row lane/4, columns 2*(lane%4) and +1, packed).
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

}  // namespace lrkv

namespace lrkv {

// int8 codes -> bf16, exactly.  A byte b read as unsigned after flipping its
// sign bit is b + 128; placed in the low mantissa bits of 2^23 that fp32 is
// 2^23 + b + 128, so subtracting 2^23 + 128 gives b as fp32.  An integer of
// magnitude <= 128 has its bf16 value in the upper half of its fp32 bits.
__device__ __forceinline__ float s8_byte_f32(uint32_t flipped, uint32_t sel) {
  return __uint_as_float(__byte_perm(flipped, 0x4B000000u, sel)) - 8388736.f;
}
__device__ __forceinline__ uint32_t bf16x2_upper(float lo, float hi) {
  return __byte_perm(__float_as_uint(lo), __float_as_uint(hi), 0x7632);
}
// Four int8 codes in w: bf16x2 of bytes (0, 1) and of bytes (2, 3).
__device__ __forceinline__ void s8x4_pairs(uint32_t w, uint32_t& b01, uint32_t& b23) {
  const uint32_t u = w ^ 0x80808080u;
  b01 = bf16x2_upper(s8_byte_f32(u, 0x7440), s8_byte_f32(u, 0x7441));
  b23 = bf16x2_upper(s8_byte_f32(u, 0x7442), s8_byte_f32(u, 0x7443));
}
// Four int8 codes in w: f16x2 of bytes (0, 1) and of bytes (2, 3), exactly.
// With the sign bit flipped a byte is u = b + 128 in [0, 255]; the f16 with
// high byte 0x64 and low byte u is 1024 + u (f16 spacing is 1 on [1024,
// 2048)), and subtracting 1152 leaves b.
__device__ __forceinline__ void s8x4_f16pairs(uint32_t w, uint32_t& h01, uint32_t& h23) {
  const uint32_t u = w ^ 0x80808080u;
  h01 = __byte_perm(u, 0x64646464u, 0x4140);
  h23 = __byte_perm(u, 0x64646464u, 0x4342);
  const uint32_t k1 = 0x3C003C00u, km = 0xE480E480u;   // f16x2 (1, 1), (-1152, -1152)
  asm("fma.rn.f16x2 %0, %0, %1, %2;" : "+r"(h01) : "r"(k1), "r"(km));
  asm("fma.rn.f16x2 %0, %0, %1, %2;" : "+r"(h23) : "r"(k1), "r"(km));
}
// Four int8 codes in w: f16x2 of bytes (0, 2) and of bytes (1, 3), exactly.
__device__ __forceinline__ void s8x4_f16evenodd(uint32_t w, uint32_t& h02, uint32_t& h13) {
  const uint32_t u = w ^ 0x80808080u;
  h02 = __byte_perm(u, 0x64646464u, 0x4240);
  h13 = __byte_perm(u, 0x64646464u, 0x4341);
  const uint32_t k1 = 0x3C003C00u, km = 0xE480E480u;   // f16x2 (1, 1), (-1152, -1152)
  asm("fma.rn.f16x2 %0, %0, %1, %2;" : "+r"(h02) : "r"(k1), "r"(km));
  asm("fma.rn.f16x2 %0, %0, %1, %2;" : "+r"(h13) : "r"(k1), "r"(km));
}
// Two floats -> f16x2 in one conversion (round to nearest even), `lo` in the low half.
__device__ __forceinline__ uint32_t cvt_f16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
// Four int8 codes in w: bf16x2 of bytes (0, 2) and of bytes (1, 3).
__device__ __forceinline__ void s8x4_evenodd(uint32_t w, uint32_t& b02, uint32_t& b13) {
  const uint32_t u = w ^ 0x80808080u;
  b02 = bf16x2_upper(s8_byte_f32(u, 0x7440), s8_byte_f32(u, 0x7442));
  b13 = bf16x2_upper(s8_byte_f32(u, 0x7441), s8_byte_f32(u, 0x7443));
}

}  // namespace lrkv
