// tcgen05 / UMMA building blocks for the tensor-core split kernel: shared-
// memory matrix and instruction descriptors, MMA issue and commit, TMEM
// loads and fences, and the warp/named-barrier helpers the kernel's roles
// synchronise with. All PTX here is hand-written inline assembly for sm_100a.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "pda_device.cuh"

namespace pda {

// Shared-memory matrix descriptor: start address, leading- and stride-
// dimension byte offsets, and the swizzle mode of the canonical layout.
// Swizzled atoms are 8 rows of 128 (SW128), 64 (SW64) or 32 (SW32) bytes
// whose 16-byte chunks are XOR-permuted by row, which keeps the tensor
// core's operand reads free of bank conflicts. Atom bases are aligned to
// 8 rows x row bytes, so the base-offset field stays 0.
constexpr uint32_t kSw128 = 2, kSw64 = 4, kSw32 = 6;
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 16 consecutive fp32 TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = __uint_as_float(r[k]);
}

// 8 consecutive fp32 TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = __uint_as_float(r[k]);
}

// Store 16 (or 8) fp32 values to consecutive TMEM columns of this thread's
// lane and wait for the stores to complete.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
      : "memory");
}

__device__ __forceinline__ float redux_max(float x) {
  float y;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void named_bar(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Named barrier over `threads` threads that also returns the OR of `v` over
// them, so every thread takes the same branch afterwards.
__device__ __forceinline__ bool named_bar_or(int id, int threads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

// Lazy max test of eight scores fused with the group barrier: returns, in
// every thread, the OR over the `threads` threads of (any s[k] > t[k]) or
// `failed`. The compares chain through one predicate (setp with .or).
__device__ __forceinline__ bool named_bar_any_gt8(int id, int threads, const float* s,
                                                  float4 t0, float4 t1, bool failed) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "setp.gt.or.f32 p, %4, %12, p;\n\t"
      "setp.gt.or.f32 p, %5, %13, p;\n\t"
      "setp.gt.or.f32 p, %6, %14, p;\n\t"
      "setp.gt.or.f32 p, %7, %15, p;\n\t"
      "setp.gt.or.f32 p, %8, %16, p;\n\t"
      "setp.gt.or.f32 p, %9, %17, p;\n\t"
      "setp.gt.or.f32 p, %10, %18, p;\n\t"
      "setp.gt.or.f32 p, %11, %19, p;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)failed), "r"(id), "r"(threads), "f"(s[0]), "f"(s[1]), "f"(s[2]),
        "f"(s[3]), "f"(s[4]), "f"(s[5]), "f"(s[6]), "f"(s[7]), "f"(t0.x), "f"(t0.y),
        "f"(t0.z), "f"(t0.w), "f"(t1.x), "f"(t1.y), "f"(t1.z), "f"(t1.w)
      : "memory");
  return r != 0;
}

// Named barrier over `threads` threads that also returns the AND of `v` over
// them, so every thread takes the same branch afterwards.
__device__ __forceinline__ bool named_bar_and(int id, int threads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

// One named barrier returning the OR of `want` over the threads; `*ok_out`
// gets the AND of `ok`. (Two barrier reductions back to back on the same id.)
__device__ __forceinline__ bool named_bar_or_and(int id, int threads, bool want, bool ok,
                                                 bool* ok_out) {
  uint32_t r_or, r_and;
  asm volatile(
      "{\n\t.reg .pred p, q, x, y;\n\tsetp.ne.u32 p, %2, 0;\n\tsetp.ne.u32 q, %3, 0;\n\t"
      "bar.red.or.pred x, %4, %5, p;\n\tbar.red.and.pred y, %4, %5, q;\n\t"
      "selp.u32 %0, 1, 0, x;\n\tselp.u32 %1, 1, 0, y;\n\t}"
      : "=r"(r_or), "=r"(r_and)
      : "r"((uint32_t)want), "r"((uint32_t)ok), "r"(id), "r"(threads)
      : "memory");
  *ok_out = r_and != 0;
  return r_or != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

}  // namespace pda
