// Device helpers shared by the paged decode kernels (sm_100a).
//
// Bulk copies: every (page, kv head) block of the HND pool is contiguous, so a
// K or V tile of `TW` tokens is one untiled cp.async.bulk from global to
// shared memory that completes on an mbarrier with a transaction count.
// All waits are bounded: on expiry the kernel records PDA_ERR_TIMEOUT in the
// device error word and gives up instead of hanging the GPU.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace pda {

constexpr int kErrUnsupported = 2;  // == PDA_ERR_UNSUPPORTED
constexpr int kErrBadPage = 6;   // == PDA_ERR_BAD_PAGE
constexpr int kErrTimeout = 7;   // == PDA_ERR_TIMEOUT

// About two seconds at the B200's top clock.
constexpr long long kWaitTimeoutCycles = 4000000000LL;

// Record the first error in the device error word (read and cleared by
// pda_last_device_error). Later errors keep the first code.
__device__ __forceinline__ void record_error_at(int* err, int code) {
  atomicCAS(err, 0, code);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(count)
               : "memory");
}

// Make mbarrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy accesses (a bulk copy refilling a buffer just read).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar,
                                                      uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
          smem_addr(bar)),
      "r"(bytes)
      : "memory");
}

// Adds `bytes` to the transaction count of the current phase, no arrival.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of `bar`. Returns false after about
// `limit` cycles and records PDA_ERR_TIMEOUT in *err.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          int* err,
                                          long long limit = kWaitTimeoutCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long start = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && clock64() - start > limit) {
      record_error_at(err, kErrTimeout);
      return false;
    }
  }
}

// Global -> shared bulk copy completing on `bar`. dst, src 16-byte aligned,
// bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src,
                                         uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Programmatic dependent launch controls.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_primary() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// 8 bf16 packed in a uint4 -> 8 floats (exact: bf16 is the top half of fp32).
__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[2 * k] = __uint_as_float(w[k] << 16);
    f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}

// 8 e4m3 codes packed in a uint2 -> 8 floats (exact: e4m3 -> f16 -> f32).
__device__ __forceinline__ void e4m3x8_to_f32(const uint2& u, float (&f)[8]) {
  const uint32_t w[2] = {u.x, u.y};
#pragma unroll
  for (int k = 0; k < 2; ++k) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __nv_fp8x2_storage_t pair =
          static_cast<__nv_fp8x2_storage_t>((w[k] >> (16 * h)) & 0xFFFFu);
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
      const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&hr));
      f[4 * k + 2 * h] = f2.x;
      f[4 * k + 2 * h + 1] = f2.y;
    }
  }
}

// 2^x with the SFU's approximate exp2 (one instruction; relative error about
// 2^-22, far inside the tolerances). ex2(-inf) = +0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 values in one 64-bit register pair, for the packed f32x2
// arithmetic of sm_100 (one issue slot, two FMAs).
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 f2_pack(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(f32x2 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 f2_fma(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 f2_mul(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 f2_add(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// One 32-bit word holding two bf16 (element 2j in the low half, 2j+1 in the
// high half) -> the fp32 pair (exact).
__device__ __forceinline__ f32x2 bf16x2_to_f2(uint32_t w) {
  return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// Two e4m3 codes (16 bits) -> the fp32 pair (exact: e4m3 -> f16 -> f32).
__device__ __forceinline__ f32x2 e4m3x2_to_f2(uint32_t h16) {
  const __half2_raw hr =
      __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(h16 & 0xFFFFu), __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
  return f2_pack(f.x, f.y);
}

// Two e2m1 codes (one byte, first element in the low nibble) -> the fp32
// pair (exact: e2m1 -> f16 -> f32).
__device__ __forceinline__ f32x2 e2m1x2_to_f2(uint32_t byte) {
  const __half2_raw hr =
      __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(byte & 0xFFu), __NV_E2M1);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
  return f2_pack(f.x, f.y);
}

// One e4m3 code -> float (exact).
__device__ __forceinline__ float e4m3_code_to_f32(uint32_t code) {
  const __half_raw h =
      __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code & 0xFFu), __NV_E4M3);
  return __half2float(*reinterpret_cast<const __half*>(&h));
}

}  // namespace pda
