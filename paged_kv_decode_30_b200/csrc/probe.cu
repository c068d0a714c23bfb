// Read-only HBM streaming probe: the read-bandwidth denominator that the
// benchmark measures in the same run as the attention kernels (decode
// attention only reads K/V, so a copy kernel's read+write figure is not the
// only fair ceiling).
//
// Every byte of the buffer is read once with 128-bit non-allocating loads,
// four loads in flight per thread per iteration, grid = 4 CTAs of 512
// threads per SM; the XOR of the words goes to *sink so no load is dead.

#include <cuda_runtime.h>
#include <stdint.h>

#include "paged_decode_attn.h"

namespace pda {

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(512) hbm_read_probe_kernel(const uint4* __restrict__ p,
                                                             long long n,
                                                             unsigned long long* sink) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t acc = 0;
  for (; i + 3 * stride < n; i += 4 * stride) {
    const uint4 a = ld_stream(p + i);
    const uint4 b = ld_stream(p + i + stride);
    const uint4 c = ld_stream(p + i + 2 * stride);
    const uint4 d = ld_stream(p + i + 3 * stride);
    acc ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w;
    acc ^= c.x ^ c.y ^ c.z ^ c.w ^ d.x ^ d.y ^ d.z ^ d.w;
  }
  for (; i < n; i += stride) {
    const uint4 a = ld_stream(p + i);
    acc ^= a.x ^ a.y ^ a.z ^ a.w;
  }
  acc = __reduce_xor_sync(0xFFFFFFFFu, acc);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, (unsigned long long)acc);
}

}  // namespace pda

extern "C" {

pda_status pda_hbm_read_probe(const void* buf, size_t bytes, uint64_t* sink,
                              pda_stream_t stream_) {
  if (bytes == 0) return PDA_OK;
  if (!buf || !sink) return PDA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(buf) & 15u) != 0 || (bytes & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(sink) & 7u) != 0)
    return PDA_ERR_MISALIGNED;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return PDA_ERR_CUDA;
  const long long n = (long long)(bytes / 16);
  long long grid = (long long)sms * 4;
  const long long need = (n + 511) / 512;
  if (grid > need) grid = need;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  pda::hbm_read_probe_kernel<<<(unsigned)grid, 512, 0, stream>>>(
      static_cast<const uint4*>(buf), n, reinterpret_cast<unsigned long long*>(sink));
  return cudaGetLastError() == cudaSuccess ? PDA_OK : PDA_ERR_CUDA;
}

}  // extern "C"
