// Tensor-core split kernel variants (FP8-E4M3 K/V, head_dim 128).
#include "split_tc.cuh"

namespace pda {

template <int NT>
static cudaError_t launch_nt(const SplitArgs& a, dim3 grid, cudaStream_t stream) {
  using C = TcCfg<NT>;
  auto kern = split_tc_kernel<NT>;
  static unsigned long long attr_set = 0;  // bit d: opt-in set on device d (< 64)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit == 0 || !(__atomic_load_n(&attr_set, __ATOMIC_ACQUIRE) & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&attr_set, bit, __ATOMIC_RELEASE);
  }
  kern<<<grid, C::THREADS, C::SMEM_ALLOC, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_split_tc(int nt, const SplitArgs& a, dim3 grid, cudaStream_t stream) {
  switch (nt) {
    case 16: return launch_nt<16>(a, grid, stream);
    case 32: return launch_nt<32>(a, grid, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace pda
