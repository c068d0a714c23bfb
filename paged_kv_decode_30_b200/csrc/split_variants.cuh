// Instantiation and launch of the FMA split kernel variants for one head_dim.
// Included by split_d64.cu / split_d128.cu / split_d256.cu, each compiled on
// its own so the variants build in parallel.
#pragma once

#include "split_fma.cuh"

namespace pda {

// Warps per CTA and ring depth of each warp (one CTA per SM). The kernel is
// bound by issue latency, not by bytes in flight: 12 warps with a 2-deep
// ring (3 warps per scheduler, 168 registers) beat 8 warps with a 3-deep
// ring by 13% on the headline shape. Variants with 8 packed rows need more
// than 168 registers, so they keep 8 warps x 3 stages.
template <int MT>
struct FmaShape {
  static constexpr int NW = MT <= 4 ? 12 : 8;
  static constexpr int STAGES = MT <= 4 ? 2 : 3;
};
inline int fma_warps(int mt) { return mt <= 4 ? 12 : 8; }

template <int D, int KV, int MT, int TW>
cudaError_t launch_variant(const SplitArgs& a, dim3 grid, cudaStream_t stream) {
  constexpr int NW = FmaShape<MT>::NW;
  constexpr int ST = FmaShape<MT>::STAGES;
  using C = FmaCfg<D, KV, MT, TW, NW, ST>;
  auto kern = split_fma_kernel<D, KV, MT, TW, NW, ST>;
  // The shared-memory opt-in is a per-device function attribute: set it the
  // first time this variant launches on each device.
  static unsigned long long attr_set = 0;  // bit d: set on device d (< 64)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit == 0 || !(__atomic_load_n(&attr_set, __ATOMIC_ACQUIRE) & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&attr_set, bit, __ATOMIC_RELEASE);
  }
  kern<<<grid, NW * 32, C::SMEM, stream>>>(a);
  return cudaGetLastError();
}

template <int D, int KV, int MT>
cudaError_t launch_tw(int tw, const SplitArgs& a, dim3 grid, cudaStream_t s) {
  constexpr int TW_FULL = 8 * (32 / (D / 8));  // 8 tokens per lane group
  if (tw == TW_FULL) return launch_variant<D, KV, MT, TW_FULL>(a, grid, s);
  if constexpr (TW_FULL / 2 >= 32 / (D / 8) && TW_FULL / 2 >= 8) {
    if (tw == TW_FULL / 2) return launch_variant<D, KV, MT, TW_FULL / 2>(a, grid, s);
  }
  if constexpr (TW_FULL / 4 >= 32 / (D / 8) && TW_FULL / 4 >= 8) {
    if (tw == TW_FULL / 4) return launch_variant<D, KV, MT, TW_FULL / 4>(a, grid, s);
  }
  return cudaErrorNotSupported;
}

template <int D>
cudaError_t launch_for_dim(int kv, int mt, int tw, const SplitArgs& a,
                           dim3 grid, cudaStream_t s) {
#define PDA_MT_CASES(KV)                                      \
  switch (mt) {                                               \
    case 1: return launch_tw<D, KV, 1>(tw, a, grid, s);       \
    case 2: return launch_tw<D, KV, 2>(tw, a, grid, s);       \
    case 4: return launch_tw<D, KV, 4>(tw, a, grid, s);       \
    case 8: return launch_tw<D, KV, 8>(tw, a, grid, s);       \
    default: return cudaErrorNotSupported;                    \
  }
  if (kv == 0) {
    PDA_MT_CASES(0)
  } else if (kv == 1) {
    PDA_MT_CASES(1)
  } else {
    PDA_MT_CASES(2)
  }
#undef PDA_MT_CASES
}

cudaError_t launch_split_d64(int kv, int mt, int tw, const SplitArgs& a, dim3 g, cudaStream_t s);
cudaError_t launch_split_d128(int kv, int mt, int tw, const SplitArgs& a, dim3 g, cudaStream_t s);
cudaError_t launch_split_d256(int kv, int mt, int tw, const SplitArgs& a, dim3 g, cudaStream_t s);

}  // namespace pda
