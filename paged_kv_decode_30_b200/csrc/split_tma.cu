// TMA-fed tensor-core split kernel: tensor maps and launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cstring>
#include <mutex>

#include "split_tma.cuh"

namespace pda {
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library does not link libcuda.
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A pool [num_pages * Hkv * P rows, 128 elements] read in boxes of
// (box_inner elements, box_rows rows) with the 128-byte swizzle.
bool make_pool_map(CUtensorMap* map, const void* base, long long rows, int elt, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {128, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(128 * elt)};
  const cuuint32_t box[2] = {(cuuint32_t)(elt == 2 ? 64 : 128), (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, elt == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KV, int NT, bool QN = false>
cudaError_t launch_cfg(const CUtensorMap& mk, const CUtensorMap& mv, const SplitArgs& a,
                       int grid, cudaStream_t stream, bool pdl) {
  using C = TmaCfg<KV, NT, QN>;
  auto kern = split_tma_kernel<KV, NT, QN>;
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
  // prologue: block 0 (counters, queue order), FP8 one block per Q image
  const long long q_blocks = KV == 1 ? (long long)a.B * a.Hkv * a.row_tiles : 0;
  if (q_blocks >= INT_MAX) return cudaErrorInvalidValue;
  split_tma_prologue<KV, NT, QN><<<dim3((unsigned)(1 + q_blocks)), 256, 0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_ALLOC;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, mk, mv, a);
}

}  // namespace

cudaError_t launch_split_tma(int kv, int nt, bool native_qk, const void* k_pages,
                             const void* v_pages, const SplitArgs& a, int grid,
                             cudaStream_t stream, bool pdl) {
  const long long rows = (long long)a.num_pages * a.Hkv * a.page_size;
  const int elt = kv == 0 ? 2 : 1;
  const int box_rows = a.page_size < 128 ? a.page_size : 128;
  alignas(64) CUtensorMap mk, mv;
  if (kv == 2) {  // NVFP4 tiles come by bulk copies: the maps are not read
    std::memset(&mk, 0, sizeof(mk));
    std::memset(&mv, 0, sizeof(mv));
    switch (nt) {
      case 4: return launch_cfg<2, 4>(mk, mv, a, grid, stream, pdl);
      case 8: return launch_cfg<2, 8>(mk, mv, a, grid, stream, pdl);
      default: return cudaErrorNotSupported;
    }
  }
  if (!make_pool_map(&mk, k_pages, rows, elt, box_rows) ||
      !make_pool_map(&mv, v_pages, rows, elt, box_rows))
    return cudaErrorInvalidValue;
  if (kv == 0) {
    switch (nt) {
      case 4: return launch_cfg<0, 4>(mk, mv, a, grid, stream, pdl);
      case 8: return launch_cfg<0, 8>(mk, mv, a, grid, stream, pdl);
      default: return cudaErrorNotSupported;
    }
  }
  if (native_qk) {
    switch (nt) {
      case 16: return launch_cfg<1, 16, true>(mk, mv, a, grid, stream, pdl);
      case 32: return launch_cfg<1, 32, true>(mk, mv, a, grid, stream, pdl);
      default: return cudaErrorNotSupported;
    }
  }
  switch (nt) {
    case 16: return launch_cfg<1, 16>(mk, mv, a, grid, stream, pdl);
    case 32: return launch_cfg<1, 32>(mk, mv, a, grid, stream, pdl);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace pda
