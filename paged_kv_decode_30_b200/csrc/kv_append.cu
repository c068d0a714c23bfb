// Paged KV append: the KV-cache producer that runs before the decode call.
//
// Source: "sglang profiler skill, fuse-overlap catalog, Fused FP8 quantize +
// paged KV cache write row" (new K/V rows quantised to FP8 and written
// straight into their pages in one kernel) and its "fused BF16 to FP4 quant
// + paged KV write" row, "b12x 0.30.0, Kernel inventory, Attention table,
// Paged attention row" (FP8-E4M3 KV caches) and the same inventory's
// "BF16-to-FP4 TMA quantization" row (packed NVFP4 plus scale tiles).
//
// One warp per (sequence, new token, kv head): it finds the slot from the
// page table (position kv_lens[b] + t), loads the bf16 K and V rows (D/32
// elements per lane, one vector load each) and stores them as bf16 bits or
// as e4m3 codes of the fp32 quotient x / kv_scale (round to nearest even,
// saturated to +-448) with the hardware converter, or as NVFP4: per block of
// 16 elements (16 / (D/32) adjacent lanes) the lanes share max |x/kv_scale|
// by shuffles, the first lane of the block writes its e4m3 scale
// e4m3(max / 6), and every lane writes the e2m1 codes of (x/kv_scale)/scale,
// two per byte. The kernel is a plain
// stream of reads and writes: coalesced 16/8/4-byte accesses per lane, a
// grid of 4 CTAs of 256 threads per SM.

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "paged_decode_attn.h"
#include "pda_device.cuh"

namespace pda {

struct AppendArgs {
  const uint16_t* k_new;  // bf16 [B, T, Hkv, D]
  const uint16_t* v_new;
  const int32_t* page_table;
  const int32_t* kv_lens;
  uint8_t* k_pages;  // pool bytes [num_pages, Hkv, P, D] (NVFP4: D/2)
  uint8_t* v_pages;
  uint8_t* k_scales;  // NVFP4: e4m3 block scales [num_pages, Hkv, P, D/16]
  uint8_t* v_scales;
  int* err;
  int B, T, Hkv, log2_page, page_size, max_pages, num_pages;
  float kv_scale;
};

template <int E>
struct BitsOf;  // E bf16 values in one vector access
template <>
struct BitsOf<2> { using T = uint32_t; };
template <>
struct BitsOf<4> { using T = uint2; };
template <>
struct BitsOf<8> { using T = uint4; };

__device__ __forceinline__ uint32_t bf16x2_to_e4m3x2(uint32_t w, float scale) {
  const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xFFFF0000u);
  uint16_t r;
  // IEEE division (the quotient the quantised code is defined on), then RNE
  // with saturation; the first operand lands in the high byte.
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(__fdiv_rn(hi, scale)),
      "f"(__fdiv_rn(lo, scale)));
  return r;
}

// One e4m3 code of v (nearest even, saturating), in the low byte.
__device__ __forceinline__ uint32_t f32_to_e4m3(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.f), "f"(v));
  return r & 0xFFu;
}

// NVFP4 of one lane's E elements (bf16 words w, E/2 of them) of a block of
// 16 that LB = 16 / E adjacent lanes share: returns the E/2 code bytes
// (element 2k in the low nibble of byte k, byte k in bits 8k..8k+7) and sets
// *scale_code to the block's e4m3 scale.
template <int E>
__device__ __forceinline__ uint32_t nvfp4_lane(const uint32_t* w, float kv_scale,
                                               uint32_t* scale_code) {
  constexpr int LB = 16 / E;
  float q[E];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < E / 2; ++k) {
    q[2 * k] = __fdiv_rn(__uint_as_float(w[k] << 16), kv_scale);
    q[2 * k + 1] = __fdiv_rn(__uint_as_float(w[k] & 0xFFFF0000u), kv_scale);
    amax = fmaxf(amax, fmaxf(fabsf(q[2 * k]), fabsf(q[2 * k + 1])));
  }
#pragma unroll
  for (int o = 1; o < LB; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  const uint32_t sc = f32_to_e4m3(__fdiv_rn(amax, 6.f));
  *scale_code = sc;
  const float sd = e4m3_code_to_f32(sc);
  uint32_t codes = 0;
  if (sd > 0.f) {
#pragma unroll
    for (int k = 0; k < E / 2; ++k) {
      const __nv_fp4x2_storage_t b = __nv_cvt_float2_to_fp4x2(
          make_float2(__fdiv_rn(q[2 * k], sd), __fdiv_rn(q[2 * k + 1], sd)), __NV_E2M1,
          cudaRoundNearest);
      codes |= (uint32_t)b << (8 * k);
    }
  }
  return codes;
}

// KVK: 0 bf16, 1 e4m3, 2 NVFP4.
template <int D, int KVK>
__global__ void __launch_bounds__(256) kv_append_kernel(const AppendArgs a) {
  constexpr int E = D / 32;  // elements per lane
  using V = typename BitsOf<E>::T;
  const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const long long rows = (long long)a.B * a.T * a.Hkv;
  for (long long r = warp_global; r < rows; r += nwarps) {
    const int h = (int)(r % a.Hkv);
    const long long bt = r / a.Hkv;
    const int t = (int)(bt % a.T);
    const int b = (int)(bt / a.T);
    const int L = __ldg(a.kv_lens + b);
    const long long pos = (long long)L + t;
    if (L < 0 || pos >= (long long)a.max_pages * a.page_size) {
      if (lane == 0) record_error_at(a.err, kErrBadPage);
      continue;
    }
    const int page = __ldg(a.page_table + (long long)b * a.max_pages + (pos >> a.log2_page));
    if ((unsigned)page >= (unsigned)a.num_pages) {
      if (lane == 0) record_error_at(a.err, kErrBadPage);
      continue;
    }
    const long long src = r * D + lane * E;
    const long long slot = ((long long)page * a.Hkv + h) * a.page_size + (pos & (a.page_size - 1));
    const V kv = *reinterpret_cast<const V*>(a.k_new + src);
    const V vv = *reinterpret_cast<const V*>(a.v_new + src);
    if constexpr (KVK == 2) {
      constexpr int LB = 16 / E;  // lanes per block of 16
      uint32_t ksc, vsc;
      const uint32_t kc = nvfp4_lane<E>(reinterpret_cast<const uint32_t*>(&kv), a.kv_scale, &ksc);
      const uint32_t vc = nvfp4_lane<E>(reinterpret_cast<const uint32_t*>(&vv), a.kv_scale, &vsc);
      const long long cb = (slot * D + lane * E) / 2;  // first code byte of this lane
      if constexpr (E == 2) {
        a.k_pages[cb] = (uint8_t)kc;
        a.v_pages[cb] = (uint8_t)vc;
      } else if constexpr (E == 4) {
        *reinterpret_cast<uint16_t*>(a.k_pages + cb) = (uint16_t)kc;
        *reinterpret_cast<uint16_t*>(a.v_pages + cb) = (uint16_t)vc;
      } else {
        *reinterpret_cast<uint32_t*>(a.k_pages + cb) = kc;
        *reinterpret_cast<uint32_t*>(a.v_pages + cb) = vc;
      }
      if (lane % LB == 0) {
        a.k_scales[slot * (D / 16) + lane / LB] = (uint8_t)ksc;
        a.v_scales[slot * (D / 16) + lane / LB] = (uint8_t)vsc;
      }
    } else if constexpr (KVK == 0) {
      *reinterpret_cast<V*>(a.k_pages + (slot * D + lane * E) * 2) = kv;
      *reinterpret_cast<V*>(a.v_pages + (slot * D + lane * E) * 2) = vv;
    } else {
      const uint32_t* kw = reinterpret_cast<const uint32_t*>(&kv);
      const uint32_t* vw = reinterpret_cast<const uint32_t*>(&vv);
      uint32_t kc[(E + 3) / 4] = {}, vc[(E + 3) / 4] = {};
#pragma unroll
      for (int w = 0; w < E / 2; ++w) {  // two bf16 -> two e4m3 codes (16 bits)
        kc[w / 2] |= bf16x2_to_e4m3x2(kw[w], a.kv_scale) << (16 * (w & 1));
        vc[w / 2] |= bf16x2_to_e4m3x2(vw[w], a.kv_scale) << (16 * (w & 1));
      }
      uint8_t* kd = a.k_pages + slot * D + lane * E;
      uint8_t* vd = a.v_pages + slot * D + lane * E;
      if constexpr (E == 2) {
        *reinterpret_cast<uint16_t*>(kd) = (uint16_t)kc[0];
        *reinterpret_cast<uint16_t*>(vd) = (uint16_t)vc[0];
      } else if constexpr (E == 4) {
        *reinterpret_cast<uint32_t*>(kd) = kc[0];
        *reinterpret_cast<uint32_t*>(vd) = vc[0];
      } else {
        *reinterpret_cast<uint2*>(kd) = make_uint2(kc[0], kc[1]);
        *reinterpret_cast<uint2*>(vd) = make_uint2(vc[0], vc[1]);
      }
    }
  }
}

template <int D>
cudaError_t launch_append(int kvk, const AppendArgs& a, int grid, cudaStream_t stream) {
  if (kvk == 2)
    kv_append_kernel<D, 2><<<grid, 256, 0, stream>>>(a);
  else if (kvk == 1)
    kv_append_kernel<D, 1><<<grid, 256, 0, stream>>>(a);
  else
    kv_append_kernel<D, 0><<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

int* device_error_word();  // paged_decode_attn.cu

}  // namespace pda

extern "C" {

pda_status paged_kv_append(const void* k_new, const void* v_new, const int32_t* page_table,
                           const int32_t* kv_lens, const pda_append_params* p, void* k_pages,
                           void* v_pages, pda_stream_t stream_) {
  if (p == nullptr) return PDA_ERR_INVALID_ARG;
  if (p->batch < 0 || p->num_new < 1 || p->num_new > 64 || p->num_kv_heads < 1 ||
      p->max_pages_per_seq < 1 || p->num_pages < 1)
    return PDA_ERR_INVALID_ARG;
  if (p->kv_dtype != PDA_KV_BF16 && p->kv_dtype != PDA_KV_FP8_E4M3 &&
      p->kv_dtype != PDA_KV_NVFP4)
    return PDA_ERR_INVALID_ARG;
  const bool fp8 = p->kv_dtype == PDA_KV_FP8_E4M3;
  const bool nvfp4 = p->kv_dtype == PDA_KV_NVFP4;
  if ((fp8 || nvfp4) && (!(p->kv_scale > 0.f) || !(p->kv_scale < 3.4e38f)))
    return PDA_ERR_INVALID_ARG;
  if ((long long)p->max_pages_per_seq * p->page_size > 0x7FFFFFFFll) return PDA_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128 && p->head_dim != 256) return PDA_ERR_UNSUPPORTED;
  if (p->page_size < 8 || p->page_size > 256 || (p->page_size & (p->page_size - 1)))
    return PDA_ERR_UNSUPPORTED;
  if (p->batch == 0) return PDA_OK;
  if (!k_new || !v_new || !page_table || !kv_lens || !k_pages || !v_pages)
    return PDA_ERR_INVALID_ARG;
  if (nvfp4 && (!p->k_scales || !p->v_scales)) return PDA_ERR_INVALID_ARG;
  auto al = [](const void* x, uintptr_t n) { return (reinterpret_cast<uintptr_t>(x) & (n - 1)) == 0; };
  if (!al(k_new, 16) || !al(v_new, 16) || !al(k_pages, 16) || !al(v_pages, 16) ||
      !al(page_table, 4) || !al(kv_lens, 4))
    return PDA_ERR_MISALIGNED;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return PDA_ERR_CUDA;
  pda::AppendArgs a{};
  a.k_new = static_cast<const uint16_t*>(k_new);
  a.v_new = static_cast<const uint16_t*>(v_new);
  a.page_table = page_table;
  a.kv_lens = kv_lens;
  a.k_pages = static_cast<uint8_t*>(k_pages);
  a.v_pages = static_cast<uint8_t*>(v_pages);
  a.k_scales = nvfp4 ? static_cast<uint8_t*>(p->k_scales) : nullptr;
  a.v_scales = nvfp4 ? static_cast<uint8_t*>(p->v_scales) : nullptr;
  a.err = pda::device_error_word();
  if (a.err == nullptr) return PDA_ERR_CUDA;
  a.B = p->batch;
  a.T = p->num_new;
  a.Hkv = p->num_kv_heads;
  a.page_size = p->page_size;
  int lg = 0;
  while ((1 << lg) < p->page_size) ++lg;
  a.log2_page = lg;
  a.max_pages = p->max_pages_per_seq;
  a.num_pages = p->num_pages;
  a.kv_scale = (fp8 || nvfp4) ? p->kv_scale : 1.f;
  const long long rows = (long long)p->batch * p->num_new * p->num_kv_heads;
  const long long want = (rows + 7) / 8;  // 8 warps per CTA, a warp per row
  const int grid = (int)(want < (long long)sms * 4 ? want : (long long)sms * 4);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  cudaError_t e;
  const int kvk = nvfp4 ? 2 : (fp8 ? 1 : 0);
  switch (p->head_dim) {
    case 64: e = pda::launch_append<64>(kvk, a, grid, stream); break;
    case 128: e = pda::launch_append<128>(kvk, a, grid, stream); break;
    default: e = pda::launch_append<256>(kvk, a, grid, stream); break;
  }
  return e == cudaSuccess ? PDA_OK : PDA_ERR_CUDA;
}

}  // extern "C"
