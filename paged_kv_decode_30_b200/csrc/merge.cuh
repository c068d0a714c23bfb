// LSE merge of split-KV partials.
//
// Sources: "b12x 0.30.0, Kernel inventory, Attention table, Paged attention
// row" (PagedPersistentMergeKernel: split-KV partials merged by a separate
// kernel) and "sglang profiler skill, fuse-overlap catalog, vLLM-origin
// attention + output quant row" (merge_attn_states).
//
// For a row r with parts s = 0..S-1 (each a softmax over a disjoint key set,
// stored normalised with its own lse):
//   lse = m + ln sum_s exp(lse_s - m),  m = max_s lse_s
//   out = sum_s exp(lse_s - lse) * o_s
// An attention-sink logit of the row's query head (optional) is one more
// part with lse = sink and o = 0: it adds to the denominator only.
// One warp per row, head_dim across the lanes in 8/16/32-byte vectors. Parts
// with lse = -inf are skipped without reading their o. Launched with
// programmatic dependent launch after the split kernel, so its CTAs are
// resident and waiting when the split grid finishes.
#pragma once

#include "pda_device.cuh"

namespace pda {

template <int D>
__global__ void __launch_bounds__(256) merge_states_kernel(
    const float* __restrict__ o_parts, const float* __restrict__ lse_parts,
    int num_splits, long long rows, float* __restrict__ out,
    float* __restrict__ lse, const float* __restrict__ sinks, int Hq) {
  pdl_wait_primary();  // no-op unless launched as a programmatic dependent
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;

  const float sink = sinks != nullptr ? __ldg(sinks + row % Hq) : -INFINITY;
  float m = sink;
  for (int s = 0; s < num_splits; ++s) m = fmaxf(m, __ldg(lse_parts + s * rows + row));
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float total = -INFINITY;
  if (m != -INFINITY) {
    float sum = 0.f;
    for (int s = 0; s < num_splits; ++s) {
      const float ls = __ldg(lse_parts + s * rows + row);
      if (ls != -INFINITY) sum += expf(ls - m);
    }
    if (sink != -INFINITY) sum += expf(sink - m);
    total = m + logf(sum);
    for (int s = 0; s < num_splits; ++s) {
      const float ls = __ldg(lse_parts + s * rows + row);
      if (ls == -INFINITY) continue;
      const float w = expf(ls - total);
      const float* src = o_parts + (s * rows + row) * D + lane * PER;
#pragma unroll
      for (int e = 0; e < PER; e += 2) {
        const float2 x = __ldg(reinterpret_cast<const float2*>(src + e));
        acc[e] = fmaf(w, x.x, acc[e]);
        acc[e + 1] = fmaf(w, x.y, acc[e + 1]);
      }
    }
  }
  float* dst = out + row * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; e += 2)
    *reinterpret_cast<float2*>(dst + e) = make_float2(acc[e], acc[e + 1]);
  if (lse != nullptr && lane == 0) lse[row] = total;
}

cudaError_t launch_merge(int D, const float* o_parts, const float* lse_parts,
                         int num_splits, long long rows, float* out, float* lse,
                         const float* sinks, int Hq, cudaStream_t stream, bool pdl);

}  // namespace pda
