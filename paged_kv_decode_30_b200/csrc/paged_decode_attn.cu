// Host side of the paged decode attention library: argument validation, the
// split planner, workspace, kernel dispatch and the exported C ABI.
//
// Sources: "AstrAI commit log, attn_paged_decode_split_kv_mma.cuh"
// (compute_num_splits / alloc_split_partials / dispatch_head_dim host
// helpers; the split kernel writes every partial slot it owns, so partials
// are never cleared) and "b12x 0.30.0, Kernel inventory, Attention table,
// Paged attention row" (split-KV or direct output; separate merge kernel).
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "merge.cuh"
#include "paged_decode_attn.h"
#include "split_tma.cuh"
#include "split_variants.cuh"

namespace pda {

// One device error word per device that loads the library.
__device__ int g_error_word = 0;

namespace {

constexpr int kMaxDevices = 64;
// Modelled cost of the merge launch, in units of one CTA iteration
// (NW warp tiles, ~64 KB of K/V at the per-SM share of HBM bandwidth).
constexpr int kMergeCostIters = 2;
// Fixed cost of one CTA (pipeline fill: the first tiles' copy latency, the
// page-id prefetch, the epilogue), in the same units.
constexpr int kCtaFillIters = 1;
constexpr int kMaxSplits = 128;

struct DeviceState {
  bool init = false;
  int num_sms = 0;
  int* err = nullptr;        // device address of g_error_word
  void* ws = nullptr;        // library-owned workspace (grow-only)
  size_t ws_bytes = 0;
};

DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

pda_status device_state(DeviceState** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return PDA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& st = g_dev[dev];
  if (!st.init) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return PDA_ERR_CUDA;
    void* err = nullptr;
    if (cudaGetSymbolAddress(&err, g_error_word) != cudaSuccess) return PDA_ERR_CUDA;
    st.num_sms = sms;
    st.err = static_cast<int*>(err);
    st.init = true;
  }
  *out = &st;
  return PDA_OK;
}

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
int ilog2(int x) { int l = 0; while ((1 << l) < x) ++l; return l; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

// Static shape of the launch that a params struct leads to.
struct Plan {
  int G, M, mt, row_tiles, tw, elt;
  long long rows;          // B * q_len * Hq
  int tiles_per_cta_iter;  // tokens one CTA iteration covers = tw * warps
  bool tc;                 // tensor-core kernel (else the FMA kernel)
};

// TMA coordinates are 32-bit: the pool's rows must fit.
bool pool_rows_fit(const pda_params* p) {
  return (long long)p->num_pages * p->num_kv_heads * p->page_size < (1ll << 31);
}

// Kernel choice for head_dim 128 (the tensor-core kernel's only width):
//  - FP8 K/V with more than 8 packed rows per kv head (G * q_len): QK^T and
//    PV are dense contractions with N = 16 or 32 rows;
//  - bf16 K/V with at most 8 packed rows: one CTA per (b, kv head) streams
//    the K/V tiles by TMA and hands the contractions to tcgen05, which keeps
//    the SMs' issue slots (and power) free; measured faster than the FMA
//    kernel at both full and power-capped clocks on the long-context bf16
//    workloads.
// The flags force either kernel.
bool use_tensor_cores(const pda_params* p, int M) {
  if (p->head_dim != 128 || p->page_size < 8 || !pool_rows_fit(p)) return false;
  if (p->flags & PDA_FLAG_CUDA_CORES) return false;
  if (p->flags & PDA_FLAG_TENSOR_CORES) return true;
  // FP8: dense contractions with 16 or 32 rows; bf16 and NVFP4 (decoded to
  // f16 tiles in shared memory): the 16-bit path with up to 8 rows
  return p->kv_dtype == PDA_KV_FP8_E4M3 ? M > 8 : M <= 8;
}

pda_status validate(const pda_params* p) {
  if (p == nullptr) return PDA_ERR_INVALID_ARG;
  if (p->batch < 0 || p->q_len < 1 || p->num_q_heads < 1 || p->num_kv_heads < 1)
    return PDA_ERR_INVALID_ARG;
  if (p->num_q_heads % p->num_kv_heads != 0) return PDA_ERR_INVALID_ARG;
  if (p->head_dim < 1 || p->page_size < 1 || p->max_pages_per_seq < 1 || p->num_pages < 1)
    return PDA_ERR_INVALID_ARG;
  if (!(p->scale > 0.f) || !std::isfinite(p->scale)) return PDA_ERR_INVALID_ARG;
  if (p->causal_offset < PDA_CAUSAL_BOTTOM_RIGHT) return PDA_ERR_INVALID_ARG;
  if (p->kv_dtype != PDA_KV_BF16 && p->kv_dtype != PDA_KV_FP8_E4M3 &&
      p->kv_dtype != PDA_KV_NVFP4)
    return PDA_ERR_INVALID_ARG;
  if (p->kv_dtype != PDA_KV_BF16 && (!(p->kv_scale > 0.f) || !std::isfinite(p->kv_scale)))
    return PDA_ERR_INVALID_ARG;
  if (p->max_kv_len < 0 || p->num_splits < 0) return PDA_ERR_INVALID_ARG;
  if ((long long)p->max_pages_per_seq * p->page_size > INT_MAX) return PDA_ERR_INVALID_ARG;
  // supported variants
  if (p->head_dim != 64 && p->head_dim != 128 && p->head_dim != 256) return PDA_ERR_UNSUPPORTED;
  if (!is_pow2(p->page_size) || p->page_size < 8 || p->page_size > 256) return PDA_ERR_UNSUPPORTED;
  if (p->q_len > 8) return PDA_ERR_UNSUPPORTED;
  if (p->batch > 65535) return PDA_ERR_UNSUPPORTED;
  return PDA_OK;
}

Plan make_plan(const pda_params* p) {
  Plan pl{};
  pl.G = p->num_q_heads / p->num_kv_heads;
  pl.M = pl.G * p->q_len;
  pl.elt = p->kv_dtype == PDA_KV_BF16 ? 2 : 1;  // NVFP4: codes are half a byte (see below)
  pl.rows = (long long)p->batch * p->q_len * p->num_q_heads;
  pl.tc = use_tensor_cores(p, pl.M);
  if (pl.tc) {
    if (p->kv_dtype == PDA_KV_FP8_E4M3)
      pl.mt = pl.M <= 16 ? 16 : 32;  // rows per CTA; MMA N = 2 * rows for S^T
    else
      pl.mt = pl.M <= 4 ? 4 : 8;     // 16-bit: N = 16 holds P^T hi and lo rows
    pl.tw = 128;                   // tokens per tile (MMA M)
    pl.tiles_per_cta_iter = 128;
  } else {
    pl.mt = pl.M >= 8 ? 8 : (pl.M >= 4 ? 4 : (pl.M >= 2 ? 2 : 1));
    const int tw_full = 8 * (32 / (p->head_dim / 8));
    pl.tw = p->page_size < tw_full ? p->page_size : tw_full;
    pl.tiles_per_cta_iter = pl.tw * fma_warps(pl.mt);
  }
  pl.row_tiles = (int)cdiv(pl.M, pl.mt);
  return pl;
}

int choose_splits(const pda_params* p, const Plan& pl, int num_sms) {
  const long long len_bound =
      p->max_kv_len > 0 ? p->max_kv_len : (long long)p->max_pages_per_seq * p->page_size;
  // Keys one row tile can see: bounded by the window (plus the spread of the
  // tile's query positions) when a window is set.
  long long span = len_bound;
  if (p->window > 0) span = std::min<long long>(span, (long long)p->window + p->q_len);
  const long long max_tiles = std::max<long long>(1, cdiv(span, pl.tw));
  if (p->num_splits > 0) return (int)std::min<long long>(p->num_splits, std::min<long long>(max_tiles, kMaxSplits));
  const long long iters = std::max<long long>(1, cdiv(span, pl.tiles_per_cta_iter));
  const long long units = (long long)p->batch * p->num_kv_heads * pl.row_tiles;
  const long long slots = std::max(1, num_sms);  // one CTA per SM
  // Persistent tensor-core kernel: its queue hands out the longest sequences
  // first, so once there are 1.5 units per SM or more the CTAs finish close
  // together without splitting, and a split only adds per-item work and the
  // merge (measured on B200: the FP8 verify and mixed-length bf16 workloads
  // run 13-15% faster unsplit). Fewer units: the wave model below.
  if (pl.tc && 2 * units >= 3 * slots) return 1;
  long long best_cost = LLONG_MAX;
  int best = 1;
  const long long smax = std::min<long long>(std::min<long long>(iters, max_tiles), kMaxSplits);
  for (long long s = 1; s <= smax; ++s) {
    if (s * p->num_kv_heads > 65535) break;
    const long long waves = cdiv(units * s, slots);
    const long long cost =
        waves * (cdiv(iters, s) + kCtaFillIters) + (s > 1 ? kMergeCostIters : 0);
    if (cost < best_cost) {
      best_cost = cost;
      best = (int)s;
    }
  }
  return best;
}

// Workspace layout. The tensor-core kernel keeps its work-queue counter and
// split-arrival counters per (sequence, kv head, row tile) at the front
// (zeroed on every call by the kernel's prologue, launched just before it on
// the call's stream), then the queue order and the FP8 Q operand images; the
// split partials follow (o_part then lse_part).
struct WsLayout {
  size_t counters;  // bytes of the counter header (0 for the FMA kernel)
  size_t order_off, qops_off;  // tensor-core kernel: queue order, FP8 Q images
  size_t o_off, lse_off, total;
};
constexpr size_t kMergeCtrOffset = 64;  // bytes: after the work-queue counters
// Batches up to this size get a longest-first queue order (one CTA sorts
// them); larger ones are handed out in sequence order.
constexpr int kMaxOrderedBatch = 1 << 16;

size_t round256(size_t x) { return (x + 255) / 256 * 256; }


WsLayout ws_layout(const pda_params* p, const Plan& pl, int splits) {
  WsLayout w{};
  size_t end = 0;
  if (pl.tc) {
    const size_t groups = (size_t)p->batch * (size_t)p->num_kv_heads * (size_t)pl.row_tiles;
    w.counters = kMergeCtrOffset + groups * pda::kMergeCtrPerGroup * sizeof(int);
    w.order_off = round256(w.counters);
    end = w.order_off + round256((size_t)p->batch * sizeof(int));
    if (p->kv_dtype == PDA_KV_FP8_E4M3) {  // Q operand image + 32 row scales per group
      const bool native = (p->flags & PDA_FLAG_NATIVE_FP8_QK) != 0;
      const size_t qop = (size_t)(native ? pl.mt : 2 * pl.mt) * 128 + 128;
      w.qops_off = end;
      end += round256(groups * qop);
    }
  }
  w.o_off = w.lse_off = w.total = end;
  if (splits > 1) {
    const size_t o_bytes = (size_t)splits * (size_t)pl.rows * (size_t)p->head_dim * sizeof(float);
    w.lse_off = w.o_off + round256(o_bytes);
    w.total = w.lse_off + (size_t)splits * (size_t)pl.rows * sizeof(float);
  }
  return w;
}

}  // namespace

// Device address of the current device's error word (nullptr if the device
// cannot be initialised); used by the other entry points of the library.
int* device_error_word() {
  DeviceState* st = nullptr;
  return device_state(&st) == PDA_OK ? st->err : nullptr;
}

cudaError_t launch_merge(int D, const float* o_parts, const float* lse_parts,
                         int num_splits, long long rows, float* out, float* lse,
                         const float* sinks, int Hq, cudaStream_t stream, bool pdl) {
  if (rows <= 0) return cudaSuccess;
  constexpr int kWarpsPerBlock = 8;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)cdiv(rows, kWarpsPerBlock));
  cfg.blockDim = dim3(kWarpsPerBlock * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  switch (D) {
    case 64: return cudaLaunchKernelEx(&cfg, merge_states_kernel<64>, o_parts, lse_parts, num_splits, rows, out, lse, sinks, Hq);
    case 128: return cudaLaunchKernelEx(&cfg, merge_states_kernel<128>, o_parts, lse_parts, num_splits, rows, out, lse, sinks, Hq);
    case 256: return cudaLaunchKernelEx(&cfg, merge_states_kernel<256>, o_parts, lse_parts, num_splits, rows, out, lse, sinks, Hq);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace pda

using namespace pda;

extern "C" {

int32_t pda_abi_version(void) { return PDA_ABI_VERSION; }

const char* pda_status_string(pda_status s) {
  switch (s) {
    case PDA_OK: return "ok";
    case PDA_ERR_INVALID_ARG: return "invalid argument";
    case PDA_ERR_UNSUPPORTED: return "unsupported configuration";
    case PDA_ERR_MISALIGNED: return "misaligned pointer";
    case PDA_ERR_WORKSPACE: return "workspace too small or allocation failed";
    case PDA_ERR_CUDA: return "CUDA error";
    case PDA_ERR_BAD_PAGE: return "page id or kv length out of range (device)";
    case PDA_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

int32_t pda_plan_kernel(const pda_params* params) {
  if (validate(params) != PDA_OK) return -1;
  return make_plan(params).tc ? PDA_KERNEL_SPLIT_TMA : PDA_KERNEL_SPLIT_FMA;
}

int32_t pda_choose_num_splits(const pda_params* params, int32_t num_sms) {
  if (validate(params) != PDA_OK || num_sms < 1) return 0;
  return choose_splits(params, make_plan(params), num_sms);
}

size_t paged_decode_attn_workspace_bytes(const pda_params* params) {
  if (validate(params) != PDA_OK) return SIZE_MAX;
  const Plan pl = make_plan(params);
  int sms = 148;
  DeviceState* st = nullptr;
  if (params->num_splits == 0 && device_state(&st) == PDA_OK) sms = st->num_sms;
  const int s = choose_splits(params, pl, sms);
  return ws_layout(params, pl, s).total;
}

pda_status paged_decode_attn(const void* q, const void* k_pages, const void* v_pages,
                             const int32_t* page_table, const int32_t* kv_lens,
                             const pda_params* params, float* out, float* lse,
                             pda_stream_t stream_) {
  pda_status st = validate(params);
  if (st != PDA_OK) return st;
  const pda_params& p = *params;
  if (p.batch == 0) {
    if (p.num_splits_out) *p.num_splits_out = 1;
    return PDA_OK;
  }
  if (!q || !k_pages || !v_pages || !page_table || !kv_lens || !out) return PDA_ERR_INVALID_ARG;
  const bool nvfp4 = p.kv_dtype == PDA_KV_NVFP4;
  if (nvfp4 && (!p.k_scales || !p.v_scales)) return PDA_ERR_INVALID_ARG;
  if (nvfp4 && (!aligned(p.k_scales, 16) || !aligned(p.v_scales, 16))) return PDA_ERR_MISALIGNED;
  if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(out, 16) ||
      !aligned(page_table, 4) || !aligned(kv_lens, 4) || (lse && !aligned(lse, 4)) ||
      (p.sinks && !aligned(p.sinks, 4)))
    return PDA_ERR_MISALIGNED;
  if (p.workspace && !aligned(p.workspace, 256)) return PDA_ERR_MISALIGNED;

  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  DeviceState* dev = nullptr;
  if ((st = device_state(&dev)) != PDA_OK) return st;

  const Plan pl = make_plan(params);
  const int splits = choose_splits(params, pl, dev->num_sms);
  if ((long long)splits * p.num_kv_heads > 65535) return PDA_ERR_UNSUPPORTED;

  SplitArgs a{};
  a.q = static_cast<const uint16_t*>(q);
  a.k_pages = static_cast<const uint8_t*>(k_pages);
  a.v_pages = static_cast<const uint8_t*>(v_pages);
  a.page_table = page_table;
  a.kv_lens = kv_lens;
  a.out = out;
  a.lse = lse;
  a.err = dev->err;
  a.B = p.batch;
  a.Lq = p.q_len;
  a.Hq = p.num_q_heads;
  a.Hkv = p.num_kv_heads;
  a.G = pl.G;
  a.M = pl.M;
  a.page_size = p.page_size;
  a.log2_page = ilog2(p.page_size);
  a.max_pages = p.max_pages_per_seq;
  a.num_pages = p.num_pages;
  a.tile_shift = pl.tc ? 0 : ilog2(p.page_size / pl.tw);
  a.num_splits = splits;
  a.sinks = p.sinks;
  a.row_tiles = pl.row_tiles;
  a.causal_offset = p.causal_offset;
  a.window = p.window;
  const float log2e = 1.4426950408889634f;
  const bool fp8 = p.kv_dtype == PDA_KV_FP8_E4M3;
  const bool scaled = p.kv_dtype != PDA_KV_BF16;  // FP8 and NVFP4 carry kv_scale
  a.qk_scale_log2 = p.scale * log2e * (scaled ? p.kv_scale : 1.f);
  a.v_scale = scaled ? p.kv_scale : 1.f;
  a.head_stride = nvfp4 ? (long long)p.page_size * p.head_dim / 2
                        : (long long)p.page_size * p.head_dim * pl.elt;
  a.page_stride = a.head_stride * p.num_kv_heads;
  if (nvfp4) {
    a.k_scales = static_cast<const uint8_t*>(p.k_scales);
    a.v_scales = static_cast<const uint8_t*>(p.v_scales);
    a.sc_head_stride = (long long)p.page_size * p.head_dim / 16;
    a.sc_page_stride = a.sc_head_stride * p.num_kv_heads;
  }

  const WsLayout wl = ws_layout(&p, pl, splits);
  if (wl.total > 0) {
    void* ws = p.workspace;
    if (ws == nullptr) {
      std::lock_guard<std::mutex> lock(g_mu);
      if (dev->ws_bytes < wl.total) {
        // Grow stream-ordered: the old buffer is released after the work
        // already queued on `stream`, the new one is ready for the work
        // queued next, and neither step synchronises the device. A call
        // being captured into a CUDA graph cannot grow the buffer (the
        // allocation would belong to the graph).
        cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return PDA_ERR_CUDA;
        if (cap != cudaStreamCaptureStatusNone) return PDA_ERR_WORKSPACE;
        if (dev->ws && cudaFreeAsync(dev->ws, stream) != cudaSuccess) return PDA_ERR_CUDA;
        dev->ws = nullptr;
        dev->ws_bytes = 0;
        void* fresh = nullptr;
        if (cudaMallocAsync(&fresh, wl.total, stream) != cudaSuccess) {
          (void)cudaGetLastError();
          return PDA_ERR_WORKSPACE;
        }
        dev->ws = fresh;
        dev->ws_bytes = wl.total;
      }
      ws = dev->ws;
    } else if (p.workspace_bytes < wl.total) {
      return PDA_ERR_WORKSPACE;
    }
    char* base = static_cast<char*>(ws);
    if (pl.tc) {
      // the kernel's prologue zeroes the counters for this call, ranks the
      // sequences into the queue order and writes the FP8 Q images
      a.sched = reinterpret_cast<int*>(base);
      a.merge_ctr = reinterpret_cast<int*>(base + kMergeCtrOffset);
      a.header_words = (int)(wl.counters / sizeof(int));
      a.order = p.batch <= kMaxOrderedBatch ? reinterpret_cast<int*>(base + wl.order_off) : nullptr;
      a.qops = fp8 ? reinterpret_cast<uint8_t*>(base + wl.qops_off) : nullptr;
    }
    if (splits > 1) {
      a.o_part = reinterpret_cast<float*>(base + wl.o_off);
      a.lse_part = reinterpret_cast<float*>(base + wl.lse_off);
    }
  }

  cudaError_t e;
  const int kv = nvfp4 ? 2 : (fp8 ? 1 : 0);
  if (pl.tc) {
    // persistent: at most one CTA per SM, items from the work queue; the
    // split that finishes last for a group of rows merges it (no merge launch)
    const long long items = (long long)p.batch * p.num_kv_heads * splits * pl.row_tiles;
    if (items > INT_MAX) return PDA_ERR_UNSUPPORTED;
    a.num_items = (int)items;
    a.fused_merge = (p.flags & PDA_FLAG_FUSED_MERGE) != 0;
    const int grid = (int)std::min<long long>(items, dev->num_sms);
    e = launch_split_tma(kv, pl.mt, fp8 && (p.flags & PDA_FLAG_NATIVE_FP8_QK) != 0, k_pages,
                         v_pages, a, grid, stream, (p.flags & PDA_FLAG_NO_PDL) == 0);
  } else {
    const dim3 grid((unsigned)pl.row_tiles, (unsigned)(splits * p.num_kv_heads), (unsigned)p.batch);
    switch (p.head_dim) {
      case 64: e = launch_split_d64(kv, pl.mt, pl.tw, a, grid, stream); break;
      case 128: e = launch_split_d128(kv, pl.mt, pl.tw, a, grid, stream); break;
      case 256: e = launch_split_d256(kv, pl.mt, pl.tw, a, grid, stream); break;
      default: e = cudaErrorNotSupported;
    }
  }
  if (e == cudaErrorNotSupported) return PDA_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return PDA_ERR_CUDA;
  if (splits > 1 && !(pl.tc && a.fused_merge)) {
    e = launch_merge(p.head_dim, a.o_part, a.lse_part, splits, pl.rows, out, lse, p.sinks,
                     p.num_q_heads, stream, (p.flags & PDA_FLAG_NO_PDL) == 0);
    if (e != cudaSuccess) return PDA_ERR_CUDA;
  }
  if (p.num_splits_out) *p.num_splits_out = splits;
  return PDA_OK;
}

pda_status pda_merge_states(const float* o_parts, const float* lse_parts, int32_t num_splits,
                            int64_t rows, int32_t head_dim, float* out, float* lse,
                            const float* sinks, int32_t num_q_heads, pda_stream_t stream) {
  if (num_splits < 1 || rows < 0) return PDA_ERR_INVALID_ARG;
  if (sinks && num_q_heads < 1) return PDA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return PDA_ERR_UNSUPPORTED;
  if (rows == 0) return PDA_OK;
  if (!o_parts || !lse_parts || !out) return PDA_ERR_INVALID_ARG;
  if (!aligned(o_parts, 16) || !aligned(out, 16) || !aligned(lse_parts, 4) ||
      (lse && !aligned(lse, 4)) || (sinks && !aligned(sinks, 4)))
    return PDA_ERR_MISALIGNED;
  const cudaError_t e = launch_merge(head_dim, o_parts, lse_parts, num_splits, rows, out, lse,
                                     sinks, sinks ? num_q_heads : 1,
                                     reinterpret_cast<cudaStream_t>(stream), false);
  return e == cudaSuccess ? PDA_OK : PDA_ERR_CUDA;
}

pda_status pda_last_device_error(pda_stream_t stream) {
  DeviceState* dev = nullptr;
  pda_status st = device_state(&dev);
  if (st != PDA_OK) return st;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PDA_ERR_CUDA;
  int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(int)) != cudaSuccess) return PDA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int)) != cudaSuccess) return PDA_ERR_CUDA;
  return static_cast<pda_status>(word);
}

}  // extern "C"
