// paged_decode_attn_no_alloc: the paged decode call with its whole workspace
// (the tensor-core kernel's counter header, work-queue order and FP8 Q
// operand images, and the split-KV partials) kept in a fixed device array
// that ships with the library, for callers that cannot allocate device
// memory. The limit applies to paged_decode_attn_workspace_bytes(params).
//
// Who cannot allocate: a serving engine that reserves nearly all of HBM for
// its own KV-cache pool at start-up and lets no library allocate afterwards;
// code on a latency-critical path, where cudaMalloc / cudaFree may
// synchronise the whole device; plugins whose host forbids allocation behind
// its back. paged_decode_attn already accepts a caller workspace; this entry
// point is for callers that cannot produce one either.
//
// The array is a file-scope __device__ symbol of PDA_NO_ALLOC_WORKSPACE_BYTES.
// Every device that loads the library holds it until the process exits. Host
// code may not use the symbol's name as a device address, so the first call
// on each device looks the address up with cudaGetSymbolAddress (with that
// device current) and keeps it.
#include <cuda_runtime.h>

#include <mutex>

#include "paged_decode_attn.h"

namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_workspace[PDA_NO_ALLOC_WORKSPACE_BYTES];

struct StaticWorkspace {
  bool ready = false;
  void* ptr = nullptr;  // device address of g_static_workspace on this device
};

StaticWorkspace g_ws[kMaxDevices];
std::mutex g_ws_mu;

// Device address of the static workspace on the current device, looked up
// once per device. Returns PDA_ERR_CUDA if the lookup fails.
pda_status static_workspace(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PDA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_ws_mu);
  StaticWorkspace& w = g_ws[dev];
  if (!w.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr)
      return PDA_ERR_CUDA;
    w.ptr = p;
    w.ready = true;
  }
  *out = w.ptr;
  return PDA_OK;
}

}  // namespace

extern "C" {

pda_status paged_decode_attn_no_alloc(const void* q, const void* k_pages, const void* v_pages,
                                      const int32_t* page_table, const int32_t* kv_lens,
                                      const pda_params* params, float* out, float* lse,
                                      pda_stream_t stream) {
  if (params == nullptr) return PDA_ERR_INVALID_ARG;
  const size_t need = paged_decode_attn_workspace_bytes(params);
  if (need == SIZE_MAX) return PDA_ERR_INVALID_ARG;
  if (need > (size_t)PDA_NO_ALLOC_WORKSPACE_BYTES) return PDA_ERR_WORKSPACE;
  pda_params p = *params;
  p.workspace = nullptr;
  p.workspace_bytes = 0;
  if (need > 0) {
    void* ws = nullptr;
    const pda_status st = static_workspace(&ws);
    if (st != PDA_OK) return st;
    p.workspace = ws;
    p.workspace_bytes = PDA_NO_ALLOC_WORKSPACE_BYTES;
  }
  return paged_decode_attn(q, k_pages, v_pages, page_table, kv_lens, &p, out, lse, stream);
}

}  // extern "C"
