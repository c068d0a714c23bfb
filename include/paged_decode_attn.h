/*
 * paged_decode_attn: paged-KV decode attention for NVIDIA B200 (sm_100a).
 *
 * The operation (one decode step of one attention layer): for every sequence
 * b, query row i and query head h, softmax attention of q[b, i, h, :] over the
 * keys of sequence b, with K/V rows gathered through a page table:
 *
 *   s_j   = scale * q . k_j              for every key j the row may see
 *   lse   = ln sum_j exp(s_j)
 *   out   = sum_j exp(s_j - lse) * v_j
 *
 * Sources (page title, section):
 *  - "AstrAI commit log, attn_paged_decode_split_kv_mma.cuh": split-KV paged
 *    decode; per-position page-table lookup when loading K/V tiles; GQA head
 *    packing; causal_offset (-1 off, >= 0 first query position); split
 *    partials written without a memset; compute_num_splits.
 *  - "b12x 0.30.0, Kernel inventory, Attention table, Paged attention row":
 *    bf16 and FP8-E4M3 KV caches, split-KV or direct output, sliding window,
 *    GQA, and a persistent merge kernel for the split partials.
 *  - "sglang profiler skill, fuse-overlap catalog, vLLM-origin attention +
 *    output quant row": merge_attn_states merges attention states by LSE.
 *
 * Where the pages leave the operation open, this library takes:
 *  - lse is a natural logarithm.
 *  - causal_offset = PDA_CAUSAL_BOTTOM_RIGHT (-2) aligns query row i of
 *    sequence b at position kv_lens[b] - q_len + i (speculative verify rows).
 *  - a window of W keys includes the query's own position: key j is visible
 *    to a row at position pos iff j >= pos - W + 1; window <= 0 is off; with
 *    causal off the window is measured from kv_lens[b] - 1.
 *  - query head h reads kv head h / (num_q_heads / num_kv_heads).
 *  - KV pools are laid out [num_pages, num_kv_heads, page_size, head_dim].
 *  - FP8: element value = e4m3 code * kv_scale, one scale shared by K and V.
 *  - NVFP4: element value = e2m1 code * e4m3 block scale * kv_scale, blocks
 *    of 16 consecutive elements of a token row, kv_scale shared by K and V.
 *  - a row that sees no key gets out = 0 and lse = -inf.
 *
 * All entry points return a status and never abort or throw. Device work is
 * asynchronous on the given stream; no entry point synchronises except
 * pda_last_device_error.
 */
#ifndef PAGED_DECODE_ATTN_H_
#define PAGED_DECODE_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PDA_API __attribute__((visibility("default")))
#else
#define PDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t); NULL is the legacy default stream. */
typedef struct CUstream_st* pda_stream_t;

#define PDA_ABI_VERSION 3

typedef enum {
  PDA_KV_BF16 = 0,      /* K/V elements are bfloat16 */
  PDA_KV_FP8_E4M3 = 1,  /* K/V elements are FP8 E4M3 codes (uint8) */
  PDA_KV_NVFP4 = 2      /* K/V elements are NVFP4: FP4 E2M1 codes, two per byte
                           (even element in the low nibble), with one E4M3
                           scale per 16 consecutive elements of a row in
                           separate scale pools (pda_params.k_scales /
                           v_scales): value = e2m1 * e4m3 scale * kv_scale.
                           "b12x 0.30.0, Kernel inventory": NVFP4
                           (float4_e2m1fn) with E4M3 scales per 16 elements;
                           "sglang profiler skill, fuse-overlap catalog": FP4
                           paged KV caches. */
} pda_kv_dtype;

typedef enum {
  PDA_OK = 0,
  PDA_ERR_INVALID_ARG = 1,  /* a size, pointer or field is out of range */
  PDA_ERR_UNSUPPORTED = 2,  /* valid, but no kernel variant for it */
  PDA_ERR_MISALIGNED = 3,   /* a pointer is not 16-byte aligned */
  PDA_ERR_WORKSPACE = 4,    /* caller workspace too small / allocation failed */
  PDA_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed */
  PDA_ERR_BAD_PAGE = 6,     /* device saw a page id or kv_len out of range */
  PDA_ERR_TIMEOUT = 7       /* device gave up waiting on a copy */
} pda_status;

#define PDA_CAUSAL_OFF (-1)           /* no causal mask */
#define PDA_CAUSAL_BOTTOM_RIGHT (-2)  /* row i at kv_lens[b] - q_len + i */

/* flags */
#define PDA_FLAG_NO_PDL 1u  /* launch the merge without programmatic dependent launch */
#define PDA_FLAG_TENSOR_CORES 2u /* use the tensor-core kernel wherever it applies
                                    (head_dim 128), not only where the planner picks it */
#define PDA_FLAG_CUDA_CORES 4u   /* always use the CUDA-core (FMA) kernel */
#define PDA_FLAG_FUSED_MERGE 8u  /* tensor-core kernel with splits: the split that
                                    finishes last for a group of rows merges them
                                    in the kernel (no merge launch) */
#define PDA_FLAG_NATIVE_FP8_QK 16u /* FP8 K/V on the tensor-core kernel: q enters
                                    QK^T as one e4m3 value per element, e4m3 of
                                    q * 2^e (nearest even; 2^e the power of two
                                    that puts max|q| of its row in [128, 256)),
                                    instead of an exact two-term split. Changes
                                    the result: equal to attention with q
                                    replaced by e4m3(q * 2^e) * 2^-e. */

typedef struct {
  int32_t batch;            /* B >= 0 */
  int32_t q_len;            /* query rows per sequence, 1..8 */
  int32_t num_q_heads;      /* Hq, a multiple of num_kv_heads */
  int32_t num_kv_heads;     /* Hkv >= 1 */
  int32_t head_dim;         /* D in {64, 128, 256} */
  int32_t page_size;        /* P, a power of two in [8, 256] */
  int32_t max_pages_per_seq;/* row stride of page_table; kv_lens[b] <= this * P */
  int32_t num_pages;        /* pages in each pool; page ids must be < this */
  float scale;              /* softmax scale (> 0), e.g. 1/sqrt(D) */
  int32_t causal_offset;    /* PDA_CAUSAL_OFF, PDA_CAUSAL_BOTTOM_RIGHT, or >= 0 */
  int32_t window;           /* <= 0 off; else keys j >= pos - window + 1 */
  int32_t kv_dtype;         /* pda_kv_dtype */
  float kv_scale;           /* FP8 / NVFP4: value = code [* block scale] * kv_scale (> 0) */
  int32_t max_kv_len;       /* host hint, >= every kv_lens[b]; 0 -> max_pages_per_seq * P.
                               Used only to choose the split count. */
  int32_t num_splits;       /* 0 -> heuristic; > 0 forces this many KV splits */
  uint32_t flags;           /* PDA_FLAG_* */
  void* workspace;          /* device scratch (any contents), or NULL */
  size_t workspace_bytes;   /* size of workspace */
  int32_t* num_splits_out;  /* optional host out: split count used */
  const float* sinks;       /* optional device float [Hq]: attention-sink logit of each
                               query head (natural log, on the scale of scale*q.k):
                               exp(sinks[h]) joins the softmax denominator and adds
                               no value; a row with no visible key then gets
                               out = 0, lse = sinks[h]. NULL: no sink. */
  const void* k_scales;     /* NVFP4 only: device uint8 E4M3 block scales of K,
                               [num_pages, Hkv, P, D/16], 16-byte aligned */
  const void* v_scales;     /* NVFP4 only: the same for V. Ignored otherwise. */
} pda_params;

/*
 * Paged decode attention.
 *
 * q           device, bf16 [B, q_len, Hq, D], contiguous.
 * k_pages     device, [num_pages, Hkv, P, D] of bf16 (PDA_KV_BF16) or uint8
 * v_pages     e4m3 codes (PDA_KV_FP8_E4M3), or [num_pages, Hkv, P, D/2] of
 *             packed e2m1 codes (PDA_KV_NVFP4, with params->k_scales and
 *             v_scales), contiguous.
 * page_table  device, int32 [B, max_pages_per_seq]; entry t of row b is the
 *             pool page holding keys [t*P, (t+1)*P) of sequence b. Entries
 *             past ceil(kv_lens[b] / P) are never read (may hold -1).
 * kv_lens     device, int32 [B], keys per sequence (0 allowed).
 * params      host, read during the call only.
 * out         device, fp32 [B, q_len, Hq, D].
 * lse         device, fp32 [B, q_len, Hq], natural log; may be NULL.
 * stream      CUDA stream for all device work.
 *
 * Inputs are read only. Slots of a page past kv_lens[b], and keys no row
 * may see, are never weighted (their bytes may be NaN). q, k_pages, v_pages
 * and out must be 16-byte aligned; page_table, kv_lens and lse 4-byte
 * aligned; a caller workspace 256-byte aligned (else PDA_ERR_MISALIGNED).
 *
 * Workspace: paged_decode_attn_workspace_bytes(params) bytes of device
 * scratch. It holds the split partials when the call splits the KV range,
 * and, for the tensor-core kernel (see pda_plan_kernel), a header of
 * counters: the work queue of its persistent CTAs and, per (sequence, kv
 * head, row tile) and softmax row group, how many splits have finished
 * (the last one merges).
 * The tensor-core kernel's prologue (a small kernel launched on `stream`
 * just before it) zeroes that header on every call, so the workspace's
 * contents before the call do not matter and a call captured in a CUDA graph
 * replays correctly. Every partial slot
 * a kernel reads was written earlier in the same call. If params->workspace is NULL the library
 * uses a grow-only buffer it owns, one per device, shared by every call on
 * that device: calls that may overlap on different streams must pass their
 * own workspace (the same holds for a caller workspace). A call that needs
 * more than that buffer holds grows it in stream order on `stream`: the old
 * buffer is released with cudaFreeAsync and the new one taken with
 * cudaMallocAsync (the device's default memory pool); neither synchronises
 * the device. During stream capture the buffer cannot grow: such a call
 * returns PDA_ERR_WORKSPACE, so make one call with the largest params before
 * capturing, or pass a workspace.
 *
 * Errors: invalid sizes or pointers return before any device work. A page
 * id >= num_pages or < 0 met on the device is never dereferenced; the kernel
 * records PDA_ERR_BAD_PAGE in a device error word (see pda_last_device_error)
 * and the affected output is unspecified.
 */
PDA_API pda_status paged_decode_attn(const void* q, const void* k_pages,
                             const void* v_pages, const int32_t* page_table,
                             const int32_t* kv_lens, const pda_params* params,
                             float* out, float* lse, pda_stream_t stream);

/*
 * paged_decode_attn for callers that cannot allocate device memory. The
 * pages describe no counterpart to this entry point; it exists for callers
 * such as a serving engine that reserves nearly all of HBM for its own
 * KV-cache pool at start-up and forbids later allocations, or code on a
 * latency-critical path where cudaMalloc / cudaFree may synchronise the
 * device, and that cannot hand the library a workspace either.
 *
 * Same arguments and results as paged_decode_attn, except that
 * params->workspace and params->workspace_bytes are ignored: the call's
 * whole workspace (the tensor-core kernel's counter header, its work-queue
 * order and FP8 Q operand images, and the split-KV partials) lives in a
 * fixed array of PDA_NO_ALLOC_WORKSPACE_BYTES compiled into the library,
 * which every device that loads the library holds until the process exits.
 * The call allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine), and never uses the library-owned buffer of paged_decode_attn.
 *
 * Limit: if paged_decode_attn_workspace_bytes(params) (the workspace of the
 * chosen or forced split count and kernel) is more than
 * PDA_NO_ALLOC_WORKSPACE_BYTES, the call returns PDA_ERR_WORKSPACE before
 * any device work.
 *
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.
 *
 * Sharing: all calls on a device use the same array, which keeps the last
 * call's contents. Nothing in it needs clearing by the caller (the
 * tensor-core kernel's prologue zeroes its counters on every call, and every
 * partial slot a call reads was written earlier in that call), but calls
 * that overlap on the GPU (on different streams) race on it: serialise them.
 */
#define PDA_NO_ALLOC_WORKSPACE_BYTES (16u * 1024u * 1024u)

PDA_API pda_status paged_decode_attn_no_alloc(const void* q, const void* k_pages,
                                              const void* v_pages,
                                              const int32_t* page_table,
                                              const int32_t* kv_lens,
                                              const pda_params* params, float* out,
                                              float* lse, pda_stream_t stream);

/* Bytes of workspace paged_decode_attn needs for these params with the
 * split count it would choose (0 for the CUDA-core kernel when it would not
 * split). SIZE_MAX if the params are invalid. The counterpart of
 * alloc_split_partials ("AstrAI commit log,
 * attn_paged_decode_split_kv_mma.cuh": split partials sized per call and
 * never cleared). params->max_kv_len, the host's bound on the sequence
 * lengths, takes the place of a separate length argument. */
PDA_API size_t paged_decode_attn_workspace_bytes(const pda_params* params);

/* The split count paged_decode_attn would use for these params on a device
 * with num_sms SMs (host-only; the heuristic of the split planner, the
 * counterpart of compute_num_splits in "AstrAI commit log,
 * attn_paged_decode_split_kv_mma.cuh", driven by batch x kv heads against
 * the SM count). Returns a value >= 1, or 0 if params are invalid. */
PDA_API int32_t pda_choose_num_splits(const pda_params* params, int32_t num_sms);

/*
 * LSE merge of split partials, the merge step on its own (merge_attn_states /
 * PagedPersistentMergeKernel):
 *   lse[r]    = m + ln sum_s exp(lse_parts[s, r] - m),  m = max_s lse_parts[s, r]
 *   out[r, :] = sum_s exp(lse_parts[s, r] - lse[r]) * o_parts[s, r, :]
 * A row whose every part has lse = -inf gets out = 0 and lse = -inf, and
 * o_parts of such parts are not read.
 *
 * o_parts    device fp32 [num_splits, rows, head_dim]
 * lse_parts  device fp32 [num_splits, rows]
 * out        device fp32 [rows, head_dim];  lse device fp32 [rows] or NULL
 * sinks      optional device fp32 [num_q_heads]: attention-sink logit of
 *            row r's head r % num_q_heads, one more part with lse = sink and
 *            o = 0 (rows laid out [..., num_q_heads]); NULL for none.
 * head_dim in {64, 128, 256}; num_splits >= 1; o_parts and out 16-byte
 * aligned, lse_parts, lse and sinks 4-byte aligned. This is also the
 * combine step of decode context parallel: the parts are the per-GPU states
 * of disjoint key shards.
 */
PDA_API pda_status pda_merge_states(const float* o_parts, const float* lse_parts,
                            int32_t num_splits, int64_t rows, int32_t head_dim,
                            float* out, float* lse, const float* sinks,
                            int32_t num_q_heads, pda_stream_t stream);

/* Parameters of paged_kv_append. */
typedef struct {
  int32_t batch;             /* B >= 0 */
  int32_t num_new;           /* new tokens per sequence, 1..64 */
  int32_t num_kv_heads;      /* Hkv >= 1 */
  int32_t head_dim;          /* D in {64, 128, 256} */
  int32_t page_size;         /* P, a power of two in [8, 256] */
  int32_t max_pages_per_seq; /* row stride of page_table */
  int32_t num_pages;         /* pages in each pool; page ids must be < this */
  int32_t kv_dtype;          /* pda_kv_dtype of the pools */
  float kv_scale;            /* FP8: code = e4m3(x / kv_scale); NVFP4: the per-tensor
                                scale of the block rule below (> 0) */
  void* k_scales;            /* NVFP4 only: device uint8 [num_pages, Hkv, P, D/16]
                                block-scale pools, written for the appended rows */
  void* v_scales;
} pda_append_params;

/*
 * Paged KV append, the KV-cache producer that runs before the decode call
 * ("sglang profiler skill, fuse-overlap catalog", "Fused FP8 quantize + paged
 * KV cache write" row): new row t of sequence b (t < num_new) is written at
 * logical position kv_lens[b] + t, i.e. page page_table[b][pos / P], slot
 * pos % P, for every kv head, in K and in V.
 *
 * k_new, v_new  device, bf16 [B, num_new, Hkv, D], contiguous, 16-byte aligned.
 * page_table    device, int32 [B, max_pages_per_seq]; the pages covering
 *               [kv_lens[b], kv_lens[b] + num_new) must already be assigned.
 * kv_lens       device, int32 [B]: lengths before the append. Read only: the
 *               caller advances them by num_new before the next decode call.
 * params        host, read during the call only.
 * k_pages, v_pages device pools [num_pages, Hkv, P, D] of bf16 or e4m3 codes
 *               (kv_dtype), 16-byte aligned. Only the appended slots are written.
 *
 * bf16 pools receive the bits unchanged. FP8 pools receive, per element, the
 * e4m3 code nearest to the fp32 quotient x / kv_scale (IEEE division), ties
 * to even, saturated to +-448 (NaN stays NaN): the encoding the decode call
 * inverts with the same kv_scale. NVFP4 pools receive, per block of 16
 * elements of a row ("b12x 0.30.0, Kernel inventory", BF16-to-FP4 TMA
 * quantization row: packed NVFP4 plus scale tiles; "sglang profiler skill,
 * fuse-overlap catalog", fused BF16 to FP4 quant + paged KV write row), all
 * in fp32 with nearest-even rounding and saturation: q = x / kv_scale,
 * block scale = e4m3(max |q| / 6), code = e2m1(q / block scale) (a block
 * whose scale is zero stores +0 codes); NaN inputs give unspecified codes.
 *
 * Errors: invalid params or pointers return before any device work
 * (PDA_ERR_INVALID_ARG / _UNSUPPORTED / _MISALIGNED). A position past
 * max_pages_per_seq * P, a negative kv_len or a page id out of range is not
 * written and records PDA_ERR_BAD_PAGE in the device error word.
 * Asynchronous on `stream`.
 */
PDA_API pda_status paged_kv_append(const void* k_new, const void* v_new,
                                   const int32_t* page_table, const int32_t* kv_lens,
                                   const pda_append_params* params, void* k_pages,
                                   void* v_pages, pda_stream_t stream);

/* Which split kernel paged_decode_attn would launch for these params
 * (host-only; the planner's choice between the two variants that "AstrAI
 * commit log, attn_paged_decode_split_kv_mma.cuh" describes: the scalar
 * variant and the tensor-core head-packing variant):
 *   PDA_KERNEL_SPLIT_TMA  tensor-core kernel (2D TMA tiles of 128 tokens,
 *                         tcgen05 MMAs with TMEM accumulators): head_dim 128
 *                         with bf16 or NVFP4 K/V and at most 8 packed rows
 *                         per kv head (G * q_len; NVFP4 tiles are decoded
 *                         exactly to f16 in shared memory), or FP8 K/V and
 *                         more than 8; any head_dim-128 case with
 *                         PDA_FLAG_TENSOR_CORES;
 *   PDA_KERNEL_SPLIT_FMA  CUDA-core kernel (warp-shuffle FMAs, cp.async.bulk
 *                         page copies): everything else, and every case with
 *                         PDA_FLAG_CUDA_CORES.
 * Returns -1 if the params are invalid. */
#define PDA_KERNEL_SPLIT_FMA 0
#define PDA_KERNEL_SPLIT_TMA 1
PDA_API int32_t pda_plan_kernel(const pda_params* params);

/*
 * Measurement helper, not part of the attention path: reads `bytes` bytes at
 * `buf` once with 128-bit streaming loads (4 CTAs of 512 threads per SM) and
 * XORs the words into *sink, so a caller can time the device's read-only
 * HBM bandwidth with the same events and in the same run as the attention
 * call. buf and bytes 16-byte aligned, sink 8-byte aligned device memory
 * (its value is meaningless). Asynchronous on `stream`.
 */
PDA_API pda_status pda_hbm_read_probe(const void* buf, size_t bytes, uint64_t* sink,
                                      pda_stream_t stream);

/* Human-readable name of a status. Never NULL. */
PDA_API const char* pda_status_string(pda_status status);

/* The pages have no counterpart to this entry point: it reports what the
 * kernels' in-bounds checks found (a debug read, the one call that
 * synchronises).
 * Synchronises `stream`, then reads and clears the current device's error
 * word: the first error a kernel recorded since the last read
 * (PDA_ERR_BAD_PAGE, PDA_ERR_TIMEOUT, or PDA_ERR_UNSUPPORTED if a kernel met
 * a launch condition it cannot handle), PDA_OK otherwise (PDA_ERR_CUDA if the
 * sync failed). */
PDA_API pda_status pda_last_device_error(pda_stream_t stream);

/* PDA_ABI_VERSION of the loaded library. */
PDA_API int32_t pda_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_DECODE_ATTN_H_ */
