// Split-KV paged decode kernel, CUDA-core (FMA) path for small packed-row
// counts (M = G * q_len rows per kv head, M_T <= 8 rows per CTA).
//
// Sources: "AstrAI commit log, attn_paged_decode_split_kv_mma.cuh" (scalar
// variant: page table resolved per position while loading the K/V tile;
// multi-stage copy pipeline keeping STAGES-1 tiles in flight; predicated
// partial tiles; split partials written without a memset), "b12x 0.30.0,
// Kernel inventory, Attention table, Paged attention row" (bf16 and
// FP8-E4M3 KV, sliding window, GQA, split-KV or direct output) and the same
// inventory's NVFP4 rows (float4_e2m1fn with E4M3 scales per 16 elements).
//
// B200 design:
//  * One CTA per (row tile, split, kv head, sequence). The CTA's key range is
//    dealt to its NW warps tile by tile (warp w takes tiles w, w+NW, ...).
//    Each warp owns a STAGES-deep ring of K/V tiles in shared memory, filled
//    by untiled bulk copies (one per K tile, one per V tile: a tile is TW
//    consecutive tokens of one page, a contiguous block of the HND pool)
//    that complete on the warp's own mbarriers. No CTA-wide barrier sits in
//    the main loop.
//  * Page ids for the warp's next 64 tiles live in registers (one per lane,
//    two batches), so the lookup latency never sits in front of a copy.
//    A page id outside [0, num_pages) is recorded as an error and replaced by
//    page 0, so no access ever leaves the pool.
//  * Lane layout: a token's D elements are split over LPT = D/8 lanes, 8
//    elements (one 16-byte bf16, 8-byte e4m3 or 4-byte NVFP4 load, plus the
//    block's e4m3 scale byte) per lane; TPI = 32/LPT
//    tokens are read per warp instruction (a warp reads 512 contiguous bytes
//    for bf16, conflict-free). Q sits in registers, pre-scaled by
//    scale*log2(e) (and kv_scale for FP8 / NVFP4), for the lane's 8 elements of each
//    of the M_T rows.
//  * Arithmetic runs on packed fp32 pairs (fma/mul.rn.f32x2: two FMAs per
//    issue slot); bf16, e4m3 and e2m1 (times its block scale, exact)
//    elements convert straight into pairs.
//  * Scores: 8*M_T partial dot products per lane per group of 8 tokens are
//    summed over the LPT lanes of a token with a reduce-scatter butterfly
//    (each step halves the values a lane carries), so a score costs about one
//    shuffle instead of log2(LPT). Each lane stores its partials in an order
//    permuted by its own lane bits (it walks its tokens and its Q rows XORed
//    with a lane mask), so that at every step all lanes keep the low half and
//    send the high half: no selects.
//  * Online softmax in fp32 with exp2; probabilities go through a small
//    per-warp shared buffer (stored as (p, p) pairs) to the P.V loop, which
//    keeps acc[M_T][8] fp32 per lane as pairs.
//  * Masking by select, never by multiplying: scores of invisible keys become
//    -inf; V of keys no row can see is zeroed before the FMA, so NaN bytes in
//    tail slots or outside the window never reach the output. Tiles fully
//    inside every row's visible range skip all mask work.
//  * End: the warps' (m, l, acc) are merged through shared memory; the CTA
//    writes out/lse directly (one split) or normalised partials (several).
#pragma once

#include "pda_device.cuh"

namespace pda {

// Split-arrival counters per (sequence, kv head, row tile): one for each
// softmax row group of the tensor-core kernel (at most four).
constexpr int kMergeCtrPerGroup = 4;

struct SplitArgs {
  const uint16_t* q;         // bf16 bits [B, Lq, Hq, D]
  const uint8_t* k_pages;    // pool bytes [num_pages, Hkv, P, D] (NVFP4: D/2)
  const uint8_t* v_pages;
  const uint8_t* k_scales;   // NVFP4: e4m3 block scales [num_pages, Hkv, P, D/16]
  const uint8_t* v_scales;
  long long sc_page_stride;  // NVFP4: bytes per page / per (page, head) block
  long long sc_head_stride;  //   of the scale pools
  const int32_t* page_table; // [B, max_pages]
  const int32_t* kv_lens;    // [B]
  float* out;                // [B, Lq, Hq, D]       (num_splits == 1)
  float* lse;                // [B, Lq, Hq] or null  (num_splits == 1)
  float* o_part;             // [S, B, Lq, Hq, D]    (num_splits > 1)
  float* lse_part;           // [S, B, Lq, Hq]
  int* err;                  // device error word
  int B, Lq, Hq, Hkv, G, M;
  int page_size, log2_page, max_pages, num_pages;
  int tile_shift;            // log2(page_size / TW): tiles per page
  int num_splits, row_tiles;
  int causal_offset, window;
  float qk_scale_log2;       // scale * log2(e) [* kv_scale for FP8 / NVFP4]
  float v_scale;             // 1, or kv_scale for FP8 / NVFP4
  long long page_stride;     // bytes per page of the code pool: Hkv * P * D * elt
  long long head_stride;     // bytes per (page, head) block: P * D * elt (NVFP4: elt 1/2)
  // persistent tensor-core kernel only (prepared by its prologue kernel,
  // which runs just before it on the same stream):
  int* sched;                // [0] next work item
  int* merge_ctr;            // [B * Hkv * row_tiles * kMergeCtrPerGroup] splits finished
                             // per (group, softmax row group)
  int header_words;          // ints from sched to the end of merge_ctr (zeroed first)
  int* order;                // [B] sequences, most visible tiles first: the queue order
  uint8_t* qops;             // FP8: Q operand image + row scales per (b, kvh, row tile)
  int num_items;             // B * Hkv * num_splits * row_tiles
  const float* sinks;        // [Hq] attention-sink logit per query head, or null
  int fused_merge;           // 1: the last split of a group merges it in-kernel
};

// KV: 0 bf16, 1 e4m3, 2 NVFP4 (e2m1 codes two per byte + an e4m3 scale per
// 16 elements; a stage then holds K codes, K scales, V codes, V scales).
template <int D, int KV, int MT, int TW, int NW, int STAGES>
struct FmaCfg {
  static constexpr int ELT = KV == 0 ? 2 : 1;  // bytes per element (KV 0, 1)
  static constexpr int CH = 8;             // elements per lane chunk
  static constexpr int LPT = D / CH;       // lanes per token
  static constexpr int TPI = 32 / LPT;     // tokens per warp instruction
  static constexpr int NTOK = TW / TPI;    // tokens per lane group per tile
  static constexpr int NV = NTOK * MT;     // partial scores per lane
  static constexpr int NVF = NV >= LPT ? NV / LPT : 1;  // after reduce-scatter
  // distinct rows among a lane's NVF slots, and the lowest xor distance
  // between lanes that hold the same rows (for row-wise max / sum)
  static constexpr int NFOLD = NVF > MT ? MT : NVF;
  static constexpr int RED_LO =
      NV >= LPT ? (NVF >= MT ? 1 : MT / NVF) : (LPT / NV) * MT;
  static constexpr int TILE_BYTES = KV == 2 ? TW * D / 2 : TW * D * ELT;  // K or V codes
  static constexpr int SC_BYTES = KV == 2 ? TW * D / 16 : 0;              // their block scales
  static constexpr int HALF_STAGE = TILE_BYTES + SC_BYTES;                // K (or V) part
  static constexpr int STAGE_BYTES = 2 * HALF_STAGE;
  static constexpr int PBUF_FLOATS = TW * MT * 2;  // (p, p) pairs
  static constexpr int WARP_SMEM_RAW =
      STAGES * STAGE_BYTES + 32 /*mbarriers*/ + PBUF_FLOATS * 4 + 64 /*alpha pairs*/;
  // lane-mask permutation of the reduce-scatter (see reduce_scatter)
  static constexpr int LOG_LPT = LPT == 8 ? 3 : (LPT == 16 ? 4 : 5);
  static constexpr int LOG_NV = NV == 1 ? 0 : NV == 2 ? 1 : NV == 4 ? 2 : NV == 8 ? 3 :
                                NV == 16 ? 4 : NV == 32 ? 5 : NV == 64 ? 6 : 7;
  static constexpr int LOG_MT = MT == 1 ? 0 : MT == 2 ? 1 : MT == 4 ? 2 : 3;
  static constexpr int RS_STEPS = LOG_NV < LOG_LPT ? LOG_NV : LOG_LPT;
  static constexpr int WARP_SMEM = (WARP_SMEM_RAW + 127) / 128 * 128;
  static constexpr int MERGE_SMEM = (2 * NW * MT + NW * MT * D) * 4;
  static constexpr int SMEM =
      NW * WARP_SMEM > MERGE_SMEM ? NW * WARP_SMEM : MERGE_SMEM;
  static_assert(D % 64 == 0 && D <= 256, "head_dim");
  static_assert(TW % TPI == 0 && NTOK >= 1, "tile");
  static_assert(STAGES <= 4, "mbarrier area holds 4");
  static_assert(TILE_BYTES % 16 == 0 && SC_BYTES % 16 == 0, "bulk copy size");
  static_assert(KV != 2 || D % 16 == 0, "NVFP4 blocks of 16 elements");
};

// Visible key range [lo, hi) of a query row at index i (reading of the
// causal_offset / window conventions in the public header).
__device__ __forceinline__ void row_range(const SplitArgs& a, int L, int i,
                                          int& lo, int& hi) {
  long long pos;
  if (a.causal_offset >= 0)
    pos = (long long)a.causal_offset + i;
  else if (a.causal_offset == -2)
    pos = (long long)L - a.Lq + i;
  else
    pos = (long long)L - 1;
  long long h = a.causal_offset != -1 ? pos + 1 : (long long)L;
  h = h < 0 ? 0 : (h > L ? L : h);
  long long l = a.window > 0 ? pos - a.window + 1 : 0;
  l = l < 0 ? 0 : (l > L ? L : l);
  lo = (int)l;
  hi = (int)h;
}

// Butterfly reduce-scatter of N values over the lanes whose ids differ in the
// bits of O, O/2, ..., 1. At each step every lane keeps v[0 .. N/2) and adds
// the partner's v[N/2 .. N): the caller has stored its values permuted by its
// lane mask, so that the low half of every lane is the half it must keep.
// After log2(N) steps each lane holds one value summed over 2^steps lanes; the
// remaining steps are plain butterflies. Values end in v[0 .. N/lanes).
template <int N, int O>
__device__ __forceinline__ void reduce_scatter(float* v) {
  if constexpr (O >= 1) {
    if constexpr (N > 1) {
#pragma unroll
      for (int i = 0; i < N / 2; ++i) v[i] += __shfl_xor_sync(0xFFFFFFFFu, v[i + N / 2], O);
      reduce_scatter<N / 2, O / 2>(v);
    } else {
      v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], O);
      reduce_scatter<1, O / 2>(v);
    }
  }
}

// NVFP4: 8 consecutive elements of one token (4 code bytes) and the e4m3
// scale of their block -> 4 fp32 pairs (exact: e2m1 * e4m3 has 5
// significant bits).
__device__ __forceinline__ void load_chunk_nvfp4(const uint8_t* codes, const uint8_t* scale,
                                                 f32x2 (&f)[4]) {
  const uint32_t c = *reinterpret_cast<const uint32_t*>(codes);
  const float sc = e4m3_code_to_f32(*scale);
  const f32x2 s2 = f2_pack(sc, sc);
#pragma unroll
  for (int k = 0; k < 4; ++k) f[k] = f2_mul(e2m1x2_to_f2(c >> (8 * k)), s2);
}

// 8 consecutive K or V elements of one token -> 4 fp32 pairs.
template <int KV>
__device__ __forceinline__ void load_chunk2(const uint8_t* p, f32x2 (&f)[4]) {
  if constexpr (KV == 0) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    f[0] = bf16x2_to_f2(u.x);
    f[1] = bf16x2_to_f2(u.y);
    f[2] = bf16x2_to_f2(u.z);
    f[3] = bf16x2_to_f2(u.w);
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    f[0] = e4m3x2_to_f2(u.x);
    f[1] = e4m3x2_to_f2(u.x >> 16);
    f[2] = e4m3x2_to_f2(u.y);
    f[3] = e4m3x2_to_f2(u.y >> 16);
  }
}

template <int D, int KV, int MT, int TW, int NW, int STAGES>
__global__ void __launch_bounds__(NW * 32, 1)
    split_fma_kernel(const SplitArgs a) {
  using C = FmaCfg<D, KV, MT, TW, NW, STAGES>;
  constexpr unsigned FULL = 0xFFFFFFFFu;
  extern __shared__ __align__(128) uint8_t smem[];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int rt = blockIdx.x;
  const int split = blockIdx.y % a.num_splits;
  const int kvh = blockIdx.y / a.num_splits;
  const int b = blockIdx.z;

  uint8_t* wbase = smem + warp * C::WARP_SMEM;
  uint64_t* mbar = reinterpret_cast<uint64_t*>(wbase + STAGES * C::STAGE_BYTES);
  float* pbuf = reinterpret_cast<float*>(wbase + STAGES * C::STAGE_BYTES + 32);
  float* abuf = pbuf + C::PBUF_FLOATS;

  // ---- key range of this CTA -------------------------------------------
  int L = __ldg(a.kv_lens + b);
  const int Lmax = a.max_pages << a.log2_page;
  if (L < 0 || L > Lmax) {
    if (threadIdx.x == 0) record_error_at(a.err, kErrBadPage);
    L = L < 0 ? 0 : Lmax;
  }
  const int R0 = rt * MT;
  const int Rlast = min(a.M, R0 + MT) - 1;
  int lo_u, hi_u, lo_x, hi_x;
  row_range(a, L, R0 / a.G, lo_u, hi_x);     // first row: union lo, intersection hi
  row_range(a, L, Rlast / a.G, lo_x, hi_u);  // last row: intersection lo, union hi
  const int k_begin = lo_u / TW;
  const int k_end = hi_u > lo_u ? (hi_u + TW - 1) / TW : k_begin;
  const int n_all = k_end - k_begin;
  const int chunk = (n_all + a.num_splits - 1) / a.num_splits;
  const int c0 = min(n_all, split * chunk);
  const int c1 = min(n_all, c0 + chunk);
  const int cta_tiles = c1 - c0;
  const int my_tiles = cta_tiles > warp ? (cta_tiles - warp + NW - 1) / NW : 0;
  const int kbase = k_begin + c0 + warp;  // absolute tile index of my tile 0

  const int tile_shift = a.tile_shift;
  const int tile_mask = (1 << tile_shift) - 1;
  const int32_t* pt_row = a.page_table + (long long)b * a.max_pages;
  const uint8_t* kbase_ptr = a.k_pages + (long long)kvh * a.head_stride;
  const uint8_t* vbase_ptr = a.v_pages + (long long)kvh * a.head_stride;
  const uint8_t* ksc_ptr = KV == 2 ? a.k_scales + (long long)kvh * a.sc_head_stride : nullptr;
  const uint8_t* vsc_ptr = KV == 2 ? a.v_scales + (long long)kvh * a.sc_head_stride : nullptr;

  // ---- barriers and page-id prefetch -------------------------------------
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < STAGES; ++s) mbar_init(&mbar[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  auto load_pid = [&](int n) -> int {
    if (n >= my_tiles) return 0;
    int pid = __ldg(pt_row + ((kbase + n * NW) >> tile_shift));
    if ((unsigned)pid >= (unsigned)a.num_pages) {
      record_error_at(a.err, kErrBadPage);
      pid = 0;
    }
    return pid;
  };
  int pid_cur = load_pid(lane);
  int pid_nxt = load_pid(32 + lane);
  int pid_batch = 0;

  auto issue = [&](int n) {  // warp-uniform
    const int nb = n >> 5;
    if (nb != pid_batch) {
      pid_cur = pid_nxt;
      pid_nxt = load_pid((nb + 1) * 32 + lane);
      pid_batch = nb;
    }
    const int pid = __shfl_sync(FULL, pid_cur, n & 31);
    if (lane == 0) {
      const int s = n % STAGES;
      const long long tip = (long long)((kbase + n * NW) & tile_mask);  // tile in page
      const long long off = (long long)pid * a.page_stride + tip * C::TILE_BYTES;
      uint8_t* dst = wbase + s * C::STAGE_BYTES;
      mbar_arrive_expect_tx(&mbar[s], C::STAGE_BYTES);
      bulk_g2s(dst, kbase_ptr + off, C::TILE_BYTES, &mbar[s]);
      bulk_g2s(dst + C::HALF_STAGE, vbase_ptr + off, C::TILE_BYTES, &mbar[s]);
      if constexpr (KV == 2) {
        const long long soff = (long long)pid * a.sc_page_stride + tip * C::SC_BYTES;
        bulk_g2s(dst + C::TILE_BYTES, ksc_ptr + soff, C::SC_BYTES, &mbar[s]);
        bulk_g2s(dst + C::HALF_STAGE + C::TILE_BYTES, vsc_ptr + soff, C::SC_BYTES, &mbar[s]);
      }
    }
  };

  const int n_pro = my_tiles < STAGES ? my_tiles : STAGES;
  for (int n = 0; n < n_pro; ++n) issue(n);

  // ---- lane mask of the select-free reduce-scatter ------------------------
  // The top RS_STEPS bits of the lane's chunk index c, placed as the top
  // bits of the NV-value index: the lane stores value v at position
  // v ^ vmask, i.e. walks tokens it ^ vmask_it and Q rows r ^ vmask_r.
  const int grp = lane / C::LPT;
  const int c = lane % C::LPT;
  const int d0 = c * C::CH;
  const int vmask = (c >> (C::LOG_LPT - C::RS_STEPS)) << (C::LOG_NV - C::RS_STEPS);
  const int vmask_r = vmask & (MT - 1);
  const int vmask_it = vmask >> C::LOG_MT;

  // ---- Q fragment (rows permuted by vmask_r), as pairs ---------------------
  f32x2 qf[MT][4];
  {
    const f32x2 sc = f2_pack(a.qk_scale_log2, a.qk_scale_log2);
#pragma unroll
    for (int r = 0; r < MT; ++r) {
      const int R = R0 + (r ^ vmask_r);
      if (R < a.M) {
        const int i = R / a.G, h = kvh * a.G + R % a.G;
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(
            a.q + ((long long)(b * a.Lq + i) * a.Hq + h) * D + d0));
        qf[r][0] = f2_mul(bf16x2_to_f2(u.x), sc);
        qf[r][1] = f2_mul(bf16x2_to_f2(u.y), sc);
        qf[r][2] = f2_mul(bf16x2_to_f2(u.z), sc);
        qf[r][3] = f2_mul(bf16x2_to_f2(u.w), sc);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) qf[r][j] = 0ull;
      }
    }
  }

  // ---- slots this lane holds after the reduce-scatter --------------------
  // slot i holds value v = vmask | i: token (v / MT) * TPI + grp, row v % MT
  int slot_tok[C::NVF], slot_row[C::NVF], slot_lo[C::NVF], slot_hi[C::NVF];
#pragma unroll
  for (int i = 0; i < C::NVF; ++i) {
    const int v = vmask | i;
    slot_tok[i] = (v / MT) * C::TPI + grp;
    slot_row[i] = v % MT;
    const int R = R0 + slot_row[i];
    if (R < a.M) {
      row_range(a, L, R / a.G, slot_lo[i], slot_hi[i]);
    } else {
      slot_lo[i] = 0;
      slot_hi[i] = 0;
    }
  }

  float m_slot[C::NVF], l_slot[C::NVF];
#pragma unroll
  for (int i = 0; i < C::NVF; ++i) {
    m_slot[i] = -INFINITY;
    l_slot[i] = 0.f;
  }
  f32x2 acc[MT][4];
#pragma unroll
  for (int r = 0; r < MT; ++r)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[r][j] = 0ull;  // (+0.f, +0.f)

  int n_fail = -1;  // tile whose copy never landed (bounded wait expired)

  // ---- main loop over this warp's tiles -----------------------------------
  for (int n = 0; n < my_tiles; ++n) {
    const int s = n % STAGES;
    if (!mbar_wait(&mbar[s], (n / STAGES) & 1, a.err)) {
      n_fail = n;
      break;
    }
    const uint8_t* kt = wbase + s * C::STAGE_BYTES;
    const uint8_t* vt = kt + C::HALF_STAGE;
    // 8 elements of token `tok` from this lane's chunk, as 4 fp32 pairs
    auto load_tok = [&](const uint8_t* tile, int tok, f32x2 (&f)[4]) {
      if constexpr (KV == 2)
        load_chunk_nvfp4(tile + (tok * D + d0) / 2, tile + C::TILE_BYTES + (tok * D + d0) / 16, f);
      else
        load_chunk2<KV>(tile + (tok * D + d0) * C::ELT, f);
    };
    const int t0 = (kbase + n * NW) * TW;
    const bool clean = t0 >= lo_x && t0 + TW <= hi_x;

    // S = Q K^T, partial over this lane's 8 elements, stored permuted
    float part[C::NV];
#pragma unroll
    for (int it = 0; it < C::NTOK; ++it) {
      const int tok = (it ^ vmask_it) * C::TPI + grp;
      f32x2 kf[4];
      load_tok(kt, tok, kf);
#pragma unroll
      for (int r = 0; r < MT; ++r) {
        f32x2 s2 = f2_mul(qf[r][0], kf[0]);
        s2 = f2_fma(qf[r][1], kf[1], s2);
        s2 = f2_fma(qf[r][2], kf[2], s2);
        s2 = f2_fma(qf[r][3], kf[3], s2);
        float lo, hi;
        f2_unpack(s2, lo, hi);
        part[it * MT + r] = lo + hi;
      }
    }
    reduce_scatter<C::NV, C::LPT / 2>(part);
    float sv[C::NVF];
#pragma unroll
    for (int i = 0; i < C::NVF; ++i) sv[i] = part[i];
    if (!clean) {
#pragma unroll
      for (int i = 0; i < C::NVF; ++i) {
        const int j = t0 + slot_tok[i];
        if (!(j >= slot_lo[i] && j < slot_hi[i])) sv[i] = -INFINITY;
      }
    }

    // tile row max over lanes holding the same rows
    float rmax[C::NFOLD];
#pragma unroll
    for (int f = 0; f < C::NFOLD; ++f) {
      rmax[f] = sv[f];
#pragma unroll
      for (int i = f + C::NFOLD; i < C::NVF; i += C::NFOLD) rmax[f] = fmaxf(rmax[f], sv[i]);
    }
#pragma unroll
    for (int o = C::RED_LO; o < 32; o <<= 1)
#pragma unroll
      for (int f = 0; f < C::NFOLD; ++f)
        rmax[f] = fmaxf(rmax[f], __shfl_xor_sync(FULL, rmax[f], o));

    // online softmax update of the slots; (p, p) and (alpha, alpha) pairs to
    // shared memory
#pragma unroll
    for (int i = 0; i < C::NVF; ++i) {
      const float m_new = fmaxf(m_slot[i], rmax[i % C::NFOLD]);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = fast_exp2(m_slot[i] - m_use);
      const float p = fast_exp2(sv[i] - m_use);
      l_slot[i] = l_slot[i] * alpha + p;
      m_slot[i] = m_new;
      reinterpret_cast<float2*>(pbuf)[slot_tok[i] * MT + slot_row[i]] = make_float2(p, p);
      if (i < C::NFOLD) reinterpret_cast<float2*>(abuf)[slot_row[i]] = make_float2(alpha, alpha);
    }
    __syncwarp();

    {
      f32x2 al[MT];
      bool rescale = false;
#pragma unroll
      for (int r = 0; r < MT; ++r) {
        const float2 x = reinterpret_cast<const float2*>(abuf)[r];
        al[r] = f2_pack(x.x, x.y);
        rescale |= x.x != 1.f;
      }
      if (rescale) {
#pragma unroll
        for (int r = 0; r < MT; ++r)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[r][j] = f2_mul(acc[r][j], al[r]);
      }
    }

    // O += P V
#pragma unroll
    for (int it = 0; it < C::NTOK; ++it) {
      const int tok = it * C::TPI + grp;
      f32x2 pr[MT];
      const float4* pp = reinterpret_cast<const float4*>(pbuf + tok * MT * 2);
      if constexpr (MT >= 2) {
#pragma unroll
        for (int r = 0; r < MT; r += 2) {
          const float4 p4 = pp[r / 2];
          pr[r] = f2_pack(p4.x, p4.y);
          pr[r + 1] = f2_pack(p4.z, p4.w);
        }
      } else {
        const float2 p2 = reinterpret_cast<const float2*>(pbuf)[tok];
        pr[0] = f2_pack(p2.x, p2.y);
      }
      f32x2 vf[4];
      load_tok(vt, tok, vf);
      if (!clean) {
        const int j = t0 + tok;
        if (j < lo_u || j >= hi_u) {
#pragma unroll
          for (int e = 0; e < 4; ++e) vf[e] = 0ull;
        }
      }
#pragma unroll
      for (int r = 0; r < MT; ++r)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[r][e] = f2_fma(pr[r], vf[e], acc[r][e]);
    }
    __syncwarp();
    if (n + STAGES < my_tiles) {
      if (lane == 0) fence_proxy_async_smem();
      issue(n + STAGES);
    }
  }

  if (n_fail >= 0) {
    // Copies n_fail .. n_fail+STAGES-1 may still be in flight into this
    // warp's ring: give each a short bounded wait before the memory is
    // reused, so no copy lands in shared memory after the CTA has moved on.
    const int issued = min(my_tiles, n_fail + STAGES);
    for (int n = n_fail + 1; n < issued; ++n)
      mbar_wait(&mbar[n % STAGES], (n / STAGES) & 1, a.err, kWaitTimeoutCycles / 8);
  }

  pdl_launch_dependents();

  // ---- combine lane groups and rows inside the warp -----------------------
  float accf[MT][8];
#pragma unroll
  for (int r = 0; r < MT; ++r)
#pragma unroll
    for (int j = 0; j < 4; ++j) f2_unpack(acc[r][j], accf[r][2 * j], accf[r][2 * j + 1]);
#pragma unroll
  for (int o = C::LPT; o < 32; o <<= 1)
#pragma unroll
    for (int r = 0; r < MT; ++r)
#pragma unroll
      for (int e = 0; e < 8; ++e) accf[r][e] += __shfl_xor_sync(FULL, accf[r][e], o);
  float lsum[C::NFOLD];
#pragma unroll
  for (int f = 0; f < C::NFOLD; ++f) {
    lsum[f] = l_slot[f];
#pragma unroll
    for (int i = f + C::NFOLD; i < C::NVF; i += C::NFOLD) lsum[f] += l_slot[i];
  }
#pragma unroll
  for (int o = C::RED_LO; o < 32; o <<= 1)
#pragma unroll
    for (int f = 0; f < C::NFOLD; ++f) lsum[f] += __shfl_xor_sync(FULL, lsum[f], o);

  // ---- merge the warps through shared memory -----------------------------
  __syncthreads();  // every warp has drained its ring; stage memory is free
  float* mrow = reinterpret_cast<float*>(smem);
  float* lrow = mrow + NW * MT;
  float* accs = lrow + NW * MT;
#pragma unroll
  for (int f = 0; f < C::NFOLD; ++f) {
    mrow[warp * MT + slot_row[f]] = m_slot[f];
    lrow[warp * MT + slot_row[f]] = lsum[f];
  }
  if (grp == 0) {
#pragma unroll
    for (int r = 0; r < MT; ++r) {
      float4* dst = reinterpret_cast<float4*>(accs + (warp * MT + r) * D + d0);
      dst[0] = make_float4(accf[r][0], accf[r][1], accf[r][2], accf[r][3]);
      dst[1] = make_float4(accf[r][4], accf[r][5], accf[r][6], accf[r][7]);
    }
  }
  __syncthreads();

  const long long rows_total = (long long)a.B * a.Lq * a.Hq;
  for (int idx = threadIdx.x; idx < MT * (D / 4); idx += NW * 32) {
    const int r = idx / (D / 4);
    const int d = (idx % (D / 4)) * 4;
    const int R = R0 + r;
    if (R >= a.M) continue;
    float mstar = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) mstar = fmaxf(mstar, mrow[w * MT + r]);
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    float lt = 0.f;
    if (mstar != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float wt = fast_exp2(mrow[w * MT + r] - mstar);
        lt += wt * lrow[w * MT + r];
        const float4 x = *reinterpret_cast<const float4*>(accs + (w * MT + r) * D + d);
        o.x += wt * x.x; o.y += wt * x.y; o.z += wt * x.z; o.w += wt * x.w;
      }
    }
    const int i = R / a.G, h = kvh * a.G + R % a.G;
    // attention sink of head h (one split only; with splits the merge adds
    // it): one more exp2(sink) term in the denominator, no value
    const float sink = a.num_splits == 1 && a.sinks ? __ldg(a.sinks + h) : -INFINITY;
    float res_lse = -INFINITY;
    if (lt > 0.f) {
      float mref = mstar, l2 = lt, scl = 1.f;
      if (sink != -INFINITY) {
        const float sl = sink * 1.4426950408889634f;
        mref = fmaxf(mstar, sl);
        scl = fast_exp2(mstar - mref);
        l2 = fmaf(lt, scl, fast_exp2(sl - mref));
      }
      const float inv = a.v_scale * scl / l2;
      o.x *= inv; o.y *= inv; o.z *= inv; o.w *= inv;
      res_lse = (mref + log2f(l2)) * 0.69314718055994531f;
    } else {
      o = make_float4(0.f, 0.f, 0.f, 0.f);
      res_lse = sink;  // no visible key: the sink alone (-inf without one)
    }
    const long long row = (long long)(b * a.Lq + i) * a.Hq + h;
    if (a.num_splits == 1) {
      *reinterpret_cast<float4*>(a.out + row * D + d) = o;
      if (d == 0 && a.lse) a.lse[row] = res_lse;
    } else {
      const long long prow = (long long)split * rows_total + row;
      *reinterpret_cast<float4*>(a.o_part + prow * D + d) = o;
      if (d == 0) a.lse_part[prow] = res_lse;
    }
  }
}

// Host-side launcher for one head_dim, defined in split_d{64,128,256}.cu.
// Returns cudaErrorNotSupported if no variant matches.
cudaError_t launch_split_fma(int D, int kv, int mt, int tw, const SplitArgs& a,
                             dim3 grid, cudaStream_t stream);

}  // namespace pda
