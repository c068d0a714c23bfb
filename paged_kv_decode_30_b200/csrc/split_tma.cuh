// Split-KV paged decode on the 5th-generation tensor cores with TMA-fed
// operands (tcgen05.mma + cp.async.bulk.tensor, 128B swizzle), head_dim 128,
// as a persistent kernel with a dynamic work queue and a fused split merge.
//
// Sources: "b12x 0.30.0, Kernel inventory, Attention table, Paged attention
// row" (bf16 and FP8-E4M3 KV, decode/verify rows, sliding window, split-KV or
// direct output, persistent merge) and "AstrAI commit log,
// attn_paged_decode_split_kv_mma.cuh" (tensor-core GQA head packing,
// multi-stage copy pipeline, predicated partial tiles, split-KV partials
// combined by log-sum-exp).
//
// Work item: the packed rows (NT of them) of one (sequence, kv head, split,
// row tile); a CTA runs items one after another, a 128-token tile at a time
// (the MMA M dimension): S^T = K Q^T, then O^T = V^T P^T. One CTA per SM;
// the grid is min(items, SMs) and items come from an atomic counter, in the
// order a prologue kernel sets (longest sequences first; it also zeroes the
// counters and writes the FP8 Q operands), so SMs that finish short items
// take the next one at once and the CTAs finish close together.
//  * warp 7 (scheduler): draws items, computes their key ranges and the page
//    ids of their first tiles into a 4-deep descriptor ring, and writes each
//    item's Q operand (bf16: a swizzled copy; FP8: one bulk copy of the
//    prologue's image) and per-row state, one item ahead of the MMAs.
//  * warp 0 (producer): TMA loads of each page segment of the K and V tiles
//    into a STAGES-deep ring in the canonical 128B-swizzled UMMA layout (one
//    tensor map per pool: rows = (page, kv head, token), 128 elements per
//    row); later page ids of an item arrive by cp.async ahead of use.
//  * warps 1 and 2 (MMA): warp 1 allocates TMEM and issues the S^T MMAs,
//    warp 2 the O^T MMAs, each from one lane as soon as their inputs are
//    ready; completion is signalled by tcgen05.commit.
//      bf16 K/V: S^T with kind::f16 (bf16) straight from the K stage;
//        O^T with kind::f16 (bf16), A = V^T straight from the V stage
//        (MN-major), B = P^T split into bf16 hi + lo rows (N = 16).
//      FP8 K/V: S^T with kind::f8f6f4 straight from the e4m3 K stage, B =
//        [Q_hi; Q_lo], an exact two-term e4m3 split of each bf16 q row
//        scaled by a power of two; O^T with kind::f8f6f4 straight from the
//        e4m3 V stage (MN-major), B = P^T as two e4m3 terms [P_hi; 16 P_lo];
//        and the row sums of P^T (the normaliser) as the same B against a
//        tile of e4m3 ones.
//  * warps 3-6 (and, FP8, 8-19 by item rows: groups of four warps with 8
//    rows each) (softmax): thread i = TMEM lane i = token i of S^T and
//    head-dim element i of O^T. p = exp2(s * c - m) in fp32 with a lazily
//    moved running max; P^T to shared memory. O^T accumulates in TMEM over
//    the item's tiles; a tile that moves the max rescales it in place first.
//    On tiles with keys that no row may see they also zero those keys' V
//    rows in the stage, so NaN bytes never meet a zero weight in the MMA.
//    An item's epilogue (normalise, store O and the LSE, or the split's
//    partials; with the fused merge, the split that arrives last for its
//    rows merges them all) runs after the next item's first tile.
//  * NVFP4 K/V: the producer bulk-copies raw tiles (e2m1 codes and e4m3
//    block scales) into a ring of their own, and warps 8-11 (converters)
//    decode them exactly into f16 tiles in the stages' layout; the MMAs then
//    run kind::f16 with f16 operands (q as f16 of q * 2^e per row).
//  * Every wait is bounded; group exits go through bar.red.and.
#pragma once

#include <cuda.h>

#include "pda_device.cuh"
#include "split_fma.cuh"  // SplitArgs, row_range
#include "tcgen05.cuh"    // descriptors, MMA issue, TMEM loads, barriers

namespace pda {

// One work item as the scheduler publishes it (shared memory).
template <int PA>
struct ItemDesc {
  int b, kvh, split, rt;   // b < 0: no more items
  int L, kfirst, ntiles;   // kv length, first tile, tile count
  int lo_u, hi_u;          // union of the rows' visible key ranges
  int lo_x, hi_x;          // intersection of the rows' visible key ranges
  int pad[5];
  int pids[PA][16];        // page ids of the item's first PA tiles (segment = page)
};

// QN (FP8 only): "native FP8 QK", Q enters the MMA as one e4m3 term per
// element (q * 2^e rounded to nearest even, per-row power-of-two 2^e)
// instead of the exact two-term split, so S^T has NT columns, not 2 NT.
// KV: 0 bf16, 1 e4m3, 2 NVFP4. NVFP4 tiles arrive raw (codes and block
// scales, by bulk copies) and converter warps decode them exactly into f16
// tiles laid out as the TMA writes bf16 ones, so from the stages on the
// NVFP4 path is the 16-bit path with f16 operands.
template <int KV, int NT, bool QN = false>
struct TmaCfg {
  static constexpr bool NV = KV == 2;
  static constexpr bool BF16 = KV == 0 || NV;  // 16-bit operands (bf16; f16 for NVFP4)
  static constexpr bool QN_ = QN;
  static constexpr int D = 128;
  static constexpr int TILE = 128;
  static constexpr int ELT = BF16 ? 2 : 1;
  static constexpr int N1 = BF16 ? 16 : (QN ? NT : 2 * NT);  // S^T columns
  // O^T columns: bf16, the P_hi and P_lo rows (N = 16); FP8, two e4m3 terms
  // per weight, P_hi and 16 P_lo, summed as O_hi + O_lo / 16. FP8 columns
  // (and S^T columns with the two-term Q) go by row group: group k owns
  // columns 16k .. 16k + 7 (hi term of rows 8k .. 8k + 7) and 16k + 8 ..
  // 16k + 15 (lo term), so a thread reads its rows' terms in one load.
  static constexpr int N2 = BF16 ? 16 : 2 * NT;
  static constexpr int STAGES = NV ? 2 : (BF16 ? 3 : 5);
  // NVFP4: a ring of raw tiles, each K codes, K block scales, V codes and V
  // scales of 128 tokens, that the converter warps decode into the stages
  static constexpr int RAW_STAGES = NV ? 3 : 0;
  static constexpr int RAW_C = TILE * D / 2;   // e2m1 codes of one K (or V) tile
  static constexpr int RAW_S = TILE * D / 16;  // their e4m3 block scales
  static constexpr int RAW_STAGE = 2 * (RAW_C + RAW_S);
  static constexpr int CONV0 = 8, CONV_WARPS = NV ? 4 : 0;  // converter warps 8-11
  static constexpr int KT = TILE * D * ELT;      // bytes of one K (or V) tile
  static constexpr int STAGE = 2 * KT;           // K then V
  static constexpr int HALF = TILE * 128;        // one 128-byte column of SW128 atoms
  static constexpr int Q_ROWS = N1;
  static constexpr int Q_BYTES = Q_ROWS * D * (BF16 ? 2 : 1);
  static constexpr int Q_HALF = (Q_ROWS / 8) * 1024;  // bf16: 64-element half of each row
  static constexpr int Q_BUF = ((Q_BYTES + 1023) / 1024) * 1024;  // one of two Q buffers
  // FP8: the prologue kernel's Q operand image of one (b, kv head, row tile)
  // in global memory: Q_BYTES as the MMA reads them, then 32 row scales
  static constexpr int QOP = Q_BYTES + 128;
  static constexpr int P_ROW = N2 * ELT;               // bytes per token row of P^T
  static constexpr int P_SBO = 8 * P_ROW;
  static constexpr int P_BYTES = (TILE / 8) * P_SBO;
  static constexpr uint32_t P_SWIZZLE = P_ROW == 64 ? 4u : 6u;  // SW64 / SW32
  // warp roles. FP8 items have 16 or 32 rows: SOFT_H groups of four
  // softmax warps (warps 3-6, then 8-11, 12-15, 16-19) take 8 rows each, so
  // each SM sub-partition interleaves SOFT_H softmax warps.
  static constexpr int PROD = 0, S_MMA = 1, O_MMA = 2, SOFT0 = 3, SCHED = 7, SOFTX = 8;
  static constexpr int SOFT_H = BF16 ? 1 : NT / 8;  // row groups
  static constexpr int RH = NT / SOFT_H;             // rows per softmax thread
  static constexpr int SOFT_THREADS = 128 * SOFT_H;
  static constexpr int WARPS = 8 + 4 * (SOFT_H - 1) + CONV_WARPS;
  static constexpr int THREADS = WARPS * 32;
  // work-queue depths
  static constexpr int DSLOTS = 4;                 // item descriptors in flight
  // Items are drawn while fewer than AHEAD_TILES tiles of drawn items are
  // left for the softmax warps: enough lead to hide an item's set-up, little
  // enough that no CTA sits on queued work when the queue runs dry.
  static constexpr int AHEAD_TILES = 2 * STAGES;
  static constexpr int PID_SLOTS = 8, PID_AHEAD = 4;
  using Desc = ItemDesc<PID_AHEAD>;
  // per-item softmax state, double buffered by item parity
  static constexpr int SL_ROWS = 0;                // int64 output row per packed row (-1 pad)
  static constexpr int SL_RANGE = SL_ROWS + 32 * 8;   // int2 visible key range per row
  static constexpr int SL_CS = SL_RANGE + 32 * 8;     // score scale (log2 domain) per row
  static constexpr int SL_CSM = SL_CS + 32 * 4;       // {score scale, -m} per row
  static constexpr int SL_THR = SL_CSM + 32 * 8;      // lazy-rescale threshold per row
  static constexpr int SL_MRAW = SL_THR + 32 * 4;     // running max per row (-inf at start)
  static constexpr int SL_SINK = SL_MRAW + 32 * 4;    // attention-sink logit per row (-inf: none)
  static constexpr int SLOT = SL_SINK + 32 * 4;
  // shared memory map (1024-aligned where swizzled)
  static constexpr int OFF_STAGE = 0;
  static constexpr int OFF_RAW = OFF_STAGE + STAGES * STAGE;
  static constexpr int OFF_Q = OFF_RAW + RAW_STAGES * RAW_STAGE;
  static constexpr int OFF_P = OFF_Q + 2 * Q_BUF;
  static constexpr int P_BUF = ((P_BYTES + 1023) / 1024) * 1024;
  // FP8: a 32-token x 128 tile of e4m3 ones, the A operand of the MMAs that
  // sum P^T per row into TMEM (the softmax normaliser)
  static constexpr int ONES = BF16 ? 0 : 32 * 128;
  static constexpr int OFF_ONES = OFF_P + 2 * P_BUF;
  static constexpr int OFF_WMAX = OFF_ONES + ONES;  // [4 warps][32 rows]
  static constexpr int OFF_ALPHA = OFF_WMAX + 4 * 32 * 4;
  static constexpr int OFF_LRED = OFF_ALPHA + 2 * 32 * 4;
  static constexpr int OFF_INV = OFF_LRED + 4 * 32 * 4;  // v_scale / l per row
  static constexpr int OFF_SLOTS = OFF_INV + 32 * 4;
  static constexpr int OFF_DESC = OFF_SLOTS + 2 * SLOT;
  static constexpr int OFF_PIDS = OFF_DESC + DSLOTS * (int)sizeof(Desc);
  static constexpr int OFF_BAR = OFF_PIDS + PID_SLOTS * 16 * 4;
  // full[S], empty[S], s_full[2], p_ready[2], o_full[2], o_free[2],
  // desc_full[4], desc_free[4], q_ready[2], st_free[2], q_free[2],
  // NVFP4: raw_full[R], raw_empty[R], k_full[S]
  static constexpr int NUM_BARS = 2 * STAGES + 8 + 2 * DSLOTS + 6 + 2 * RAW_STAGES + (NV ? STAGES : 0);
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + NUM_BARS * 8;
  // [0] abort, [1] tiles done, [4 + k] merge flag of row group k
  static constexpr int OFF_FLAGS = OFF_TMEM_SLOT + 8;
  static constexpr int SMEM = OFF_FLAGS + 32;
  static constexpr int SMEM_ALLOC = SMEM + 1024;  // slack for the 1024-byte alignment check
  // S^T and O^T regions (two each), then, FP8, two row-sum regions
  static constexpr int COL_S = 0, COL_O = 2 * N1, COL_L = COL_O + 2 * N2;
  static constexpr int COLS_USED = COL_L + (BF16 ? 0 : 2 * N2);
  static constexpr int TMEM_COLS = COLS_USED <= 64 ? 64 : COLS_USED <= 128 ? 128 : COLS_USED <= 256 ? 256 : 512;
  static_assert(BF16 ? (NT == 4 || NT == 8) : (NT == 16 || NT == 32), "rows per CTA");
  static_assert(!(BF16 && QN), "native QK is an FP8 option");
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory");
  static_assert(OFF_Q % 1024 == 0 && OFF_P % 1024 == 0 && OFF_ONES % 1024 == 0, "alignment");
  static_assert(!NV || SOFT_H == 1, "NVFP4: one softmax group, converter warps at 8-11");
  static_assert(BF16 || RH == 8, "FP8: 8 rows per softmax thread");
  static_assert(sizeof(Desc) % 16 == 0 && OFF_DESC % 16 == 0 && OFF_SLOTS % 16 == 0, "alignment");
};

// Instruction descriptor, kind::f8f6f4 with e4m3 A and B, fp32 D, K-major.
__host__ __device__ constexpr uint32_t umma_idesc_e4m3(int M, int N) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
// kind::f8f6f4 with e4m3 A and B, fp32 D, both operands MN-major (A = V^T
// with the head dimension contiguous, B = P^T with the rows contiguous).
__host__ __device__ constexpr uint32_t umma_idesc_e4m3_mn(int M, int N) {
  return umma_idesc_e4m3(M, N) | (1u << 15) | (1u << 16);
}
// kind::f16 with bf16 A and B (f16 A and B when f16 is set), fp32 D.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, bool a_mn, bool b_mn,
                                                       bool f16 = false) {
  return (1u << 4) | (f16 ? 0u : (1u << 7) | (1u << 10)) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 2D TMA tile load (x = element column, y = row) completing on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_ld16_raw(uint32_t taddr, float* v) {
  float (&vv)[16] = *reinterpret_cast<float(*)[16]>(v);
  tmem_ld16(taddr, vv);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Two floats -> two e4m3 codes (round to nearest even, saturating), low
// byte = first.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}

// Two weights -> their two-term e4m3 split, low byte first: returns
// e4m3(p) in the low 16 bits and e4m3(16 (p - e4m3(p))) in the high 16.
// Done in f16x2: p (<= 2^8) rounds to f16 first; p16 - hi is then exact in
// f16 (hi is p16 on e4m3's coarser grid) and so is the factor 16, so the
// pair keeps about 8 significant bits of p.
__device__ __forceinline__ uint32_t e4m3_split2(float p0, float p1) {
  const __half2 a = __floats2half2_rn(p0, p1);
  const __nv_fp8x2_storage_t h =
      __nv_cvt_halfraw2_to_fp8x2(static_cast<__half2_raw>(a), __NV_SATFINITE, __NV_E4M3);
  const __half2 d = static_cast<__half2>(__nv_cvt_fp8x2_to_halfraw2(h, __NV_E4M3));
  const __half2 l = __hmul2(__hsub2(a, d), __float2half2_rn(16.f));
  const __nv_fp8x2_storage_t lo =
      __nv_cvt_halfraw2_to_fp8x2(static_cast<__half2_raw>(l), __NV_SATFINITE, __NV_E4M3);
  return (uint32_t)h | ((uint32_t)lo << 16);
}

// Eight e2m1 codes (one word, element 2k in the low nibble of byte k) ->
// four f16 pairs (exact), element 2k in the low half of h[k].
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t* h) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code & 0xFF), __NV_E4M3);
  return __half2float(*reinterpret_cast<const __half*>(&h));
}

// Same phase-parity wait as mbar_wait, on a barrier of an ItemDesc ring etc.,
// but non-blocking: true once the phase of `parity` has completed.
__device__ __forceinline__ bool mbar_ready(uint64_t* bar, uint32_t parity) {
  return mbar_test(bar, parity);
}

// Item t of the queue -> (b, kvh, split, rt); rt varies fastest, so the
// splits of one group are drawn close together and their merge comes early.
// Sequences come in the prologue's order (most visible tiles first), so the
// queue ends on short items and the CTAs finish close together.
__device__ __forceinline__ void decode_item(const SplitArgs& a, int t, int& b, int& kvh,
                                            int& split, int& rt) {
  rt = t % a.row_tiles;
  int u = t / a.row_tiles;
  split = u % a.num_splits;
  u /= a.num_splits;
  kvh = u % a.Hkv;
  b = u / a.Hkv;
  if (a.order) b = __ldcg(a.order + b);
}

template <int KV, int NT, bool QN = false>
__global__ void __launch_bounds__(TmaCfg<KV, NT, QN>::THREADS, 1)
    split_tma_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                     const SplitArgs a) {
  using C = TmaCfg<KV, NT, QN>;
  using Desc = typename C::Desc;
  constexpr int PA = C::PID_AHEAD;
  constexpr unsigned FULL = 0xFFFFFFFFu;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // swizzle atoms need 1024-byte aligned bases
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                       // [S] TMA landed
  uint64_t* empty = bars + C::STAGES;          // [S] stage consumed
  uint64_t* s_full = bars + 2 * C::STAGES;     // [2] S^T in TMEM
  uint64_t* p_ready = s_full + 2;              // [2] P^T in shared memory
  uint64_t* o_full = s_full + 4;               // [2] O^T in TMEM
  uint64_t* o_free = s_full + 6;               // [2] O^T region of an item read back
  uint64_t* desc_full = s_full + 8;            // [4] item descriptor published
  uint64_t* desc_free = desc_full + C::DSLOTS; // [4] item finished (descriptor reusable)
  uint64_t* q_ready = desc_free + C::DSLOTS;   // [2] Q operand + per-row state written
  uint64_t* st_free = q_ready + 2;             // [2] per-row state of an item released
  uint64_t* q_free = st_free + 2;              // [2] S^T MMAs of an item done (its Q reusable)
  uint64_t* raw_full = q_free + 2;             // NVFP4 [R] raw tile landed
  uint64_t* raw_empty = raw_full + C::RAW_STAGES;  // NVFP4 [R] raw tile decoded
  uint64_t* k_full = raw_empty + C::RAW_STAGES;    // NVFP4 [S] f16 K of the stage written
                                                   // (full[]: its V too)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  volatile int* tiles_done = abort_flag + 1;  // tiles the softmax warps have finished
  volatile int* merge_flag = abort_flag + 4;  // [row group]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);
  Desc* descs = reinterpret_cast<Desc*>(smem + C::OFF_DESC);
  auto slot_of = [&](int j) { return smem + C::OFF_SLOTS + (j & 1) * C::SLOT; };

  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      // TMA: the producer's arrive and the copies' bytes; NVFP4: every
      // converter thread's arrive once the f16 tile is written
      mbar_init(&full[s], C::NV ? 32 * C::CONV_WARPS : 1);
      mbar_init(&empty[s], 1);  // the O^T MMAs of the tile are done
    }
    for (int s = 0; s < C::RAW_STAGES; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], 32 * C::CONV_WARPS);
    }
    if constexpr (C::NV)
      for (int s = 0; s < C::STAGES; ++s) mbar_init(&k_full[s], 32 * C::CONV_WARPS);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], C::SOFT_THREADS);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], C::SOFT_THREADS);
      mbar_init(&q_ready[i], 32);
      mbar_init(&st_free[i], C::SOFT_H);  // one arrival per softmax row group
      mbar_init(&q_free[i], 1);
    }
    for (int i = 0; i < C::DSLOTS; ++i) {
      mbar_init(&desc_full[i], 32);
      mbar_init(&desc_free[i], C::SOFT_H);
    }
    abort_flag[0] = 0;
    for (int k = 0; k < 4; ++k) merge_flag[k] = 0;
    tiles_done[0] = 0;
    fence_mbar_init();
  }
  if (warp == C::S_MMA) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp >= C::SOFT0 && warp < C::SOFT0 + 4) {
    // Q rows that no item writes (bf16: rows >= NT) and P^T rows >= 2*NT
    // (bf16) stay zero for the whole kernel.
    const int i = tid - C::SOFT0 * 32;
    for (int c = i; c < 2 * C::Q_BUF / 16; c += 128)
      reinterpret_cast<uint4*>(smem + C::OFF_Q)[c] = make_uint4(0, 0, 0, 0);
    if constexpr (C::BF16) {
      for (int c = i; c < 2 * C::P_BUF / 16; c += 128)
        reinterpret_cast<uint4*>(smem + C::OFF_P)[c] = make_uint4(0, 0, 0, 0);
    } else {
      for (int c = i; c < C::ONES / 16; c += 128)  // e4m3 1.0 = 0x38
        reinterpret_cast<uint4*>(smem + C::OFF_ONES)[c] =
            make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
    }
    fence_proxy_async_smem();  // read by the tensor core
  }
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Everything above overlaps the prologue kernel; the counters, the queue
  // order and the Q images it writes are read only after this.
  pdl_wait_primary();

  if (warp == C::SCHED) {
    // ======================= scheduler (whole warp) ==========================
    // Publishes item descriptors up to DSLOTS ahead of the items the softmax
    // warps have finished (and while fewer than AHEAD_TILES drawn tiles are
    // pending), and writes the Q operand and per-row state of item j into
    // buffer j & 1 once the S^T MMAs and the softmax warps are done with
    // item j-2.
    auto publish = [&](int j) -> bool {
      Desc& d = descs[j & (C::DSLOTS - 1)];
      int t = 0;
      if (lane == 0) t = atomicAdd(a.sched, 1);
      t = __shfl_sync(FULL, t, 0);
      const bool more = t < a.num_items;
      if (more) {
        int b, kvh, split, rt;
        decode_item(a, t, b, kvh, split, rt);
        int L = __ldg(a.kv_lens + b);
        const int Lmax = a.max_pages << a.log2_page;
        if (L < 0 || L > Lmax) {
          if (lane == 0) record_error_at(a.err, kErrBadPage);
          L = L < 0 ? 0 : Lmax;
        }
        const int R0 = rt * NT;
        const int Rlast = min(a.M, R0 + NT) - 1;
        int lo_u, hi_u, lo_x, hi_x;
        row_range(a, L, R0 / a.G, lo_u, hi_x);     // first row: union lo, intersection hi
        row_range(a, L, Rlast / a.G, lo_x, hi_u);  // last row: intersection lo, union hi
        const int k_begin = lo_u / C::TILE;
        const int k_end = hi_u > lo_u ? (hi_u + C::TILE - 1) / C::TILE : k_begin;
        const int n_all = k_end - k_begin;
        const int chunk = (n_all + a.num_splits - 1) / a.num_splits;
        const int c0 = min(n_all, split * chunk);
        const int ntiles = min(n_all, c0 + chunk) - c0;
        const int kfirst = k_begin + c0;
        // page ids of the first PA tiles, one (tile, segment) pair per lane
        const int seq_pages = (L + a.page_size - 1) >> a.log2_page;
        const int32_t* pt_row = a.page_table + (long long)b * a.max_pages;
        for (int e = lane; e < PA * 16; e += 32) {
          const int n = e >> 4, g = e & 15;
          int pid = 0;
          if (n < ntiles) {
            const int first = ((kfirst + n) * C::TILE) >> a.log2_page;
            const int nseg =
                a.page_size >= C::TILE ? 1 : min(C::TILE >> a.log2_page, seq_pages - first);
            if (g < nseg) {
              pid = __ldg(pt_row + first + g);
              if ((unsigned)pid >= (unsigned)a.num_pages) {
                record_error_at(a.err, kErrBadPage);
                pid = 0;
              }
            }
          }
          d.pids[n][g] = pid;
        }
        if (lane == 0) {
          d.b = b;
          d.kvh = kvh;
          d.split = split;
          d.rt = rt;
          d.L = L;
          d.kfirst = kfirst;
          d.ntiles = ntiles;
          d.lo_u = lo_u;
          d.hi_u = hi_u;
          d.lo_x = lo_x;
          d.hi_x = hi_x;
        }
      } else if (lane == 0) {
        d.b = -1;
        d.ntiles = 0;
      }
      __syncwarp();
      mbar_arrive(&desc_full[j & (C::DSLOTS - 1)]);
      return more;
    };
    // bf16: Q rows of an item are prefetched into L2 when the item is
    // published (one bulk prefetch per query row position: its G heads are
    // contiguous), so preparing its Q operand later reads L2, not HBM. (FP8
    // copies the prologue kernel's image instead.)
    auto prefetch_q = [&](int j) {
      const Desc& d = descs[j & (C::DSLOTS - 1)];
      if (C::BF16 && lane < a.Lq) {
        const uint16_t* src = a.q + ((long long)(d.b * a.Lq + lane) * a.Hq + d.kvh * a.G) * C::D;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src),
                     "r"((uint32_t)(a.G * C::D * 2))
                     : "memory");
      }
    };
    // Write item j's Q operand and per-row state.
    auto prep = [&](int j) {
      const Desc& d = descs[j & (C::DSLOTS - 1)];
      uint8_t* sl = slot_of(j);
      const int b = d.b, kvh = d.kvh, R0 = d.rt * NT;
      if (lane < NT) {  // per-row state
        const int R = R0 + lane;
        int lo = 0, hi = 0;
        long long row = -1;  // output row [b, qi, h] of packed row R (-1: padding)
        float sink = -INFINITY;
        if (R < a.M) {
          const int qi = R / a.G, h = kvh * a.G + (R - qi * a.G);
          row_range(a, d.L, qi, lo, hi);
          row = (long long)(b * a.Lq + qi) * a.Hq + h;
          if (a.sinks) sink = __ldg(a.sinks + h);
        }
        reinterpret_cast<float*>(sl + C::SL_SINK)[lane] = sink;
        reinterpret_cast<long long*>(sl + C::SL_ROWS)[lane] = row;
        reinterpret_cast<int2*>(sl + C::SL_RANGE)[lane] = make_int2(lo, hi);
        reinterpret_cast<float2*>(sl + C::SL_CSM)[lane] = make_float2(1.f, 0.f);
        reinterpret_cast<float*>(sl + C::SL_THR)[lane] = -INFINITY;
        reinterpret_cast<float*>(sl + C::SL_MRAW)[lane] = -INFINITY;
      }
      float* cs = reinterpret_cast<float*>(sl + C::SL_CS);
      uint8_t* qbuf = smem + C::OFF_Q + (j & 1) * C::Q_BUF;
      if constexpr (C::BF16) {
        // rows 0..NT-1 of the SW128 K-major bf16 operand: 16 chunks of 8
        // elements per row, chunk jj in half jj / 8
        constexpr int QREG = (NT * 16 + 31) / 32;
        uint4 qv[QREG];
#pragma unroll
        for (int k = 0; k < QREG; ++k) {  // all loads first
          const int c = lane + 32 * k, n = c >> 4, jj = c & 15;
          const int R = R0 + n;
          qv[k] = make_uint4(0, 0, 0, 0);
          if (n < NT && R < a.M) {
            const int qi = R / a.G, h = kvh * a.G + R % a.G;
            qv[k] = __ldg(reinterpret_cast<const uint4*>(
                a.q + ((long long)(b * a.Lq + qi) * a.Hq + h) * C::D + jj * 8));
          }
        }
        if constexpr (C::NV) {
          // NVFP4: the MMAs take f16, so each bf16 q row enters as f16 of
          // q * 2^e, 2^e the power of two that puts the row's max |q| in
          // [2^14, 2^15): exact for every element within 2^28 of the row's
          // max (smaller ones round in f16's subnormal range); the score
          // scale of the row carries 2^-e. The 16 lanes of a row are adjacent.
#pragma unroll
          for (int k = 0; k < QREG; ++k) {
            const int c = lane + 32 * k, n = c >> 4, jj = c & 15;
            float f[8];
            bf16x8_to_f32(qv[k], f);
            float mx = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(f[e]));
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
            const int e2 = mx > 0.f ? 14 - ilogbf(mx) : 0;
            uint32_t hw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __half2 h = __floats2half2_rn(ldexpf(f[2 * e], e2), ldexpf(f[2 * e + 1], e2));
              hw[e] = *reinterpret_cast<const uint32_t*>(&h);
            }
            qv[k] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            if (jj == 0 && n < NT) cs[n] = ldexpf(a.qk_scale_log2, -e2);
          }
        }
#pragma unroll
        for (int k = 0; k < QREG; ++k) {
          const int c = lane + 32 * k, n = c >> 4, jj = c & 15;
          if (n < NT)
            *reinterpret_cast<uint4*>(qbuf + (jj >> 3) * C::Q_HALF + (n >> 3) * 1024 +
                                      (n & 7) * 128 + (((jj & 7) ^ (n & 7)) << 4)) = qv[k];
        }
        if (!C::NV && lane < NT) cs[lane] = a.qk_scale_log2;
      } else {
        // the prologue kernel's image of this (b, kv head, row tile): one bulk
        // copy, counted on q_ready next to the 32 lanes' arrivals below
        const uint8_t* img = a.qops + (((long long)b * a.Hkv + kvh) * a.row_tiles + d.rt) * C::QOP;
        if (lane == 0) {
          mbar_expect_tx(&q_ready[j & 1], C::Q_BYTES);
          bulk_g2s(qbuf, img, C::Q_BYTES, &q_ready[j & 1]);
        }
        if (lane < NT) cs[lane] = __ldcg(reinterpret_cast<const float*>(img + C::Q_BYTES) + lane);
      }
      fence_proxy_async_smem();  // the Q operand is read by the tensor core
      __syncwarp();
      mbar_arrive(&q_ready[j & 1]);
    };

    int jd = 0, jq = 0, last = -1;  // last: index of the end-of-queue descriptor
    int drawn_tiles = 0;             // tiles of the items published so far
    long long idle_since = clock64();
    while (true) {
      if (*abort_flag) break;
      bool progressed = false;
      if (last < 0) {
        bool r = false;
        if (lane == 0)
          r = drawn_tiles - *tiles_done < C::AHEAD_TILES &&
              (jd < C::DSLOTS || mbar_ready(&desc_free[jd & (C::DSLOTS - 1)], ((jd / C::DSLOTS) - 1) & 1));
        const bool can = __shfl_sync(FULL, r, 0);
        if (can) {
          if (publish(jd)) {
            prefetch_q(jd);
            drawn_tiles += descs[jd & (C::DSLOTS - 1)].ntiles;
          } else {
            last = jd;
          }
          ++jd;
          progressed = true;
        }
      }
      if (jq < jd && jq != last) {
        bool r = false;
        if (lane == 0)
          r = jq < 2 || (mbar_ready(&q_free[jq & 1], ((jq >> 1) - 1) & 1) &&
                         mbar_ready(&st_free[jq & 1], ((jq >> 1) - 1) & 1));
        if (__shfl_sync(FULL, r, 0)) {
          prep(jq);
          ++jq;
          progressed = true;
        }
      }
      if (last >= 0 && jq == last) break;
      if (progressed) {
        idle_since = clock64();
      } else {
        if (clock64() - idle_since > kWaitTimeoutCycles) {
          if (lane == 0) {
            record_error_at(a.err, kErrTimeout);
            *abort_flag = 1;
          }
          break;
        }
        __nanosleep(32);
      }
    }
    __syncwarp();
  } else if (warp == C::PROD) {
    // ======================= TMA producer (whole warp) =======================
    // Tile g (counted over all items of this CTA) goes to stage g % STAGES.
    // Page ids: the first PA tiles of an item come with its descriptor; tile
    // n >= PA arrives by cp.async PA tiles ahead (one commit group per tile,
    // so "tile n's group is complete" is cp.async.wait_group PA-1).
    int32_t* sm_pids = reinterpret_cast<int32_t*>(smem + C::OFF_PIDS);
    const uint32_t sbase = smem_addr(smem);
    if (!C::NV && lane == 0) {  // (NVFP4 copies take no tensor map)
      asm volatile("prefetch.tensormap [%0];" ::"l"(&tmk) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(&tmv) : "memory");
    }
    int g = 0;
    bool ok = true;
    for (int j = 0; ok; ++j) {
      ok = !*abort_flag && mbar_wait(&desc_full[j & (C::DSLOTS - 1)], (j / C::DSLOTS) & 1, a.err);
      if (!__all_sync(FULL, ok)) {
        ok = false;
        break;
      }
      const Desc& d = descs[j & (C::DSLOTS - 1)];
      const int b = d.b;
      if (b < 0) break;
      const int kvh = d.kvh, kfirst = d.kfirst, ntiles = d.ntiles;
      const int seq_pages = (d.L + a.page_size - 1) >> a.log2_page;
      const int32_t* pt_row = a.page_table + (long long)b * a.max_pages;
      const int seg_rows = a.page_size < C::TILE ? a.page_size : C::TILE;
      auto nseg_of = [&](int n) {
        const int first = ((kfirst + n) * C::TILE) >> a.log2_page;
        return a.page_size >= C::TILE ? 1 : min(C::TILE >> a.log2_page, seq_pages - first);
      };
      for (int n = 0; n < ntiles; ++n, ++g) {
        int pid = 0;
        if (n < PA) {
          pid = d.pids[n][lane & 15];
        } else {
          asm volatile("cp.async.wait_group %0;" ::"n"(PA - 1) : "memory");
          if (lane < nseg_of(n)) {
            pid = sm_pids[(n % C::PID_SLOTS) * 16 + lane];
            if ((unsigned)pid >= (unsigned)a.num_pages) {
              record_error_at(a.err, kErrBadPage);
              pid = 0;
            }
          }
        }
        __syncwarp();  // slot n % PID_SLOTS is read before it can be refilled
        {
          const int m = n + PA;  // prefetch the page ids of tile n + PA
          if (m < ntiles && lane < nseg_of(m)) {
            const int32_t* src = pt_row + (((kfirst + m) * C::TILE) >> a.log2_page) + lane;
            const uint32_t dst = smem_addr(sm_pids + (m % C::PID_SLOTS) * 16 + lane);
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
          }
          asm volatile("cp.async.commit_group;" ::: "memory");
        }
        const int tok0 = (kfirst + n) * C::TILE;
        const int nseg = nseg_of(n);
        if constexpr (C::NV) {
          // raw NVFP4 tile: per page segment, its codes (64 bytes per token)
          // and block scales (8 bytes per token) of K and V, four bulk copies
          // into raw slot g % RAW_STAGES, decoded by the converter warps
          const int rs = g % C::RAW_STAGES;
          ok = !*abort_flag;
          if (ok && g >= C::RAW_STAGES)
            ok = mbar_wait(&raw_empty[rs], ((g / C::RAW_STAGES) - 1) & 1, a.err);
          if (!__all_sync(FULL, ok)) {
            ok = false;
            break;
          }
          uint8_t* raw = smem + C::OFF_RAW + rs * C::RAW_STAGE;
          uint64_t* rb = &raw_full[rs];
          if (lane == 0)
            mbar_arrive_expect_tx(rb, 2u * (uint32_t)(nseg * seg_rows) * (uint32_t)(C::D / 2 + C::D / 16));
          __syncwarp();  // the transaction count is set before any copy completes
          if (lane < nseg) {
            const long long row = (long long)(pid * a.Hkv + kvh) * a.page_size +
                                  (a.page_size >= C::TILE ? (tok0 & (a.page_size - 1)) : 0);
            const uint32_t cbytes = (uint32_t)seg_rows * (C::D / 2);
            const uint32_t sbytes = (uint32_t)seg_rows * (C::D / 16);
            uint8_t* kc = raw + lane * cbytes;
            uint8_t* ks = raw + C::RAW_C + lane * sbytes;
            uint8_t* vc = raw + C::RAW_C + C::RAW_S + lane * cbytes;
            uint8_t* vs = raw + 2 * C::RAW_C + C::RAW_S + lane * sbytes;
            bulk_g2s(kc, a.k_pages + row * (C::D / 2), cbytes, rb);
            bulk_g2s(ks, a.k_scales + row * (C::D / 16), sbytes, rb);
            bulk_g2s(vc, a.v_pages + row * (C::D / 2), cbytes, rb);
            bulk_g2s(vs, a.v_scales + row * (C::D / 16), sbytes, rb);
          }
        } else {
          const int st = g % C::STAGES;
          ok = !*abort_flag;
          if (ok && g >= C::STAGES) ok = mbar_wait(&empty[st], ((g / C::STAGES) - 1) & 1, a.err);
          if (!__all_sync(FULL, ok)) {
            ok = false;
            break;
          }
          const uint32_t seg_bytes = (uint32_t)seg_rows * 128u * (C::BF16 ? 2u : 1u);
          const uint32_t kdst = sbase + C::OFF_STAGE + st * C::STAGE;
          const uint32_t vdst = kdst + C::KT;
          if (lane == 0) mbar_arrive_expect_tx(&full[st], 2u * seg_bytes * (uint32_t)nseg);
          __syncwarp();  // the transaction count is set before any copy completes
          if (lane < nseg) {  // lane s copies segment s: a tile's copies go out together
            const int row = (pid * a.Hkv + kvh) * a.page_size +
                            (a.page_size >= C::TILE ? (tok0 & (a.page_size - 1)) : 0);
            const uint32_t off = (uint32_t)lane * seg_rows * 128u;
            tma_load_2d(kdst + off, &tmk, 0, row, &full[st]);
            tma_load_2d(vdst + off, &tmv, 0, row, &full[st]);
            if constexpr (C::BF16) {  // second 64-element half of each row
              tma_load_2d(kdst + C::HALF + off, &tmk, 64, row, &full[st]);
              tma_load_2d(vdst + C::HALF + off, &tmv, 64, row, &full[st]);
            }
          }
        }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // none left in flight at exit
    if (!ok) {
      if (lane == 0) {
        *abort_flag = 1;
        // copies already issued land before the CTA's shared memory goes away
        if constexpr (C::NV) {
          for (int n = max(0, g - C::RAW_STAGES); n < g; ++n)
            mbar_wait(&raw_full[n % C::RAW_STAGES], (n / C::RAW_STAGES) & 1, a.err,
                      kWaitTimeoutCycles / 16);
        } else {
          for (int n = max(0, g - C::STAGES); n < g; ++n)
            mbar_wait(&full[n % C::STAGES], (n / C::STAGES) & 1, a.err, kWaitTimeoutCycles / 16);
        }
      }
    }
    __syncwarp();
  } else if (warp == C::S_MMA || warp == C::O_MMA) {
    // ======================= MMA issuers: S^T (warp 1), O^T (warp 2) =========
    if (lane == 0) {
      const uint32_t sbase = smem_addr(smem);
      bool ok = true;
      int g = 0, issued = 0;
      for (int j = 0; ok; ++j) {
        ok = !*abort_flag && mbar_wait(&desc_full[j & (C::DSLOTS - 1)], (j / C::DSLOTS) & 1, a.err);
        if (!ok) break;
        const Desc& d = descs[j & (C::DSLOTS - 1)];
        if (d.b < 0) break;
        const int ntiles = d.ntiles;
        if (warp == C::S_MMA) {
          ok = mbar_wait(&q_ready[j & 1], (j >> 1) & 1, a.err);  // Q of item j
          for (int n = 0; ok && n < ntiles; ++n, ++g) {
            const int bb = g & 1;
            ok = !*abort_flag && mbar_wait(C::NV ? &k_full[g % C::STAGES] : &full[g % C::STAGES],
                                           (g / C::STAGES) & 1, a.err);  // K of tile g
            if (ok && g >= 2) ok = mbar_wait(&p_ready[bb], ((g - 2) >> 1) & 1, a.err);
            if (!ok) break;
            tmem_fence_after();
            const uint32_t ka = sbase + C::OFF_STAGE + (g % C::STAGES) * C::STAGE;
            const uint32_t qa = sbase + C::OFF_Q + (j & 1) * C::Q_BUF;
            const uint32_t dt = tmem + C::COL_S + bb * C::N1;
            if constexpr (C::BF16) {
              constexpr uint32_t idesc = umma_idesc_bf16(128, C::N1, false, false, C::NV);
#pragma unroll
              for (int s = 0; s < C::D / 16; ++s)
                umma_f16(dt, umma_desc(ka + (s >> 2) * C::HALF + (s & 3) * 32, 16, 1024, kSw128),
                         umma_desc(qa + (s >> 2) * C::Q_HALF + (s & 3) * 32, 16, 1024, kSw128),
                         idesc, s > 0);
            } else {
              constexpr uint32_t idesc = umma_idesc_e4m3(128, C::N1);
#pragma unroll
              for (int s = 0; s < C::D / 32; ++s)
                umma_f8(dt, umma_desc(ka + s * 32, 16, 1024, kSw128),
                        umma_desc(qa + s * 32, 16, 1024, kSw128), idesc, s > 0);
            }
            umma_commit(&s_full[bb]);
            issued = g + 1;
          }
          if (ok) umma_commit(&q_free[j & 1]);  // arrives once item j's S^T MMAs are done
        } else {
          // O^T (FP8: and the row sums) of item j accumulate over its tiles
          // in TMEM region j & 1, free once the softmax warps read item j-2's.
          if (j >= 2) ok = mbar_wait(&o_free[j & 1], ((j >> 1) - 1) & 1, a.err);
          for (int n = 0; ok && n < ntiles; ++n, ++g) {
            const int bb = g & 1;
            ok = !*abort_flag && mbar_wait(&p_ready[bb], (g >> 1) & 1, a.err);
            // NVFP4: the f16 V of the stage (written after its K)
            if (C::NV && ok) ok = mbar_wait(&full[g % C::STAGES], (g / C::STAGES) & 1, a.err);
            if (!ok) break;
            tmem_fence_after();
            const uint32_t pa = sbase + C::OFF_P + bb * C::P_BUF;
            const uint32_t dt = tmem + C::COL_O + (j & 1) * C::N2;
            const uint32_t va = sbase + C::OFF_STAGE + (g % C::STAGES) * C::STAGE + C::KT;
            if constexpr (C::BF16) {
              constexpr uint32_t idesc = umma_idesc_bf16(128, C::N2, true, true, C::NV);
#pragma unroll
              for (int s = 0; s < C::TILE / 16; ++s)
                umma_f16(dt, umma_desc(va + s * 2048, C::HALF, 1024, kSw128),
                         umma_desc(pa + s * 2 * C::P_SBO, C::P_BYTES, C::P_SBO, C::P_SWIZZLE),
                         idesc, n > 0 || s > 0);
            } else {
              // A = V^T straight from the e4m3 V stage: each token row is one
              // 128-byte swizzle row holding all 128 head-dim elements, so the
              // MN-major atom is 128 elements x 8 tokens; 32 tokens per MMA.
              constexpr uint32_t idesc = umma_idesc_e4m3_mn(128, C::N2);
#pragma unroll
              for (int s = 0; s < C::TILE / 32; ++s)
                umma_f8(dt, umma_desc(va + s * 4096, C::HALF, 1024, kSw128),
                        umma_desc(pa + s * 4 * C::P_SBO, C::P_BYTES, C::P_SBO, C::P_SWIZZLE),
                        idesc, n > 0 || s > 0);
              // row sums of P^T (the normaliser, in every TMEM lane): the same
              // B operand against a tile of ones
              const uint32_t lt = tmem + C::COL_L + (j & 1) * C::N2;
#pragma unroll
              for (int s = 0; s < C::TILE / 32; ++s)
                umma_f8(lt, umma_desc(sbase + C::OFF_ONES, C::HALF, 1024, kSw128),
                        umma_desc(pa + s * 4 * C::P_SBO, C::P_BYTES, C::P_SBO, C::P_SWIZZLE),
                        idesc, n > 0 || s > 0);
            }
            umma_commit(&empty[g % C::STAGES]);  // K and V of the stage are consumed
            umma_commit(&o_full[bb]);
            issued = g + 1;
          }
        }
      }
      if (!ok) *abort_flag = 1;
      if (*abort_flag && issued > 0) {  // MMAs already issued finish before TMEM is freed
        uint64_t* last = warp == C::S_MMA ? &s_full[(issued - 1) & 1] : &o_full[(issued - 1) & 1];
        mbar_wait(last, ((issued - 1) >> 1) & 1, a.err, kWaitTimeoutCycles / 16);
      }
    }
    __syncwarp();
  } else if (C::NV && warp >= C::CONV0 && warp < C::CONV0 + C::CONV_WARPS) {
    if constexpr (C::NV) {  // (compiled for NVFP4 only)
      // ======================= NVFP4 converters (warps 8-11) ====================
      // Tile g: raw slot g % RAW_STAGES -> f16 stage g % STAGES, K then V. A
      // task is 32 consecutive elements of one token (16 code bytes, two
      // 16-element blocks): task k = token k / 4, quarter k % 4, so a warp's
      // loads of one instruction cover 512 contiguous bytes. Each byte of two
      // e2m1 codes becomes an f16 pair (cvt.rn.f16x2.e2m1x2), times its
      // block's scale (an f16 pair from cvt.rn.f16x2.e4m3x2): exact, since an
      // e2m1 x e4m3 product has 5 significant bits and lies in f16's normal
      // range. The f16 rows go to the 128B-swizzled layout the TMA writes for
      // bf16 (two 64-element halves of 8-row atoms), which the MMAs read.
      const int ct = tid - C::CONV0 * 32;  // 0 .. 32 * CONV_WARPS - 1
      constexpr int CT = 32 * C::CONV_WARPS;
      int g = 0;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        ok = !*abort_flag && mbar_wait(&desc_full[j & (C::DSLOTS - 1)], (j / C::DSLOTS) & 1, a.err);
        if (!__all_sync(FULL, ok)) {
          ok = false;
          break;
        }
        const Desc& d = descs[j & (C::DSLOTS - 1)];
        if (d.b < 0) break;
        const int ntiles = d.ntiles;
        for (int n = 0; n < ntiles; ++n, ++g) {
          const int rs = g % C::RAW_STAGES, st = g % C::STAGES;
          const uint8_t* raw = smem + C::OFF_RAW + rs * C::RAW_STAGE;
          uint8_t* stage = smem + C::OFF_STAGE + st * C::STAGE;
          ok = !*abort_flag && mbar_wait(&raw_full[rs], (g / C::RAW_STAGES) & 1, a.err);
          if (!__all_sync(FULL, ok)) {
            ok = false;
            break;
          }
#pragma unroll 1
          for (int pool = 0; ok && pool < 2; ++pool) {
            // K of the stage is free once the S^T MMAs of tile g - STAGES are
            // done, V once its O^T MMAs are (S^T(g) cannot complete before this
            // K is written, so the s_full phase waited for is the right one)
            if (g >= C::STAGES)
              ok = pool == 0 ? mbar_wait(&s_full[(g - C::STAGES) & 1], ((g - C::STAGES) >> 1) & 1, a.err)
                             : mbar_wait(&empty[st], ((g / C::STAGES) - 1) & 1, a.err);
            if (!__all_sync(FULL, ok)) {
              ok = false;
              break;
            }
            const uint8_t* codes = raw + pool * (C::RAW_C + C::RAW_S);
            const uint8_t* scales = codes + C::RAW_C;
            uint8_t* dst = stage + pool * C::KT;
#pragma unroll
            for (int k = ct; k < C::TILE * 4; k += CT) {
              const int t = k >> 2, qq = k & 3;
              const uint4 c = *reinterpret_cast<const uint4*>(codes + t * (C::D / 2) + qq * 16);
              const uint32_t sc2 = *reinterpret_cast<const uint16_t*>(scales + t * (C::D / 16) + 2 * qq);
              const __half2_raw sr = __nv_cvt_fp8x2_to_halfraw2(
                  static_cast<__nv_fp8x2_storage_t>(sc2), __NV_E4M3);
              const __half2 s2 = *reinterpret_cast<const __half2*>(&sr);
              const __half2 sa = __low2half2(s2), sb = __high2half2(s2);
              const uint32_t w[4] = {c.x, c.y, c.z, c.w};  // block 2qq: w[0..1]; 2qq + 1: w[2..3]
              uint32_t o[16];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                e2m1x8_to_f16x8(w[q], o + 4 * q);
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                  const __half2 h = __hmul2(*reinterpret_cast<const __half2*>(&o[4 * q + b]), q < 2 ? sa : sb);
                  o[4 * q + b] = *reinterpret_cast<const uint32_t*>(&h);
                }
              }
              // elements 32 qq .. 32 qq + 31: half qq / 2, chunks 4 (qq & 1) .. + 3
              uint8_t* row = dst + (qq >> 1) * C::HALF + (t >> 3) * 1024 + (t & 7) * 128;
              const int cb = (qq & 1) * 4;
#pragma unroll
              for (int k4 = 0; k4 < 4; ++k4)
                *reinterpret_cast<uint4*>(row + (((cb + k4) ^ (t & 7)) << 4)) =
                    make_uint4(o[4 * k4], o[4 * k4 + 1], o[4 * k4 + 2], o[4 * k4 + 3]);
            }
            fence_proxy_async_smem();  // read by the tensor core (and, once both
                                       // pools are done, the raw slot is refilled)
            mbar_arrive(pool == 0 ? &k_full[st] : &full[st]);
          }
          if (!ok) break;
          mbar_arrive(&raw_empty[rs]);
        }
        if (!ok) break;
      }
      if (!ok) *abort_flag = 1;
    }
  } else if ((warp >= C::SOFT0 && warp < C::SOFT0 + 4) ||
             (C::SOFT_H > 1 && warp >= C::SOFTX && warp < C::SOFTX + 4 * (C::SOFT_H - 1))) {
    // ======================= softmax ==========================================
    // A group of four warps (one per TMEM lane quarter) owns RH rows and
    // synchronises only within itself, on named barrier 2 + group; the
    // groups meet only through mbarriers (p_ready and o_free count every
    // softmax thread, st_free and desc_free one arrival per group), so no
    // group ever waits on a named barrier for another.
    constexpr int RH = C::RH;
    constexpr int GT = 128;          // threads of a group
    const int q4 = warp & 3;
    const int grp = warp < C::SCHED ? 0 : 1 + (warp - C::SOFTX) / 4;  // row group
    const int gbar = 2 + grp;        // the group's named barrier
    const int r0 = grp * RH;         // this thread's rows: r0 .. r0 + RH - 1
    const int i = 32 * q4 + lane;    // TMEM lane: token of S^T, element of O^T
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    float* wmax = reinterpret_cast<float*>(smem + C::OFF_WMAX);
    float* sm_alpha = reinterpret_cast<float*>(smem + C::OFF_ALPHA);
    float* lred = reinterpret_cast<float*>(smem + C::OFF_LRED);
    float* sm_lse = reinterpret_cast<float*>(smem + C::OFF_INV);  // fused merge (reuses sm_inv)
    const long long rows_total = (long long)a.B * a.Lq * a.Hq;
    constexpr float kLn2 = 0.69314718055994531f, kLog2e = 1.4426950408889634f;
    // this thread's column offset in an S^T / O^T / row-sum region
    const uint32_t col_s = C::BF16 ? 0 : (C::QN_ ? r0 : 2 * r0);
    const uint32_t col_o = C::BF16 ? 0 : 2 * r0;
    // wait until the O^T MMAs of tile k have completed (all lanes agree)
    auto wait_o = [&](int k) -> bool {
      const bool ok_w = __all_sync(FULL, mbar_wait(&o_full[k & 1], (k >> 1) & 1, a.err));
      if (ok_w) tmem_fence_after();
      return ok_w;
    };
    // Epilogue of item jj (last tile g_last, nt tiles, status ok_in; lp: bf16
    // partial row sums): reads O^T (FP8: and the row sums) from TMEM region
    // jj & 1 and releases it, normalises, stores O and the LSE (or the
    // split's partials), runs the fused merge and releases the item's state
    // slot and descriptor. It runs after the next item's first tile, when
    // item jj's last MMAs are long done. Returns the group's agreement that
    // nothing failed.
    auto epilogue = [&](int jj, int g_last, int nt, bool ok_in, const float* lp) -> bool {
      const Desc& dd = descs[jj & (C::DSLOTS - 1)];
      const int split = dd.split;
      const uint8_t* sl = slot_of(jj);
      const long long* rows = reinterpret_cast<const long long*>(sl + C::SL_ROWS);
      const float2* sm_csm = reinterpret_cast<const float2*>(sl + C::SL_CSM);
      const float* sm_sink = reinterpret_cast<const float*>(sl + C::SL_SINK);
      const uint32_t o_tm = tmem + lane_off + C::COL_O + (jj & 1) * C::N2 + col_o;
      const uint32_t l_tm = tmem + lane_off + C::COL_L + (jj & 1) * C::N2 + col_o;
      float acc[RH], lsum[RH];
#pragma unroll
      for (int r = 0; r < RH; ++r) {
        acc[r] = 0.f;
        lsum[r] = 0.f;
      }
      bool e_ok = ok_in;
      if (__all_sync(FULL, e_ok && nt > 0 && !*abort_flag)) {
        e_ok = wait_o(g_last);
        if (e_ok) {
          float o[16];
          tmem_ld16_raw(o_tm, o);
          if constexpr (C::BF16) {
#pragma unroll
            for (int r = 0; r < RH; ++r) acc[r] = o[r] + o[NT + r];  // P = P_hi + P_lo
          } else {
#pragma unroll
            for (int r = 0; r < RH; ++r) acc[r] = fmaf(o[RH + r], 0.0625f, o[r]);  // P_hi + (16 P_lo) / 16
            tmem_ld16_raw(l_tm, o);
#pragma unroll
            for (int r = 0; r < RH; ++r) lsum[r] = fmaf(o[RH + r], 0.0625f, o[r]);
          }
        }
      }
      tmem_fence_before();
      mbar_arrive(&o_free[jj & 1]);  // region jj & 1 may take item jj + 2
      const bool eok = named_bar_and(gbar, GT, e_ok);
      if (!eok) *abort_flag = 1;

      // ---- epilogue: normaliser and LSE per row, then the O rows ----------
      if constexpr (C::BF16) {
        // row sums: over the lanes, then over the group's four warps
#pragma unroll
        for (int r = 0; r < RH; ++r) {
          float v = lp[r];
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
          lsum[r] = v;
        }
        if (lane == 0) {
#pragma unroll
          for (int r = 0; r < RH; ++r) lred[q4 * 32 + r0 + r] = lsum[r];
        }
        named_bar(gbar, GT);
#pragma unroll
        for (int r = 0; r < RH; ++r)
          lsum[r] = lred[r0 + r] + lred[32 + r0 + r] + lred[64 + r0 + r] + lred[96 + r0 + r];
      }
      // Thread i < RH derives row r0 + i's normaliser and LSE (the row sum
      // is in every thread: FP8 from TMEM, bf16 from the reduction above)
      // and shares the normaliser through shared memory.
      const bool failed = !eok;
      float* sm_inv = reinterpret_cast<float*>(smem + C::OFF_INV);
      if (i < RH) {
        float lt = 0.f;
#pragma unroll
        for (int r = 0; r < RH; ++r)
          if (r == i) lt = lsum[r];
        const int rr = r0 + i;
        const long long row = rows[rr];
        // attention sink of the row's head (one split only; with splits the
        // merge adds it): one more exp2(sink) term in the denominator
        const float sink = a.num_splits == 1 ? sm_sink[rr] : -INFINITY;
        float inv = 0.f, res = failed ? -INFINITY : sink;
        if (lt > 0.f && !failed) {
          const float m = -sm_csm[rr].y;
          float mref = m, l2 = lt, scl = 1.f;
          if (sink != -INFINITY) {
            const float sink2 = sink * kLog2e;
            mref = fmaxf(m, sink2);
            scl = fast_exp2(m - mref);
            l2 = fmaf(lt, scl, fast_exp2(sink2 - mref));
          }
          inv = a.v_scale * scl / l2;
          res = (mref + log2f(l2)) * kLn2;
        }
        sm_inv[rr] = inv;
        if (row >= 0) {
          if (a.num_splits == 1) {
            if (a.lse) a.lse[row] = res;
          } else {
            a.lse_part[(long long)split * rows_total + row] = res;
          }
        }
      }
      named_bar(gbar, GT);
      float* dst = a.num_splits == 1 ? a.out : a.o_part + (long long)split * rows_total * C::D;
#pragma unroll
      for (int r = 0; r < RH; ++r) {
        const long long row = rows[r0 + r];
        if (row >= 0) dst[row * C::D + i] = acc[r] * sm_inv[r0 + r];
      }

      // ---- fused merge (PDA_FLAG_FUSED_MERGE): the split that arrives last
      // for these rows combines every split's partials by log-sum-exp; each
      // row group counts and merges its own rows --------------------------
      if (a.num_splits > 1 && a.fused_merge) {
        __threadfence();  // this split's partials are visible device-wide ...
        named_bar(gbar, GT);  // (and every sm_inv read is done: sm_lse reuses it)
        if (i == 0) {     // ... before the group counts itself in
          int* ctr = a.merge_ctr +
                     (((long long)dd.b * a.Hkv + dd.kvh) * a.row_tiles + dd.rt) * kMergeCtrPerGroup + grp;
          merge_flag[grp] = atomicAdd(ctr, 1) == a.num_splits - 1;
        }
        named_bar(gbar, GT);
        if (merge_flag[grp]) {
          __threadfence();
          const int S = a.num_splits;  // <= 128
          // (1) per row: lse = m + ln sum_s exp(lse_s - m); warp q4 takes the
          // group's rows q4, q4 + 4, ...; lane l holds splits l, l + 32, l + 64, l + 96.
          constexpr int RW = (RH + 3) / 4;
          float v[RW][4];
#pragma unroll
          for (int k = 0; k < RW; ++k) {
            const int rr = q4 + 4 * k;
            const long long row = rr < RH ? rows[r0 + rr] : -1;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int spl = c * 32 + lane;
              v[k][c] = row >= 0 && spl < S ? __ldcg(a.lse_part + (long long)spl * rows_total + row)
                                            : -INFINITY;
            }
          }
#pragma unroll
          for (int k = 0; k < RW; ++k) {
            // the row's attention sink is one more part: lse = sink, o = 0
            const int rr = q4 + 4 * k;
            const long long rrow = rr < RH ? rows[r0 + rr] : -1;
            const float sink = rrow >= 0 ? sm_sink[r0 + rr] : -INFINITY;
            float m = fmaxf(fmaxf(v[k][0], v[k][1]), fmaxf(v[k][2], v[k][3]));
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
            m = fmaxf(m, sink);
            float sum = 0.f;
            if (m != -INFINITY) {
#pragma unroll
              for (int c = 0; c < 4; ++c)
                if (v[k][c] != -INFINITY) sum += fast_exp2((v[k][c] - m) * kLog2e);
              if (lane == 0 && sink != -INFINITY) sum += fast_exp2((sink - m) * kLog2e);
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(FULL, sum, o);
            if (lane == 0 && rr < RH) sm_lse[r0 + rr] = m == -INFINITY ? -INFINITY : m + log2f(sum) * kLn2;
          }
          named_bar(gbar, GT);
          // (2) out[row, i] = sum_s exp(lse_s - lse) * o_s[row, i] over this
          // thread's rows; the rows' loads of one split go out together
#pragma unroll
          for (int r = 0; r < RH; ++r) acc[r] = 0.f;
          for (int spl = 0; spl < S; ++spl) {
            float ls[RH], ov[RH];
#pragma unroll
            for (int r = 0; r < RH; ++r) {
              const long long row = rows[r0 + r];
              const long long idx = (long long)spl * rows_total + (row >= 0 ? row : 0);
              ls[r] = row >= 0 ? __ldcg(a.lse_part + idx) : -INFINITY;
              ov[r] = row >= 0 ? __ldcg(a.o_part + idx * C::D + i) : 0.f;
            }
#pragma unroll
            for (int r = 0; r < RH; ++r)
              if (ls[r] != -INFINITY)
                acc[r] = fmaf(fast_exp2((ls[r] - sm_lse[r0 + r]) * kLog2e), ov[r], acc[r]);
          }
#pragma unroll
          for (int r = 0; r < RH; ++r) {
            const long long row = rows[r0 + r];
            if (row >= 0) a.out[row * C::D + i] = acc[r];
          }
          if (i < RH && rows[r0 + i] >= 0 && a.lse) a.lse[rows[r0 + i]] = sm_lse[r0 + i];
        }
      }
      named_bar(gbar, GT);  // the group no longer reads item jj's state and descriptor
      if (i == 0) {
        mbar_arrive(&st_free[jj & 1]);
        mbar_arrive(&desc_free[jj & (C::DSLOTS - 1)]);
      }
      return eok;
    };

    int g = 0;  // tiles of this CTA so far (over all items)
    bool ok = true, acc_prev = true;
    // the item whose epilogue is pending (-1: none), its last tile, tile
    // count, status and partial row sums (bf16; FP8 sums by MMA)
    int pend = -1, pend_g = 0, pend_nt = 0;
    bool pend_ok = true;
    float l_pend[RH];
#pragma unroll
    for (int r = 0; r < RH; ++r) l_pend[r] = 0.f;
    for (int j = 0;; ++j) {
      bool w = acc_prev && !*abort_flag &&
               mbar_wait(&desc_full[j & (C::DSLOTS - 1)], (j / C::DSLOTS) & 1, a.err);
      if (w && descs[j & (C::DSLOTS - 1)].b >= 0) w = mbar_wait(&q_ready[j & 1], (j >> 1) & 1, a.err);
      if (!named_bar_and(gbar, GT, w)) ok = false;
      const Desc& d = descs[j & (C::DSLOTS - 1)];
      const bool last = !ok || d.b < 0;  // no item j: only the pending epilogue is left
      const int ntiles = last ? 0 : d.ntiles;
      bool acc_ok = ok;
      float l_part[RH];  // bf16: this thread's part of item j's row sums
#pragma unroll
      for (int r = 0; r < RH; ++r) l_part[r] = 0.f;
      const int kfirst = d.kfirst;
      const int lo_u = d.lo_u, hi_u = d.hi_u, lo_x = d.lo_x, hi_x = d.hi_x;
      uint8_t* sl = slot_of(j);
      const int2* rng = reinterpret_cast<const int2*>(sl + C::SL_RANGE);
      const float* sm_cs = reinterpret_cast<const float*>(sl + C::SL_CS);
      float2* sm_csm = reinterpret_cast<float2*>(sl + C::SL_CSM);
      float* sm_thr = reinterpret_cast<float*>(sl + C::SL_THR);
      float* sm_mraw = reinterpret_cast<float*>(sl + C::SL_MRAW);
      // O^T (and, FP8, the row sums) of this item accumulate in TMEM region
      // j & 1: bf16, 16 columns (r: P_hi, NT + r: P_lo), all read by every
      // thread; FP8, this group's 16 columns (hi terms of its rows, then lo).
      const uint32_t o_tm = tmem + lane_off + C::COL_O + (j & 1) * C::N2 + col_o;
      // this thread's rows' lazy-rescale thresholds, kept in registers and
      // reloaded whenever a tile moves the max
      float4 thr4[RH / 4];
      auto load_row_consts = [&]() {
#pragma unroll
        for (int k = 0; k < RH / 4; ++k) thr4[k] = reinterpret_cast<const float4*>(sm_thr + r0)[k];
      };
      load_row_consts();
      const uint32_t l_tm = tmem + lane_off + C::COL_L + (j & 1) * C::N2 + col_o;
      for (int n = 0; n < ntiles; ++n, ++g) {
        const int bb = g & 1;
        bool ok_s = acc_ok && !*abort_flag;
        if (ok_s) ok_s = mbar_wait(&s_full[bb], (g >> 1) & 1, a.err);
        ok_s = __all_sync(FULL, ok_s);
        float s[RH];  // scores (then probabilities) of this thread's rows
        if (ok_s) {
          tmem_fence_after();
          const uint32_t ta = tmem + lane_off + C::COL_S + bb * C::N1 + col_s;
          if constexpr (C::BF16) {
            float sraw[16];
            tmem_ld16_raw(ta, sraw);
#pragma unroll
            for (int r = 0; r < RH; ++r) s[r] = sraw[r];
          } else if constexpr (C::QN_) {  // S = S_hi
            tmem_ld8(ta, s);
          } else {  // S = S_hi + S_lo / 16 (the group's hi columns, then lo)
            float sraw[16];
            tmem_ld16_raw(ta, sraw);
#pragma unroll
            for (int r = 0; r < RH; ++r) s[r] = fmaf(sraw[RH + r], 0.0625f, sraw[r]);
          }
        } else {
#pragma unroll
          for (int r = 0; r < RH; ++r) s[r] = -INFINITY;
        }
        const int t0 = (kfirst + n) * C::TILE;
        const int jt = t0 + i;
        const bool clean = t0 >= lo_x && t0 + C::TILE <= hi_x;
        if (!clean) {
#pragma unroll
          for (int r = 0; r < RH; ++r) {
            const int2 lh = rng[r0 + r];
            if (!(jt >= lh.x && jt < lh.y)) s[r] = -INFINITY;
          }
          // zero V row i of the stage (bf16: 2 halves) where no row sees key
          // jt; group 0 only. Chunks in rotated order: the 8 rows of a
          // 1 KB swizzle atom hit 8 different bank groups.
          if (grp == 0 && (jt < lo_u || jt >= hi_u)) {
            // NVFP4: the f16 V of the stage is written after its K, so wait
            // for it before zeroing rows (no later write can come: the next
            // tile into this stage waits for this one's O^T MMAs)
            if (C::NV && !mbar_wait(&full[g % C::STAGES], (g / C::STAGES) & 1, a.err))
              acc_ok = false;
            uint8_t* vrow = smem + C::OFF_STAGE + (g % C::STAGES) * C::STAGE + C::KT + i * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const int cc = (c + i) & 7;
              *reinterpret_cast<uint4*>(vrow + cc * 16) = make_uint4(0, 0, 0, 0);
              if constexpr (C::BF16) *reinterpret_cast<uint4*>(vrow + C::HALF + cc * 16) = make_uint4(0, 0, 0, 0);
            }
          }
        }
        // Lazy rescale: the running max m of each row (log2 domain) only moves
        // when a score exceeds it by more than kRescaleLog2, so p = exp2(x - m)
        // stays <= 2^kRescaleLog2 (well inside f16 and e4m3) and most tiles
        // skip the per-tile max exchange. The test runs on raw scores against
        // thr = (m + kRescaleLog2) / cs (-inf until the row's first finite
        // score), so it is one compare per score.
        constexpr float kRescaleLog2 = 8.f;
        auto wants = [&]() {
          bool w = false;
#pragma unroll
          for (int r = 0; r < RH; r += 4) {
            const float4 t = thr4[r / 4];
            w = w | (s[r] > t.x) | (s[r + 1] > t.y) | (s[r + 2] > t.z) | (s[r + 3] > t.w);
          }
          return w;
        };
        // One group barrier decides for the tile: a failed wait counts as a
        // want, and only then (rarely) do the OR of the wants and the AND of
        // the waits' outcomes follow separately.
        bool any;
        if constexpr (!C::BF16) any = named_bar_any_gt8(gbar, GT, s, thr4[0], thr4[1], !ok_s);
        else any = named_bar_or(gbar, GT, wants() || !ok_s);
        bool flag = false;
        if (any) {
          flag = named_bar_or_and(gbar, GT, wants(), ok_s, &ok_s);
          if (!ok_s) {
            acc_ok = false;
            break;
          }
        }
        if (flag) {
#pragma unroll
          for (int r = 0; r < RH; ++r) {
            const float wm = redux_max(s[r]);
            if (lane == r) wmax[q4 * 32 + r0 + r] = wm;
          }
          named_bar(gbar, GT);
          if (i < RH) {
            const int rr = r0 + i;
            const float cs = sm_cs[rr];
            const float st = fmaxf(fmaxf(wmax[rr], wmax[32 + rr]), fmaxf(wmax[64 + rr], wmax[96 + rr]));
            const float m_old = sm_mraw[rr];
            const float m_new = fmaxf(m_old, st * cs);  // -inf stays -inf (cs > 0)
            const float m_use = m_new == -INFINITY ? 0.f : m_new;
            sm_alpha[bb * 32 + rr] = m_old == -INFINITY ? 0.f : fast_exp2(m_old - m_use);
            sm_mraw[rr] = m_new;
            sm_csm[rr] = make_float2(cs, -m_use);
            sm_thr[rr] = m_new == -INFINITY ? -INFINITY : (m_use + kRescaleLog2) / cs;
          }
          named_bar(gbar, GT);
          load_row_consts();
          const float* al = sm_alpha + bb * 32 + r0;
          if constexpr (C::BF16) {
#pragma unroll
            for (int r = 0; r < RH; ++r) l_part[r] *= al[r];
          }
          // What the tiles before this one accumulated (O^T, FP8 also the row
          // sums) moves to the new max before this tile's MMAs add to it
          // (rare: the max moves on an item's first tile, then only on a jump
          // of 2^8). A failed wait only clears acc_ok: the group's next
          // barrier then stops all four of its warps together.
          if (n > 0) {
            if (wait_o(g - 1)) {
              if constexpr (C::BF16) {
                float o[16];
                tmem_ld16_raw(o_tm, o);
#pragma unroll
                for (int c = 0; c < 16; ++c) o[c] *= al[c % NT];
                tmem_st16(o_tm, o);
              } else {  // 8 columns at a time (O hi, O lo, sums hi, sums lo)
#pragma unroll 1
                for (int part = 0; part < 4; ++part) {
                  const uint32_t ta = (part < 2 ? o_tm : l_tm) + (part & 1) * RH;
                  float o[RH];
                  tmem_ld8(ta, o);
#pragma unroll
                  for (int c = 0; c < RH; ++c) o[c] *= al[c];
                  tmem_st8(ta, o);
                }
              }
              tmem_fence_before();
            } else {
              acc_ok = false;
            }
          }
        }
        float* p = s;
#pragma unroll
        for (int r = 0; r < RH; r += 2) {
          const float4 c = reinterpret_cast<const float4*>(sm_csm + r0)[r / 2];
          p[r] = fast_exp2(fmaf(s[r], c.x, c.y));
          p[r + 1] = fast_exp2(fmaf(s[r + 1], c.z, c.w));
          if constexpr (C::BF16) {
            l_part[r] += p[r];
            l_part[r + 1] += p[r + 1];
          }
        }
        // P^T buffer bb was last read by the MMAs of tile g - 2. Waiting for
        // them every tile also keeps this warp's o_full phases in step, so
        // the o_full(g - 1) waits above and after the loop never see a phase
        // that is two behind.
        // (Each lane waits for itself: no TMEM access follows, and a lane whose
        // wait fails clears acc_ok, which the next group barrier spreads.)
        if (g >= 2 && !mbar_wait(&o_full[g & 1], ((g - 2) >> 1) & 1, a.err)) acc_ok = false;
        // P^T row of token i (row-major over the N2 columns, swizzled chunks)
        uint8_t* sp = smem + C::OFF_P + bb * C::P_BUF + (i >> 3) * C::P_SBO + (i & 7) * C::P_ROW;
        const int pswz = C::P_ROW == 64 ? ((i & 7) >> 1) & 3 : ((i & 7) >> 2) & 1;
        if constexpr (C::BF16) {
          // columns 0..NT-1: bf16(p); NT..2NT-1: bf16(p - bf16(p)); rest stay 0
          // (NVFP4: the same two terms in f16, the MMAs' operand type)
          uint32_t w[NT];  // NT/2 words of hi, then NT/2 of lo
#pragma unroll
          for (int r = 0; r < NT; r += 2) {
            if constexpr (C::NV) {
              const __half2 h = __floats2half2_rn(p[r], p[r + 1]);
              const float2 hf = __half22float2(h);
              const __half2 l = __floats2half2_rn(p[r] - hf.x, p[r + 1] - hf.y);
              w[r / 2] = *reinterpret_cast<const uint32_t*>(&h);
              w[NT / 2 + r / 2] = *reinterpret_cast<const uint32_t*>(&l);
            } else {
              const __nv_bfloat162 h = __floats2bfloat162_rn(p[r], p[r + 1]);
              const float2 hf = __bfloat1622float2(h);
              w[r / 2] = *reinterpret_cast<const uint32_t*>(&h);
              w[NT / 2 + r / 2] = pack_bf16x2(p[r] - hf.x, p[r + 1] - hf.y);
            }
          }
          if constexpr (NT == 8) {
            *reinterpret_cast<uint4*>(sp + ((0 ^ pswz) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4*>(sp + ((1 ^ pswz) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
          } else {
            *reinterpret_cast<uint4*>(sp + ((0 ^ pswz) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          // the group's 16 columns (one 16-byte chunk): e4m3 P_hi = e4m3(p)
          // of its 8 rows, then 16 (p - P_hi) in e4m3, so P_hi + P_lo / 16
          // keeps about 8 significant bits (p <= 2^8, inside the e4m3 range)
          uint32_t hi[2], lo[2];
#pragma unroll
          for (int r = 0; r < RH; r += 4) {
            const uint32_t s01 = e4m3_split2(p[r], p[r + 1]);
            const uint32_t s23 = e4m3_split2(p[r + 2], p[r + 3]);
            hi[r / 4] = __byte_perm(s01, s23, 0x5410);  // the e4m3(p) halves
            lo[r / 4] = __byte_perm(s01, s23, 0x7632);  // the residual halves
          }
          *reinterpret_cast<uint4*>(sp + ((grp ^ pswz) << 4)) = make_uint4(hi[0], hi[1], lo[0], lo[1]);
        }
        fence_proxy_async_smem();
        tmem_fence_before();
        mbar_arrive(&p_ready[bb]);
        if (grp == 0 && i == 0) *tiles_done = g + 1;  // lets the scheduler draw more work
        if (n == 0 && pend >= 0) {  // the previous item's epilogue
          if (!epilogue(pend, pend_g, pend_nt, pend_ok, l_pend)) acc_ok = false;
          pend = -1;
        }
      }
      // the item's O^T (FP8: and row sums) once its last tile's MMAs are done
      if (pend >= 0) {  // no tile of item j ran the pending epilogue (none, or the end)
        if (!epilogue(pend, pend_g, pend_nt, pend_ok && ok, l_pend)) acc_ok = false;
        pend = -1;
      }
      if (last) break;
      pend = j;
      pend_g = g - 1;
      pend_nt = ntiles;
      pend_ok = acc_ok;
#pragma unroll
      for (int r = 0; r < RH; ++r) l_pend[r] = l_part[r];
      acc_prev = acc_ok;
    }
    if (!ok) *abort_flag = 1;
  }

  pdl_launch_dependents();
  tmem_fence_before();
  __syncthreads();
  if (warp == C::S_MMA) {
    tmem_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::TMEM_COLS)
                 : "memory");
  }
}

// Buckets of the prologue's counting sort: sequences with this many or more
// visible tiles share the last one.
constexpr int kOrderBuckets = 1024;

// Prologue of split_tma_kernel, launched just before it on the same stream
// (the main kernel waits for it with griddepcontrol.wait):
//  * block 0 zeroes the counter header, then ranks the sequences by their
//    visible 128-token tiles, most first (a counting sort; ties in any
//    order: an item's result does not depend on the CTA that runs it), into
//    a.order, the order in which the work queue hands them out;
//  * FP8, blocks 1.. : the Q operand of one (b, kv head, row tile) each,
//    written as the S^T MMA reads it (the same scale choice and two-term
//    split as the in-kernel path), then its 32 row scales.
template <int KV, int NT, bool QN = false>
__global__ void __launch_bounds__(256) split_tma_prologue(const SplitArgs a) {
  using C = TmaCfg<KV, NT, QN>;
  constexpr unsigned FULL = 0xFFFFFFFFu;
  pdl_launch_dependents();  // the main kernel may start its own set-up now
  const int tid = threadIdx.x;
  if (blockIdx.x == 0) {
    __shared__ int hist[kOrderBuckets];
    __shared__ int wsum[8];
    for (int w = tid; w < a.header_words; w += 256) a.sched[w] = 0;
    if (a.order == nullptr) return;
    for (int k = tid; k < kOrderBuckets; k += 256) hist[k] = 0;
    __syncthreads();
    const int Lmax = a.max_pages << a.log2_page;
    auto bucket = [&](int b) {  // descending visible tiles -> ascending bucket
      const int L = min(max(__ldg(a.kv_lens + b), 0), Lmax);
      int lo, hi0, lo1, hi;
      row_range(a, L, 0, lo, hi0);        // first query row: the union's start
      row_range(a, L, a.Lq - 1, lo1, hi);  // last query row: the union's end
      const int n = hi > lo ? (hi + C::TILE - 1) / C::TILE - lo / C::TILE : 0;
      return kOrderBuckets - 1 - min(n, kOrderBuckets - 1);
    };
    for (int b = tid; b < a.B; b += 256) atomicAdd(&hist[bucket(b)], 1);
    __syncthreads();
    // exclusive scan of the histogram: 4 buckets per thread, then warps
    constexpr int PT = kOrderBuckets / 256;
    int v[PT], own = 0;
#pragma unroll
    for (int k = 0; k < PT; ++k) {
      v[k] = hist[tid * PT + k];
      own += v[k];
    }
    const int lane = tid & 31, warp = tid >> 5;
    int inc = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(FULL, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += wsum[w];
    int run = base + inc - own;
#pragma unroll
    for (int k = 0; k < PT; ++k) {
      hist[tid * PT + k] = run;
      run += v[k];
    }
    __syncthreads();
    for (int b = tid; b < a.B; b += 256) a.order[atomicAdd(&hist[bucket(b)], 1)] = b;
    return;
  }
  if constexpr (!C::BF16) {
    // item q = (b, kvh, rt), rt fastest; thread: row n = tid / 8, 16-element
    // chunk c = tid % 8 of it (the 8 threads of a row are adjacent lanes)
    const int q = blockIdx.x - 1;
    const int rt = q % a.row_tiles, kvh = (q / a.row_tiles) % a.Hkv, b = q / (a.row_tiles * a.Hkv);
    uint8_t* img = a.qops + (long long)q * C::QOP;
    const int n = tid >> 3, c = tid & 7;
    if (n >= NT) return;  // whole groups of 8 lanes
    const int R = rt * NT + n;
    const bool live = R < a.M;
    float f[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) f[e] = 0.f;
    if (live) {
      const int qi = R / a.G, h = kvh * a.G + R % a.G;
      const uint4* src = reinterpret_cast<const uint4*>(a.q + ((long long)(b * a.Lq + qi) * a.Hq + h) * C::D);
      bf16x8_to_f32(__ldg(src + 2 * c), *reinterpret_cast<float(*)[8]>(f));
      bf16x8_to_f32(__ldg(src + 2 * c + 1), *reinterpret_cast<float(*)[8]>(f + 8));
    }
    float mx = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(f[e]));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
    // q * 2^e2 = hi + lo / 16 exactly, with 2^e2 the power of two that puts
    // max|q| of the row in [128, 256) (native QK: hi alone)
    const int e2 = mx > 0.f ? 8 - ilogbf(mx) - 1 : 0;
    const float sc = ldexpf(1.f, e2);
    if (c == 0) reinterpret_cast<float*>(img + C::Q_BYTES)[n] = ldexpf(a.qk_scale_log2, -e2);
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t hv = 0, lv = 0;
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const float x0 = f[4 * w + e] * sc, x1 = f[4 * w + e + 1] * sc;
        const uint32_t h2 = f32x2_to_e4m3x2(x0, x1);
        const float r0 = (x0 - e4m3_to_f32(h2)) * 16.f;
        const float r1 = (x1 - e4m3_to_f32(h2 >> 8)) * 16.f;
        hv |= h2 << (8 * e);
        lv |= f32x2_to_e4m3x2(r0, r1) << (8 * e);
      }
      hw[w] = hv;
      lw[w] = lv;
    }
    // operand rows in row-group order (as the in-kernel path writes them)
    const int rh = C::QN_ ? n : 16 * (n >> 3) + (n & 7), rl = rh + 8;
    *reinterpret_cast<uint4*>(img + (rh >> 3) * 1024 + (rh & 7) * 128 + ((c ^ (rh & 7)) << 4)) =
        make_uint4(hw[0], hw[1], hw[2], hw[3]);
    if constexpr (!C::QN_)
      *reinterpret_cast<uint4*>(img + (rl >> 3) * 1024 + (rl & 7) * 128 + ((c ^ (rl & 7)) << 4)) =
          make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

// Host launcher (split_tma.cu): the prologue kernel, then split_tma_kernel
// (its programmatic dependent when pdl). kv: 0 bf16, 1 e4m3; nt: rows per
// CTA; native_qk: FP8 with one-term e4m3 Q; grid: persistent CTAs (at most
// one per SM).
cudaError_t launch_split_tma(int kv, int nt, bool native_qk, const void* k_pages,
                             const void* v_pages, const SplitArgs& a, int grid,
                             cudaStream_t stream, bool pdl);

}  // namespace pda
