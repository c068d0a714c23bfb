// Split-KV paged decode on the 5th-generation tensor cores with TMA-fed
// operands (tcgen05.mma + cp.async.bulk.tensor, 128B swizzle), head_dim 128.
//
// Sources: "b12x 0.30.0, Kernel inventory, Attention table, Paged attention
// row" (bf16 and FP8-E4M3 KV, decode/verify rows, sliding window, split-KV or
// direct output, native FP8 QK option) and "AstrAI commit log,
// attn_paged_decode_split_kv_mma.cuh" (tensor-core GQA head packing,
// multi-stage copy pipeline, predicated partial tiles).
//
// Per CTA: the packed rows of one kv head (NT rows), a 128-token tile at a
// time (the MMA M dimension), S^T = K Q^T and O^T = V^T P^T:
//  * warp 0 (producer): TMA loads of each page segment of the K and V tiles
//    straight into a STAGES-deep ring in the canonical 128B-swizzled UMMA
//    layout (one tensor map per pool: rows = (page, kv head, token), 128
//    elements per row).
//  * warps 1 and 2 (MMA): warp 1 allocates TMEM and issues the S^T MMAs,
//    warp 2 the O^T MMAs, each from one lane as soon as their inputs are
//    ready, with completion signalled by tcgen05.commit. A tcgen05.mma of
//    M=128 costs about 110 cycles of issue latency whatever its N (measured
//    on B200), so the two groups of each tile go out on two issue streams.
//      bf16 K/V: S^T with kind::f16 (bf16) straight from the K stage;
//        O^T with kind::f16 (bf16), A = V^T straight from the V stage
//        (MN-major), B = P^T split into bf16 hi + lo rows (N = 16).
//      FP8 K/V: S^T with kind::f8f6f4 straight from the e4m3 K stage, B =
//        [Q_hi; Q_lo], an exact two-term e4m3 split of each bf16 q row
//        scaled by a power of two; O^T with kind::f16 on V converted to f16
//        by warps 6-9.
//  * warps 3-6 (softmax): thread i = TMEM lane i = token i of S^T and
//    head-dim element i of O^T. Row maxima by redux.sync.max.f32 merged
//    over the four warps; p = exp2(s * c - m) in fp32; P^T to shared memory;
//    O^T folded into fp32 registers with the online-softmax rescale. On tiles
//    with keys that no row may see they also zero those keys' V rows in the
//    stage (bf16), so NaN bytes never meet a zero weight in the MMA.
//  * warps 7-10 (FP8 only, converters): V stage e4m3 -> f16 operand tile.
//  * The producer warp loads the next tile's page ids across its lanes while
//    the current tile's copies are in flight.
//  * Every wait is bounded; group exits go through bar.red.and.
#pragma once

#include <cuda.h>

#include "pda_device.cuh"
#include "split_fma.cuh"  // SplitArgs, row_range
#include "tcgen05.cuh"    // descriptors, MMA issue, TMEM loads, barriers

namespace pda {

template <int KV, int NT>
struct TmaCfg {
  static constexpr bool BF16 = KV == 0;
  static constexpr int D = 128;
  static constexpr int TILE = 128;
  static constexpr int ELT = BF16 ? 2 : 1;
  static constexpr int N1 = BF16 ? 16 : 2 * NT;  // S^T columns
  static constexpr int N2 = BF16 ? 16 : NT;      // O^T columns
  static constexpr int STAGES = BF16 ? 3 : 4;
  static constexpr int KT = TILE * D * ELT;      // bytes of one K (or V) tile
  static constexpr int STAGE = 2 * KT;           // K then V
  static constexpr int HALF = TILE * 128;        // one 128-byte column of SW128 atoms
  static constexpr int VC = TILE * D * 2;        // converted f16 V tile (FP8 only)
  static constexpr int NVC = BF16 ? 0 : 2;
  static constexpr int Q_ROWS = N1;
  static constexpr int Q_BYTES = Q_ROWS * D * (BF16 ? 2 : 1);
  static constexpr int Q_HALF = (Q_ROWS / 8) * 1024;  // bf16: 64-element half of each row
  static constexpr int P_ROW = N2 * 2;                 // bytes per token row of P^T
  static constexpr int P_SBO = 8 * P_ROW;
  static constexpr int P_BYTES = (TILE / 8) * P_SBO;
  static constexpr uint32_t P_SWIZZLE = P_ROW == 64 ? 4u : 6u;  // SW64 / SW32
  static constexpr int SOFT0 = 3;                      // first softmax warp
  static constexpr int CONV0 = 7;                      // first converter warp
  static constexpr int WARPS = BF16 ? 7 : 11;
  static constexpr int THREADS = WARPS * 32;
  // shared memory map (1024-aligned where swizzled)
  static constexpr int OFF_STAGE = 0;
  static constexpr int OFF_VC = OFF_STAGE + STAGES * STAGE;
  static constexpr int OFF_Q = OFF_VC + NVC * VC;
  static constexpr int OFF_P = OFF_Q + ((Q_BYTES + 1023) / 1024) * 1024;
  static constexpr int OFF_WMAX = OFF_P + 2 * ((P_BYTES + 1023) / 1024) * 1024;
  static constexpr int P_BUF = ((P_BYTES + 1023) / 1024) * 1024;
  static constexpr int OFF_CSM = OFF_WMAX + 4 * 32 * 4;  // {score scale, -m} per row
  static constexpr int OFF_ALPHA = OFF_CSM + 2 * 32 * 4;
  static constexpr int OFF_CS = OFF_ALPHA + 2 * 32 * 4;   // per-row score scale
  static constexpr int OFF_MRAW = OFF_CS + 32 * 4;       // running max per row
  static constexpr int OFF_THR = OFF_MRAW + 32 * 4;      // rescale threshold per row
  static constexpr int OFF_LRED = OFF_THR + 32 * 4;
  static constexpr int OFF_INV = OFF_LRED + 4 * 32 * 4;  // v_scale / l per row
  static constexpr int OFF_ROWS = OFF_INV + 32 * 4;      // output row of each packed row
  static constexpr int OFF_RANGE = OFF_ROWS + 32 * 8;
  // page ids of upcoming tiles: PID_SLOTS tiles x 16 segments, filled by
  // cp.async PID_AHEAD tiles ahead of the copies that use them
  static constexpr int PID_SLOTS = 8, PID_AHEAD = 4;
  static constexpr int OFF_PIDS = OFF_RANGE + 32 * 8;
  static constexpr int OFF_BAR = OFF_PIDS + PID_SLOTS * 16 * 4;
  // full[S], empty[S], s_full[2], p_ready[2], o_full[2], o_free[2], v_ready[2]
  static constexpr int NUM_BARS = 2 * STAGES + 10;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_FLAGS = OFF_TMEM_SLOT + 8;
  static constexpr int SMEM = OFF_FLAGS + 8;
  static constexpr int SMEM_ALLOC = SMEM + 4096;  // slack: no operand read leaves the CTA
  static constexpr int TMEM_COLS = 2 * N1 + 2 * N2 <= 64 ? 64 : (2 * N1 + 2 * N2 <= 128 ? 128 : 256);
  static constexpr int COL_S = 0, COL_O = 2 * N1;
  static_assert(BF16 ? (NT == 4 || NT == 8) : (NT == 16 || NT == 32), "rows per CTA");
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory");
  static_assert(OFF_VC % 1024 == 0 && OFF_Q % 1024 == 0 && OFF_P % 1024 == 0, "alignment");
};

// Instruction descriptor, kind::f8f6f4 with e4m3 A and B, fp32 D, K-major.
__host__ __device__ constexpr uint32_t umma_idesc_e4m3(int M, int N) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
// kind::f16 with bf16 A and B.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
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
__device__ __forceinline__ void tmem_ld32_raw(uint32_t taddr, float* v) {
  float (&vv)[32] = *reinterpret_cast<float(*)[32]>(v);
  tmem_ld32(taddr, vv);
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

__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code & 0xFF), __NV_E4M3);
  return __half2float(*reinterpret_cast<const __half*>(&h));
}

template <int KV, int NT>
__global__ void __launch_bounds__(TmaCfg<KV, NT>::THREADS, 1)
    split_tma_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                     const SplitArgs a) {
  using C = TmaCfg<KV, NT>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int rt = blockIdx.x;
  const int split = blockIdx.y % a.num_splits;
  const int kvh = blockIdx.y / a.num_splits;
  const int b = blockIdx.z;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                       // [S] TMA landed
  uint64_t* empty = bars + C::STAGES;          // [S] stage consumed
  uint64_t* s_full = bars + 2 * C::STAGES;     // [2]
  uint64_t* p_ready = s_full + 2;              // [2]
  uint64_t* o_full = s_full + 4;               // [2]
  uint64_t* o_free = s_full + 6;               // [2]
  uint64_t* v_ready = s_full + 8;              // [2] (FP8)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);
  float* sm_cs = reinterpret_cast<float*>(smem + C::OFF_CS);

  // ---- key range of this CTA (tiles of 128 tokens) -------------------------
  int L = __ldg(a.kv_lens + b);
  const int Lmax = a.max_pages << a.log2_page;
  if (L < 0 || L > Lmax) {
    if (tid == 0) record_error_at(a.err, kErrBadPage);
    L = L < 0 ? 0 : Lmax;
  }
  const int R0 = rt * NT;
  const int Rlast = min(a.M, R0 + NT) - 1;
  int lo_u, hi_u, lo_x, hi_x;
  row_range(a, L, R0 / a.G, lo_u, hi_x);
  row_range(a, L, Rlast / a.G, lo_x, hi_u);
  const int k_begin = lo_u / C::TILE;
  const int k_end = hi_u > lo_u ? (hi_u + C::TILE - 1) / C::TILE : k_begin;
  const int n_all = k_end - k_begin;
  const int chunk = (n_all + a.num_splits - 1) / a.num_splits;
  const int c0 = min(n_all, split * chunk);
  int ntiles = min(n_all, c0 + chunk) - c0;
  const int kfirst = k_begin + c0;
  if ((smem_addr(smem) & 1023u) != 0) {  // swizzle atoms need 1024-byte alignment
    if (tid == 0) record_error_at(a.err, kErrUnsupported);
    ntiles = 0;
  }

  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::BF16 ? 1 : 2);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], 128);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], 128);
      mbar_init(&v_ready[i], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // ---- TMA producer state (warp 0). Lane g holds the page id of segment g
  // of a tile (a tile of 128 tokens spans at most 16 pages of >= 8 tokens).
  const int seq_pages = (L + a.page_size - 1) >> a.log2_page;
  const int32_t* pt_row = a.page_table + (long long)b * a.max_pages;
  const int seg_rows = a.page_size < C::TILE ? a.page_size : C::TILE;
  auto nseg_of = [&](int n) {
    const int first = ((kfirst + n) * C::TILE) >> a.log2_page;
    return a.page_size >= C::TILE ? 1 : min(C::TILE >> a.log2_page, seq_pages - first);
  };
  // Page ids reach shared memory by 4-byte cp.async, one commit group per
  // tile, PID_AHEAD tiles before they are used: the producer never waits on
  // a global load of the page table (a register hand-off would stall on the
  // load's full latency every tile).
  int32_t* sm_pids = reinterpret_cast<int32_t*>(smem + C::OFF_PIDS);
  auto prefetch_pids = [&](int n) {
    if (n < ntiles && lane < nseg_of(n)) {
      const int32_t* src = pt_row + (((kfirst + n) * C::TILE) >> a.log2_page) + lane;
      const uint32_t dst = smem_addr(sm_pids + (n % C::PID_SLOTS) * 16 + lane);
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  auto read_pid = [&](int n) -> int {  // after tile n's group completed
    if (lane >= nseg_of(n)) return 0;
    int pid = sm_pids[(n % C::PID_SLOTS) * 16 + lane];
    if ((unsigned)pid >= (unsigned)a.num_pages) {
      record_error_at(a.err, kErrBadPage);
      pid = 0;
    }
    return pid;
  };
  int p_issued = 0;
  // Issue tiles [p_issued, n_end): wait for the stage to be free, set the
  // transaction count, then lane g copies segment g (K and V, both halves
  // of each row for bf16) so the copies of a tile go out together.
  auto produce = [&](int n_end) {
    const uint32_t sbase = smem_addr(smem);
    for (int n = p_issued; n < n_end; ++n) {
      // groups complete in order: at most PID_AHEAD - 1 younger than tile n
      asm volatile("cp.async.wait_group %0;" ::"n"(C::PID_AHEAD - 1) : "memory");
      __syncwarp();
      const int pid_cur = read_pid(n);
      __syncwarp();  // slot n % PID_SLOTS is read before it can be refilled
      prefetch_pids(n + C::PID_AHEAD);
      const int st = n % C::STAGES;
      bool ok = !*abort_flag;
      if (ok && n >= C::STAGES) ok = mbar_wait(&empty[st], ((n / C::STAGES) - 1) & 1, a.err);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      const int tok0 = (kfirst + n) * C::TILE;
      const int nseg = nseg_of(n);
      const uint32_t seg_bytes = (uint32_t)seg_rows * 128u * (C::BF16 ? 2u : 1u);
      const uint32_t kdst = sbase + C::OFF_STAGE + st * C::STAGE;
      const uint32_t vdst = kdst + C::KT;
      if (lane == 0) mbar_arrive_expect_tx(&full[st], 2u * seg_bytes * (uint32_t)nseg);
      __syncwarp();  // the transaction count is set before any copy completes
      if (lane < nseg) {
        const int row = (pid_cur * a.Hkv + kvh) * a.page_size +
                        (a.page_size >= C::TILE ? (tok0 & (a.page_size - 1)) : 0);
        const uint32_t off = (uint32_t)lane * seg_rows * 128u;
        tma_load_2d(kdst + off, &tmk, 0, row, &full[st]);
        tma_load_2d(vdst + off, &tmv, 0, row, &full[st]);
        if constexpr (C::BF16) {
          tma_load_2d(kdst + C::HALF + off, &tmk, 64, row, &full[st]);
          tma_load_2d(vdst + C::HALF + off, &tmv, 64, row, &full[st]);
        }
      }
      p_issued = n + 1;
    }
  };
  if (warp == 0) {
    // The first STAGES tiles need no free stage: issue them now, so their
    // page-table reads and copies overlap the Q set-up of the other warps.
    __syncwarp();  // barrier init (lane 0) is ordered before the copies
    if (ntiles > 0) {
      if (lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmk) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmv) : "memory");
      }
      for (int n = 0; n < C::PID_AHEAD; ++n) prefetch_pids(n);
      produce(min(C::STAGES, ntiles));
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }

  // ---- Q operand (softmax warps), before the first barrier ----------------
  if (warp >= C::SOFT0 && warp < C::SOFT0 + 4) {
    const int i = tid - C::SOFT0 * 32;  // 0..127
    if constexpr (C::BF16) {
      // Q_ROWS = 16 rows (rows >= NT zero), bf16, SW128 K-major: 16 chunks
      // of 8 elements per row, chunk j in half j/8.
      for (int c = i; c < C::Q_ROWS * 16; c += 128) {
        const int n = c % C::Q_ROWS, j = c / C::Q_ROWS;
        const int R = R0 + n;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (n < NT && R < a.M) {
          const int qi = R / a.G, h = kvh * a.G + R % a.G;
          u = __ldg(reinterpret_cast<const uint4*>(
              a.q + ((long long)(b * a.Lq + qi) * a.Hq + h) * C::D + j * 8));
        }
        *reinterpret_cast<uint4*>(smem + C::OFF_Q + (j >> 3) * C::Q_HALF + (n >> 3) * 1024 +
                                  (n & 7) * 128 + (((j & 7) ^ (n & 7)) << 4)) = u;
      }
      if (i < 32) sm_cs[i] = a.qk_scale_log2;
    } else {
      // Rows hi (0..NT-1) and lo (NT..2NT-1) in e4m3, one 128-byte row each,
      // SW128 K-major. Four threads share a row (32 elements each).
      const int n = i >> 2, part = i & 3;
      const int R = R0 + n;
      float f[32];
      float mx = 0.f;
      if (n < NT && R < a.M) {
        const int qi = R / a.G, h = kvh * a.G + R % a.G;
        const uint16_t* src = a.q + ((long long)(b * a.Lq + qi) * a.Hq + h) * C::D + part * 32;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(src + k * 8));
          float g[8];
          bf16x8_to_f32(u, g);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            f[8 * k + e] = g[e];
            mx = fmaxf(mx, fabsf(g[e]));
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) f[e] = 0.f;
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
      // power-of-two scale 2^e with max|q| * 2^e <= 448: q * 2^e stays exact
      int e2 = 0;
      if (mx > 0.f) {
        e2 = 8 - ilogbf(mx) - 1;  // 2^(ilogb+1) > mx, so mx * 2^e2 < 2^8 = 256 <= 448
      }
      const float sc = ldexpf(1.f, e2);
      if (n < NT && part == 0) sm_cs[n] = ldexpf(a.qk_scale_log2, -e2);
      if (n < NT) {
        uint32_t hiw[8], low[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          uint32_t hw = 0, lw = 0;
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            const float x0 = f[4 * k + e] * sc, x1 = f[4 * k + e + 1] * sc;
            const uint32_t h2 = f32x2_to_e4m3x2(x0, x1);
            const float r0 = (x0 - e4m3_to_f32(h2)) * 16.f;
            const float r1 = (x1 - e4m3_to_f32(h2 >> 8)) * 16.f;
            const uint32_t l2 = f32x2_to_e4m3x2(r0, r1);
            hw |= h2 << (8 * e);
            lw |= l2 << (8 * e);
          }
          hiw[k] = hw;
          low[k] = lw;
        }
        // this thread's 32 bytes are chunks 2*part, 2*part+1 of the row
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int ch = 2 * part + cc;
          const uint4 hv = make_uint4(hiw[4 * cc], hiw[4 * cc + 1], hiw[4 * cc + 2], hiw[4 * cc + 3]);
          const uint4 lv = make_uint4(low[4 * cc], low[4 * cc + 1], low[4 * cc + 2], low[4 * cc + 3]);
          const int rh = n, rl = NT + n;
          *reinterpret_cast<uint4*>(smem + C::OFF_Q + (rh >> 3) * 1024 + (rh & 7) * 128 +
                                    ((ch ^ (rh & 7)) << 4)) = hv;
          *reinterpret_cast<uint4*>(smem + C::OFF_Q + (rl >> 3) * 1024 + (rl & 7) * 128 +
                                    ((ch ^ (rl & 7)) << 4)) = lv;
        }
      }
    }
    if constexpr (C::BF16) {
      // P^T rows >= 2*NT stay zero for the whole kernel
      for (int c = i; c < 2 * C::P_BUF / 16; c += 128)
        reinterpret_cast<uint4*>(smem + C::OFF_P)[c] = make_uint4(0, 0, 0, 0);
    }
    if (i < 32) {  // rows start with no finite score: m = -inf, p = 0
      reinterpret_cast<float2*>(smem + C::OFF_CSM)[i] = make_float2(1.f, 0.f);
      reinterpret_cast<float*>(smem + C::OFF_MRAW)[i] = -INFINITY;
      reinterpret_cast<float*>(smem + C::OFF_THR)[i] = -INFINITY;
    }
    // visible key range of each row of the tile, read on boundary tiles
    int2* rng = reinterpret_cast<int2*>(smem + C::OFF_RANGE);
    if (i < NT) {
      const int R = R0 + i;
      int lo = 0, hi = 0;
      long long row = -1;  // output row [b, qi, h] of packed row R (-1: padding)
      if (R < a.M) {
        const int qi = R / a.G;
        row_range(a, L, qi, lo, hi);
        row = (long long)(b * a.Lq + qi) * a.Hq + kvh * a.G + (R - qi * a.G);
      }
      rng[i] = make_int2(lo, hi);
      reinterpret_cast<long long*>(smem + C::OFF_ROWS)[i] = row;
    }
    fence_proxy_async_smem();  // Q and P^T zeros are read by the tensor core
  }
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ======================= TMA producer (whole warp) ======================
    // Tiles [0, STAGES) went out before the CTA-wide barrier.
    produce(ntiles);
    asm volatile("cp.async.wait_all;" ::: "memory");  // none left in flight at exit
    if (lane == 0 && *abort_flag) {
      for (int n = max(0, p_issued - C::STAGES); n < p_issued; ++n)
        mbar_wait(&full[n % C::STAGES], (n / C::STAGES) & 1, a.err, kWaitTimeoutCycles / 16);
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ======================= MMA issuers: S^T (warp 1), O^T (warp 2) ========
    if (lane == 0) {
      const uint32_t sbase = smem_addr(smem);
      bool ok = true;
      int issued = 0;
      if (warp == 1) {
        for (int k = 0; k < ntiles; ++k) {
          const int bb = k & 1;
          ok = !*abort_flag && mbar_wait(&full[k % C::STAGES], (k / C::STAGES) & 1, a.err);
          if (ok && k >= 2) ok = mbar_wait(&p_ready[bb], ((k - 2) >> 1) & 1, a.err);
          if (!ok) break;
          tmem_fence_after();
          const uint32_t ka = sbase + C::OFF_STAGE + (k % C::STAGES) * C::STAGE;
          const uint32_t qa = sbase + C::OFF_Q;
          const uint32_t d = tmem + C::COL_S + bb * C::N1;
          if constexpr (C::BF16) {
            constexpr uint32_t idesc = umma_idesc_bf16(128, C::N1, false, false);
#pragma unroll
            for (int s = 0; s < C::D / 16; ++s)
              umma_f16(d, umma_desc(ka + (s >> 2) * C::HALF + (s & 3) * 32, 16, 1024, kSw128),
                       umma_desc(qa + (s >> 2) * C::Q_HALF + (s & 3) * 32, 16, 1024, kSw128),
                       idesc, s > 0);
          } else {
            constexpr uint32_t idesc = umma_idesc_e4m3(128, C::N1);
#pragma unroll
            for (int s = 0; s < C::D / 32; ++s)
              umma_f8(d, umma_desc(ka + s * 32, 16, 1024, kSw128),
                      umma_desc(qa + s * 32, 16, 1024, kSw128), idesc, s > 0);
            umma_commit(&empty[k % C::STAGES]);  // the K half of the stage is consumed
          }
          umma_commit(&s_full[bb]);
          issued = k + 1;
        }
        if (!ok) *abort_flag = 1;
        if (*abort_flag && issued > 0)  // MMAs already issued finish before TMEM is freed
          mbar_wait(&s_full[(issued - 1) & 1], ((issued - 1) >> 1) & 1, a.err,
                    kWaitTimeoutCycles / 16);
      } else {
        for (int k = 0; k < ntiles; ++k) {
          const int bb = k & 1;
          ok = !*abort_flag && mbar_wait(&p_ready[bb], (k >> 1) & 1, a.err);
          if (ok && k >= 2) ok = mbar_wait(&o_free[bb], ((k - 2) >> 1) & 1, a.err);
          if constexpr (!C::BF16) {
            if (ok) ok = mbar_wait(&v_ready[bb], (k >> 1) & 1, a.err);
          }
          if (!ok) break;
          tmem_fence_after();
          const uint32_t pa = sbase + C::OFF_P + bb * C::P_BUF;
          const uint32_t d = tmem + C::COL_O + bb * C::N2;
          if constexpr (C::BF16) {
            constexpr uint32_t idesc = umma_idesc_bf16(128, C::N2, true, true);
            const uint32_t va = sbase + C::OFF_STAGE + (k % C::STAGES) * C::STAGE + C::KT;
#pragma unroll
            for (int s = 0; s < C::TILE / 16; ++s)
              umma_f16(d, umma_desc(va + s * 2048, C::HALF, 1024, kSw128),
                       umma_desc(pa + s * 2 * C::P_SBO, C::P_BYTES, C::P_SBO, C::P_SWIZZLE),
                       idesc, s > 0);
            umma_commit(&empty[k % C::STAGES]);  // K and V of the stage are consumed
          } else {
            constexpr uint32_t idesc = umma_idesc_f16(128, C::N2, true, true);
            const uint32_t va = sbase + C::OFF_VC + bb * C::VC;
#pragma unroll
            for (int s = 0; s < C::TILE / 16; ++s)
              umma_f16(d, umma_desc(va + s * 2048, C::HALF, 1024, kSw128),
                       umma_desc(pa + s * 2 * C::P_SBO, C::P_BYTES, C::P_SBO, C::P_SWIZZLE),
                       idesc, s > 0);
          }
          umma_commit(&o_full[bb]);
          issued = k + 1;
        }
        if (!ok) *abort_flag = 1;
        if (*abort_flag && issued > 0)
          mbar_wait(&o_full[(issued - 1) & 1], ((issued - 1) >> 1) & 1, a.err,
                    kWaitTimeoutCycles / 16);
      }
    }
    __syncwarp();
  } else if (warp >= C::SOFT0 && warp < C::SOFT0 + 4) {
    // ======================= softmax / accumulate ===========================
    const int q4 = warp & 3;
    const int i = 32 * q4 + lane;  // TMEM lane: token of S^T, element of O^T
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    float* wmax = reinterpret_cast<float*>(smem + C::OFF_WMAX);
    float2* sm_csm = reinterpret_cast<float2*>(smem + C::OFF_CSM);
    float* sm_thr = reinterpret_cast<float*>(smem + C::OFF_THR);
    float* sm_alpha = reinterpret_cast<float*>(smem + C::OFF_ALPHA);
    float* sm_mraw = reinterpret_cast<float*>(smem + C::OFF_MRAW);  // running max (-inf at start)
    const int2* rng = reinterpret_cast<const int2*>(smem + C::OFF_RANGE);
    uint32_t resc = 0;  // bit (k & 1): tile k rescaled the running max
    float l_part[NT], acc[NT];
#pragma unroll
    for (int r = 0; r < NT; ++r) {
      l_part[r] = 0.f;
      acc[r] = 0.f;
    }
    bool ok = true;

    auto accumulate = [&](int k) -> bool {
      const int bb = k & 1;
      const bool ok_w = __all_sync(0xFFFFFFFFu, mbar_wait(&o_full[bb], (k >> 1) & 1, a.err));
      if (!ok_w) return false;
      tmem_fence_after();
      float o[C::N2];
      if constexpr (C::N2 == 16) {
        tmem_ld16_raw(tmem + lane_off + C::COL_O + bb * C::N2, o);
      } else {
        tmem_ld32_raw(tmem + lane_off + C::COL_O + bb * C::N2, o);
      }
      tmem_fence_before();
      mbar_arrive(&o_free[bb]);
      const float* al = sm_alpha + bb * 32;
      const bool rs = (resc >> bb) & 1u;
#pragma unroll
      for (int r = 0; r < NT; ++r) {
        const float ov = C::BF16 ? o[r] + o[NT + r] : o[r];  // P = P_hi + P_lo
        acc[r] = rs ? fmaf(acc[r], al[r], ov) : acc[r] + ov;
      }
      return true;
    };

    bool acc_ok = true;
    for (int n = 0; n < ntiles; ++n) {
      const int bb = n & 1;
      bool ok_s = acc_ok && !*abort_flag;
      if (ok_s) ok_s = mbar_wait(&s_full[bb], (n >> 1) & 1, a.err);
      ok_s = __all_sync(0xFFFFFFFFu, ok_s);
      float sraw[C::N1];
      if (ok_s) {
        tmem_fence_after();
        const uint32_t ta = tmem + lane_off + C::COL_S + bb * C::N1;
        if constexpr (C::N1 == 16) {
          tmem_ld16_raw(ta, sraw);
        } else {
#pragma unroll
          for (int c = 0; c < C::N1 / 32; ++c) tmem_ld32_raw(ta + 32 * c, sraw + 32 * c);
        }
      } else {
#pragma unroll
        for (int r = 0; r < C::N1; ++r) sraw[r] = -INFINITY;
      }
      float* s = sraw;  // scores (then probabilities) overwrite the raw columns
      if constexpr (!C::BF16) {
#pragma unroll
        for (int r = 0; r < NT; ++r) s[r] = fmaf(sraw[NT + r], 0.0625f, sraw[r]);  // S_hi + S_lo/16
      }
      const int t0 = (kfirst + n) * C::TILE;
      const int j = t0 + i;
      const bool clean = t0 >= lo_x && t0 + C::TILE <= hi_x;
      if (!clean) {
#pragma unroll
        for (int r = 0; r < NT; ++r) {
          const int2 lh = rng[r];
          if (!(j >= lh.x && j < lh.y)) s[r] = -INFINITY;
        }
        if constexpr (C::BF16) {
          if (j < lo_u || j >= hi_u) {  // zero V row i of the stage (2 halves)
            uint8_t* vrow = smem + C::OFF_STAGE + (n % C::STAGES) * C::STAGE + C::KT + i * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              *reinterpret_cast<uint4*>(vrow + c * 16) = make_uint4(0, 0, 0, 0);
              *reinterpret_cast<uint4*>(vrow + C::HALF + c * 16) = make_uint4(0, 0, 0, 0);
            }
          }
        }
      }
      // Lazy rescale: the running max m of each row (log2 domain) only moves
      // when a score exceeds it by more than kRescaleLog2, so p = exp2(x - m)
      // stays <= 2^kRescaleLog2 (well inside f16) and most tiles skip the
      // per-tile max exchange. The test runs on raw scores against
      // thr = (m + kRescaleLog2) / cs (-inf until the row's first finite
      // score), so it is one compare per score.
      constexpr float kRescaleLog2 = 8.f;
      bool want = false;
#pragma unroll
      for (int r = 0; r < NT; r += 4) {
        const float4 t = reinterpret_cast<const float4*>(sm_thr)[r / 4];
        want = want | (s[r] > t.x) | (s[r + 1] > t.y) | (s[r + 2] > t.z) | (s[r + 3] > t.w);
      }
      // one barrier decides for the whole tile (and propagates failures)
      const bool flag = named_bar_or_and(2, 128, want, ok_s, &ok_s);
      if (!ok_s) {
        ok = false;
        break;
      }
      resc = (resc & ~(1u << bb)) | ((uint32_t)flag << bb);
      if (flag) {
#pragma unroll
        for (int r = 0; r < NT; ++r) {
          const float wm = redux_max(s[r]);
          if (lane == r) wmax[q4 * 32 + r] = wm;
        }
        named_bar(2, 128);
        if (i < NT) {
          const float cs = sm_cs[i];
          const float st = fmaxf(fmaxf(wmax[i], wmax[32 + i]), fmaxf(wmax[64 + i], wmax[96 + i]));
          const float m_old = sm_mraw[i];
          const float m_new = fmaxf(m_old, st * cs);  // -inf stays -inf (cs > 0)
          const float m_use = m_new == -INFINITY ? 0.f : m_new;
          sm_alpha[bb * 32 + i] = m_old == -INFINITY ? 0.f : fast_exp2(m_old - m_use);
          sm_mraw[i] = m_new;
          sm_csm[i] = make_float2(cs, -m_use);
          sm_thr[i] = m_new == -INFINITY ? -INFINITY : (m_use + kRescaleLog2) / cs;
        }
        named_bar(2, 128);
#pragma unroll
        for (int r = 0; r < NT; ++r) l_part[r] *= sm_alpha[bb * 32 + r];
      }
      float* p = s;
#pragma unroll
      for (int r = 0; r < NT; r += 2) {
        const float4 c = reinterpret_cast<const float4*>(sm_csm)[r / 2];
        p[r] = fast_exp2(fmaf(s[r], c.x, c.y));
        p[r + 1] = fast_exp2(fmaf(s[r + 1], c.z, c.w));
        l_part[r] += p[r];
        l_part[r + 1] += p[r + 1];
      }
      // P^T row of token i (row-major over the N2 columns, swizzled chunks)
      uint8_t* sp = smem + C::OFF_P + bb * C::P_BUF + (i >> 3) * C::P_SBO + (i & 7) * C::P_ROW;
      const int pswz = C::P_ROW == 64 ? ((i & 7) >> 1) & 3 : ((i & 7) >> 2) & 1;
      if constexpr (C::BF16) {
        // columns 0..NT-1: bf16(p); NT..2NT-1: bf16(p - bf16(p)); rest stay 0
        uint32_t w[NT];  // NT/2 words of hi, then NT/2 of lo
#pragma unroll
        for (int r = 0; r < NT; r += 2) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(p[r], p[r + 1]);
          const float2 hf = __bfloat1622float2(h);
          w[r / 2] = *reinterpret_cast<const uint32_t*>(&h);
          w[NT / 2 + r / 2] = pack_bf16x2(p[r] - hf.x, p[r + 1] - hf.y);
        }
        if constexpr (NT == 8) {
          *reinterpret_cast<uint4*>(sp + ((0 ^ pswz) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(sp + ((1 ^ pswz) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
        } else {
          *reinterpret_cast<uint4*>(sp + ((0 ^ pswz) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      } else {
#pragma unroll
        for (int g = 0; g < NT / 8; ++g) {
          uint4 w;
          w.x = pack_f16x2(p[8 * g + 0], p[8 * g + 1]);
          w.y = pack_f16x2(p[8 * g + 2], p[8 * g + 3]);
          w.z = pack_f16x2(p[8 * g + 4], p[8 * g + 5]);
          w.w = pack_f16x2(p[8 * g + 6], p[8 * g + 7]);
          *reinterpret_cast<uint4*>(sp + ((g ^ pswz) << 4)) = w;
        }
      }
      fence_proxy_async_smem();
      tmem_fence_before();
      mbar_arrive(&p_ready[bb]);
      if (n >= 1) acc_ok = accumulate(n - 1);
    }
    if (__all_sync(0xFFFFFFFFu, ok && ntiles > 0 && acc_ok && !*abort_flag))
      acc_ok = accumulate(ntiles - 1);
    ok = named_bar_and(2, 128, ok && acc_ok);
    if (!ok) *abort_flag = 1;

    // ---- epilogue --------------------------------------------------------
#pragma unroll
    for (int r = 0; r < NT; ++r) {
      float v = l_part[r];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
      l_part[r] = v;
    }
    float* lred = reinterpret_cast<float*>(smem + C::OFF_LRED);
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < NT; ++r) lred[q4 * 32 + r] = l_part[r];
    }
    named_bar(2, 128);
    // One thread per row: normaliser, lse; then all threads store O rows.
    // Row offsets come from shared memory: per-row index arithmetic here
    // (a runtime division per row) made the store loop latency-bound.
    const bool failed = !ok;
    const long long rows_total = (long long)a.B * a.Lq * a.Hq;
    const long long* rows = reinterpret_cast<const long long*>(smem + C::OFF_ROWS);
    float* sm_inv = reinterpret_cast<float*>(smem + C::OFF_INV);
    if (i < NT) {
      const float lt = lred[i] + lred[32 + i] + lred[64 + i] + lred[96 + i];
      const bool live = lt > 0.f && !failed;
      sm_inv[i] = live ? a.v_scale / lt : 0.f;
      const long long row = rows[i];
      if (row >= 0) {
        const float res = live ? (log2f(lt) - sm_csm[i].y) * 0.69314718055994531f : -INFINITY;
        if (a.num_splits == 1) {
          if (a.lse) a.lse[row] = res;
        } else {
          a.lse_part[(long long)split * rows_total + row] = res;
        }
      }
    }
    named_bar(2, 128);
    float* dst = a.num_splits == 1 ? a.out : a.o_part + (long long)split * rows_total * C::D;
#pragma unroll
    for (int r = 0; r < NT; ++r) {
      const long long row = rows[r];
      if (row >= 0) dst[row * C::D + i] = acc[r] * sm_inv[r];
    }
  } else if constexpr (!C::BF16) {
    // ======================= V converters (FP8) ============================
    const int t = tid - C::CONV0 * 32;  // token 0..127
    for (int n = 0; n < ntiles; ++n) {
      const int st = n % C::STAGES;
      const int bb = n & 1;
      bool ok = !*abort_flag;
      if (ok) ok = mbar_wait(&full[st], (n / C::STAGES) & 1, a.err);
      if (ok && n >= 2) ok = mbar_wait(&o_full[bb], ((n - 2) >> 1) & 1, a.err);
      uint4 raw[8];
      if (ok) {
        const uint8_t* vrow = smem + C::OFF_STAGE + st * C::STAGE + C::KT + (t >> 3) * 1024 + (t & 7) * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          raw[c] = *reinterpret_cast<const uint4*>(vrow + ((c ^ (t & 7)) << 4));
      }
      if (!named_bar_and(1, 128, ok)) {
        *abort_flag = 1;
        break;
      }
      if (t == 0) mbar_arrive(&empty[st]);  // the V half of the stage is consumed
      const int j = (kfirst + n) * C::TILE + t;
      const bool v_zero = j < lo_u || j >= hi_u;
      uint8_t* dst = smem + C::OFF_VC + bb * C::VC + (t >> 3) * 1024 + (t & 7) * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {  // 16 e4m3 -> two 8-element f16 chunks
        const int j0 = 2 * c, j1 = 2 * c + 1;
        const uint4 f0 = v_zero ? make_uint4(0, 0, 0, 0) : e4m3x8_to_f16x8(make_uint2(raw[c].x, raw[c].y));
        const uint4 f1 = v_zero ? make_uint4(0, 0, 0, 0) : e4m3x8_to_f16x8(make_uint2(raw[c].z, raw[c].w));
        *reinterpret_cast<uint4*>(dst + (j0 >> 3) * C::HALF + (((j0 & 7) ^ (t & 7)) << 4)) = f0;
        *reinterpret_cast<uint4*>(dst + (j1 >> 3) * C::HALF + (((j1 & 7) ^ (t & 7)) << 4)) = f1;
      }
      fence_proxy_async_smem();
      mbar_arrive(&v_ready[bb]);
    }
  }

  pdl_launch_dependents();
  tmem_fence_before();
  __syncthreads();
  if (warp == 1) {
    tmem_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::TMEM_COLS)
                 : "memory");
  }
}

// Host launcher (split_tma.cu). kv: 0 bf16, 1 e4m3; nt: rows per CTA.
cudaError_t launch_split_tma(int kv, int nt, const void* k_pages, const void* v_pages,
                             const SplitArgs& a, dim3 grid, cudaStream_t stream);

}  // namespace pda
