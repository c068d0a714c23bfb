// Split-KV paged decode kernel on the 5th-generation tensor cores (tcgen05),
// for FP8-E4M3 K/V with head_dim 128 and enough packed rows per kv head
// (M = G * q_len, up to NT = 32 per CTA) that QK^T and PV are real dense
// contractions: per 128-token tile, S^T = K Q^T is 128 x NT x 128 and
// O^T = V^T P^T is 128 x NT x 128.
//
// Sources: "b12x 0.30.0, Kernel inventory, Attention table, Paged attention
// row" (FP8-E4M3 KV decode and verify rows, sliding window, split-KV or
// direct output) and "AstrAI commit log, attn_paged_decode_split_kv_mma.cuh"
// (tensor-core GQA head packing, multi-stage copy pipeline, predicated
// partial tiles).
//
// B200 design (one CTA per SM, 9 warps):
//  * warps 0-3, converters: a 2-stage ring of raw FP8 tiles (128 tokens of K
//    and of V, bulk-copied from contiguous (page, head) blocks; thread 0 is
//    the copy producer). Each thread owns one token: it reads its 128-byte K
//    and V rows, converts e4m3 -> f16 (exact) and writes them in the
//    canonical no-swizzle UMMA layout into double-buffered K and V tiles. V
//    rows of keys that no row may see are written as zeros, so NaN bytes in
//    unused slots never reach P.V.
//  * warp 8, MMA issuer (one lane): per tile, 8 tcgen05.mma (K = 16 each) for
//    S^T = K Q^T into a TMEM accumulator, and after softmax 8 more for
//    O^T = V^T P^T into another (both double buffered in TMEM), each
//    completion signalled by tcgen05.commit to an mbarrier.
//  * warps 4-7, softmax: thread i owns TMEM lane i, i.e. token i of S^T and
//    head-dim element i of O^T. Row maxima over the tile's tokens come from
//    one redux.sync.max.f32 per row and warp, merged over the 4 warps in
//    shared memory; p = exp2(s * c - m) in fp32, written to shared memory as
//    f16 (P^T, the B operand of PV); O^T tiles are read back from TMEM and
//    folded into fp32 registers with the online-softmax rescale.
//  * Precision: K, V exact in f16 (e4m3 -> f16 is exact); Q rounded bf16 ->
//    f16 (exact for |q| in [2^-14, 65504]); P in f16 (relative 2^-11); all
//    accumulation in fp32; the softmax scale and kv_scale are applied in
//    fp32 outside the MMAs.
//  * Every wait is a bounded mbarrier wait; on expiry the CTA records
//    PDA_ERR_TIMEOUT, stops its loops, drains and frees its TMEM.
#pragma once

#include "pda_device.cuh"
#include "split_fma.cuh"  // SplitArgs, row_range

namespace pda {

template <int NT>
struct TcCfg {
  static constexpr int D = 128;
  static constexpr int TILE = 128;                   // tokens per tile (MMA M)
  static constexpr int CONV_WARPS = 4, SOFT_WARPS = 4;
  static constexpr int MMA_WARP = CONV_WARPS + SOFT_WARPS;
  static constexpr int THREADS = (CONV_WARPS + SOFT_WARPS + 1) * 32;
  static constexpr int RAW_STAGES = 2;
  static constexpr int RAW_TILE = TILE * D;          // bytes of one FP8 K (or V) tile
  static constexpr int RAW_STAGE = 2 * RAW_TILE;     // K + V
  static constexpr int OP_TILE = TILE * D * 2;       // one f16 K (or V) operand tile
  static constexpr int Q_BYTES = NT * D * 2;
  // K, V (tokens x head_dim) and Q (rows x head_dim) share one physical
  // layout: two 64-element halves of head_dim, each a column of SW128 atoms
  // (8 rows x 128 B), atom g of rows 8g..8g+7 at g*1024. The same bytes are
  // the K-major operand K (S^T = K Q^T) and the MN-major operand V^T.
  static constexpr int KV_HALF = (TILE / 8) * 1024;  // one 64-element half
  static constexpr int Q_HALF = (NT / 8) * 1024;
  // P^T (rows x tokens, rows contiguous): one atom of 8 tokens x NT rows,
  // SW64 (NT = 32, 64-byte rows) or SW32 (NT = 16, 32-byte rows)
  static constexpr int P_ROW = NT * 2;               // bytes per token row
  static constexpr int P_SBO = 8 * P_ROW;            // token-group stride
  static constexpr int P_BYTES = (TILE / 8) * P_SBO;
  static constexpr uint32_t P_SWIZZLE = NT == 32 ? 4u : 6u;  // SW64 / SW32
  // shared memory map
  static constexpr int OFF_RAW = 0;
  static constexpr int OFF_K = OFF_RAW + RAW_STAGES * RAW_STAGE;
  static constexpr int OFF_V = OFF_K + 2 * OP_TILE;
  static constexpr int OFF_Q = OFF_V + 2 * OP_TILE;
  static constexpr int OFF_P = OFF_Q + Q_BYTES;
  static constexpr int OFF_WMAX = OFF_P + 2 * P_BYTES;        // [4][NT] f32
  static constexpr int OFF_M = OFF_WMAX + SOFT_WARPS * NT * 4;  // [2][NT] f32
  static constexpr int OFF_ALPHA = OFF_M + 2 * NT * 4;          // [2][NT] f32
  static constexpr int OFF_LRED = OFF_ALPHA + 2 * NT * 4;       // [4][NT] f32
  static constexpr int OFF_RANGE = OFF_LRED + SOFT_WARPS * NT * 4;  // [NT] int2 (lo, hi)
  static constexpr int OFF_BAR = OFF_RANGE + NT * 8;
  // mbarriers: raw_full[2], kv_ready[2], s_full[2], p_ready[2], o_full[2], o_free[2]
  static constexpr int NUM_BARS = 12;
  static constexpr int OFF_TMEM_SLOT = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_FLAGS = OFF_TMEM_SLOT + 8;
  static constexpr int SMEM = OFF_FLAGS + 8;
  // Launch with 4 KB of slack past the last object, so that no descriptor
  // read can leave the CTA's shared memory even near the end of a buffer.
  static constexpr int SMEM_ALLOC = SMEM + 4096;
  // TMEM columns: S^T[2] then O^T[2], NT fp32 columns each
  static constexpr int TMEM_COLS = 128;
  static constexpr int COL_S = 0, COL_O = 2 * NT;
  static_assert(NT == 16 || NT == 32, "rows per CTA");
  static_assert(4 * NT <= TMEM_COLS, "TMEM columns");
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory");
  static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && OFF_Q % 1024 == 0 &&
                    OFF_P % 1024 == 0 && P_BYTES % 1024 == 0,
                "swizzle atoms need 1024-byte aligned bases");
};

// ---- tcgen05 / UMMA helpers ------------------------------------------------

// Shared-memory matrix descriptor: start address, leading- and stride-
// dimension byte offsets, and the swizzle mode of the canonical layout.
// Swizzled atoms are 8 rows of 128 (SW128), 64 (SW64) or 32 (SW32) bytes
// whose 16-byte chunks are XOR-permuted by row, which keeps the tensor
// core's operand reads free of bank conflicts. Atom bases are aligned to
// 8 rows x row bytes, so the base-offset field stays 0.
constexpr uint32_t kSw128 = 2, kSw64 = 4, kSw32 = 6;
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Instruction descriptor of tcgen05.mma kind::f16: f16 A and B, fp32 D.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N, bool a_mn_major,
                                                      bool b_mn_major) {
  return (1u << 4)                              // D format: f32
         | (0u << 7) | (0u << 10)               // A, B format: f16
         | ((a_mn_major ? 1u : 0u) << 15)
         | ((b_mn_major ? 1u : 0u) << 16)
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(r[k]);
}

// 16 consecutive fp32 TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = __uint_as_float(r[k]);
}

template <int NT>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, float (&v)[NT]) {
  if constexpr (NT == 32) {
    tmem_ld32(taddr, v);
  } else {
    tmem_ld16(taddr, v);
  }
}

__device__ __forceinline__ float redux_max(float x) {
  float y;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void named_bar(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Named barrier over `threads` threads that also returns the AND of `v` over
// them, so every thread takes the same branch afterwards.
__device__ __forceinline__ bool named_bar_and(int id, int threads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

// One named barrier returning the OR of `want` over the threads; `*ok_out`
// gets the AND of `ok`. (Two barrier reductions back to back on the same id.)
__device__ __forceinline__ bool named_bar_or_and(int id, int threads, bool want, bool ok,
                                                 bool* ok_out) {
  uint32_t r_or, r_and;
  asm volatile(
      "{\n\t.reg .pred p, q, x, y;\n\tsetp.ne.u32 p, %2, 0;\n\tsetp.ne.u32 q, %3, 0;\n\t"
      "bar.red.or.pred x, %4, %5, p;\n\tbar.red.and.pred y, %4, %5, q;\n\t"
      "selp.u32 %0, 1, 0, x;\n\tselp.u32 %1, 1, 0, y;\n\t}"
      : "=r"(r_or), "=r"(r_and)
      : "r"((uint32_t)want), "r"((uint32_t)ok), "r"(id), "r"(threads)
      : "memory");
  *ok_out = r_and != 0;
  return r_or != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// 8 e4m3 codes -> 8 f16 packed as a uint4 (exact).
__device__ __forceinline__ uint4 e4m3x8_to_f16x8(uint2 u) {
  uint4 o;
  uint32_t* w = reinterpret_cast<uint32_t*>(&o);
  const uint32_t in[2] = {u.x, u.y};
#pragma unroll
  for (int k = 0; k < 2; ++k) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>((in[k] >> (16 * h)) & 0xFFFFu), __NV_E4M3);
      w[2 * k + h] = (uint32_t)hr.x | ((uint32_t)hr.y << 16);
    }
  }
  return o;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---- the kernel ------------------------------------------------------------

template <int NT>
__global__ void __launch_bounds__(TcCfg<NT>::THREADS, 1) split_tc_kernel(const SplitArgs a) {
  using C = TcCfg<NT>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int rt = blockIdx.x;
  const int split = blockIdx.y % a.num_splits;
  const int kvh = blockIdx.y / a.num_splits;
  const int b = blockIdx.z;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* raw_full = bars + 0;   // [2] copy landed (tx count)
  uint64_t* kv_ready = bars + 2;   // [2] converted K/V tile written (128 arrivals)
  uint64_t* s_full = bars + 4;     // [2] S^T in TMEM (commit)
  uint64_t* p_ready = bars + 6;    // [2] P^T written, S^T read (128 arrivals)
  uint64_t* o_full = bars + 8;     // [2] O^T in TMEM, K/V/P operands free (commit)
  uint64_t* o_free = bars + 10;    // [2] O^T read back (128 arrivals)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);

  // ---- key range of this CTA (tiles of 128 tokens, absolute-aligned) -----
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
  // The swizzle patterns below assume 1024-byte aligned atoms.
  if ((smem_addr(smem) & 1023u) != 0) {
    if (tid == 0) record_error_at(a.err, kErrUnsupported);
    ntiles = 0;
  }

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&kv_ready[i], 128);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], 128);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {  // TMEM allocation is warp-wide
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem = *tmem_slot;

  const long long head_off = (long long)kvh * a.head_stride;
  const int32_t* pt_row = a.page_table + (long long)b * a.max_pages;
  // tile k covers tokens [k*128, k*128+128): pages (k*128)>>log2P ... ; a
  // page of P tokens is P*128 contiguous bytes of the (page, head) block
  const int seq_pages = (L + a.page_size - 1) >> a.log2_page;
  // Tile k covers tokens [k*128, k*128+128). A page holds P tokens of one kv
  // head as P*128 contiguous bytes of its (page, head) block. Pages past the
  // sequence's last page are not copied (their slots are keys >= kv_len,
  // masked for K and zeroed for V); the transaction count matches the bytes
  // actually copied.
  auto issue_tile = [&](int n) {  // thread 0 only
    const int st = n % C::RAW_STAGES;
    uint8_t* dst = smem + C::OFF_RAW + st * C::RAW_STAGE;
    const int tok0 = (kfirst + n) * C::TILE;
    if (a.page_size >= C::TILE) {
      int pid = __ldg(pt_row + (tok0 >> a.log2_page));
      if ((unsigned)pid >= (unsigned)a.num_pages) {
        record_error_at(a.err, kErrBadPage);
        pid = 0;
      }
      const long long off = (long long)pid * a.page_stride + head_off +
                            (long long)(tok0 & (a.page_size - 1)) * C::D;
      mbar_arrive_expect_tx(&raw_full[st], C::RAW_STAGE);
      bulk_g2s(dst, a.k_pages + off, C::RAW_TILE, &raw_full[st]);
      bulk_g2s(dst + C::RAW_TILE, a.v_pages + off, C::RAW_TILE, &raw_full[st]);
    } else {
      const int first = tok0 >> a.log2_page;
      const int npg = min(C::TILE >> a.log2_page, seq_pages - first);  // >= 1
      const uint32_t bytes = (uint32_t)a.page_size * C::D;
      mbar_arrive_expect_tx(&raw_full[st], 2u * bytes * (uint32_t)npg);
      for (int g = 0; g < npg; ++g) {
        int pid = __ldg(pt_row + first + g);
        if ((unsigned)pid >= (unsigned)a.num_pages) {
          record_error_at(a.err, kErrBadPage);
          pid = 0;
        }
        const long long off = (long long)pid * a.page_stride + head_off;
        bulk_g2s(dst + g * bytes, a.k_pages + off, bytes, &raw_full[st]);
        bulk_g2s(dst + C::RAW_TILE + g * bytes, a.v_pages + off, bytes, &raw_full[st]);
      }
    }
  };

  // scale of S (raw f16 Q . f16 K) into the log2 domain
  const float cs = a.qk_scale_log2;

  if (warp < C::CONV_WARPS) {
    // ======================= converters (thread = token) ===================
    const int t = tid;  // 0..127
    // Q (rows R0 .. R0+NT-1) -> f16, K-major canonical layout; row >= M -> 0
    for (int c = t; c < NT * 16; c += 128) {
      const int n = c % NT, j = c / NT;  // row, 8-element chunk of head_dim
      const int R = R0 + n;
      uint4 o = make_uint4(0, 0, 0, 0);
      if (R < a.M) {
        const int i = R / a.G, h = kvh * a.G + R % a.G;
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(
            a.q + ((long long)(b * a.Lq + i) * a.Hq + h) * C::D + j * 8));
        float f[8];
        bf16x8_to_f32(u, f);
        o.x = pack_f16x2(f[0], f[1]);
        o.y = pack_f16x2(f[2], f[3]);
        o.z = pack_f16x2(f[4], f[5]);
        o.w = pack_f16x2(f[6], f[7]);
      }
      *reinterpret_cast<uint4*>(smem + C::OFF_Q + (j >> 3) * C::Q_HALF + (n >> 3) * 1024 +
                                (n & 7) * 128 + (((j & 7) ^ (n & 7)) << 4)) = o;
    }
    int issued = 0;  // tiles whose copies thread 0 has issued
    if (t == 0) {
      for (; issued < C::RAW_STAGES && issued < ntiles; ++issued) issue_tile(issued);
    }
    const int rot = t & 7;
    for (int n = 0; n < ntiles; ++n) {
      const int st = n % C::RAW_STAGES;
      const int bb = n & 1;
      bool ok = !*abort_flag;
      if (ok) ok = mbar_wait(&raw_full[st], (n / C::RAW_STAGES) & 1, a.err);
      if (ok && n >= 2) ok = mbar_wait(&o_full[bb], ((n - 2) >> 1) & 1, a.err);
      const uint8_t* raw = smem + C::OFF_RAW + st * C::RAW_STAGE;
      uint2 kr[16], vr[16];
      if (ok) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {  // rotated 16-byte chunks: no bank conflicts
          const int ch = (c + rot) & 7;
          const uint4 k4 = *reinterpret_cast<const uint4*>(raw + t * C::D + ch * 16);
          const uint4 v4 =
              *reinterpret_cast<const uint4*>(raw + C::RAW_TILE + t * C::D + ch * 16);
          kr[2 * c] = make_uint2(k4.x, k4.y);
          kr[2 * c + 1] = make_uint2(k4.z, k4.w);
          vr[2 * c] = make_uint2(v4.x, v4.y);
          vr[2 * c + 1] = make_uint2(v4.z, v4.w);
        }
      }
      // every converter has read the raw stage (or the group stops together)
      if (!named_bar_and(1, 128, ok)) {
        *abort_flag = 1;
        break;
      }
      if (t == 0 && issued < ntiles) {
        fence_proxy_async_smem();
        issue_tile(issued);
        ++issued;
      }
      const int j_tok = (kfirst + n) * C::TILE + t;
      const bool v_zero = j_tok < lo_u || j_tok >= hi_u;
      const int row_off = (t >> 3) * 1024 + (t & 7) * 128;
      uint8_t* sk = smem + C::OFF_K + bb * C::OP_TILE + row_off;
      uint8_t* sv = smem + C::OFF_V + bb * C::OP_TILE + row_off;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int j = ((c >> 1) + rot) & 7;  // 16-byte raw chunk (c>>1) rotated
        const int chunk8 = 2 * j + (c & 1);  // which 8 head-dim elements
        const int off = (chunk8 >> 3) * C::KV_HALF + (((chunk8 & 7) ^ (t & 7)) << 4);
        *reinterpret_cast<uint4*>(sk + off) = e4m3x8_to_f16x8(kr[c]);
        const uint4 vv = v_zero ? make_uint4(0, 0, 0, 0) : e4m3x8_to_f16x8(vr[c]);
        *reinterpret_cast<uint4*>(sv + off) = vv;
      }
      fence_proxy_async_smem();
      mbar_arrive(&kv_ready[bb]);
    }
    if (t == 0 && *abort_flag) {
      // copies already issued land before the CTA releases its shared memory
      for (int n = max(0, issued - C::RAW_STAGES); n < issued; ++n)
        mbar_wait(&raw_full[n % C::RAW_STAGES], (n / C::RAW_STAGES) & 1, a.err,
                  kWaitTimeoutCycles / 16);
    }
  } else if (warp == C::MMA_WARP) {
    // ======================= MMA issuer (one lane) ==========================
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_f16(128, NT, false, false);  // K, Q both K-major
      constexpr uint32_t idesc_o = umma_idesc_f16(128, NT, true, true);    // V^T, P^T MN-major
      const uint32_t sbase = smem_addr(smem);
      auto issue_s = [&](int n) {  // S^T = K Q^T, K = head_dim in steps of 16
        const int bb = n & 1;
        const uint32_t ka = sbase + C::OFF_K + bb * C::OP_TILE;
        const uint32_t qa = sbase + C::OFF_Q;
#pragma unroll
        for (int s = 0; s < C::D / 16; ++s)
          umma_f16(tmem + C::COL_S + bb * NT,
                   umma_desc(ka + (s >> 2) * C::KV_HALF + (s & 3) * 32, 16, 1024, kSw128),
                   umma_desc(qa + (s >> 2) * C::Q_HALF + (s & 3) * 32, 16, 1024, kSw128),
                   idesc_s, s > 0);
        umma_commit(&s_full[bb]);
      };
      auto issue_o = [&](int n) {  // O^T = V^T P^T, K = tokens in steps of 16
        const int bb = n & 1;
        const uint32_t va = sbase + C::OFF_V + bb * C::OP_TILE;
        const uint32_t pa = sbase + C::OFF_P + bb * C::P_BYTES;
#pragma unroll
        for (int s = 0; s < C::TILE / 16; ++s)
          umma_f16(tmem + C::COL_O + bb * NT, umma_desc(va + s * 2048, C::KV_HALF, 1024, kSw128),
                   umma_desc(pa + s * 2 * C::P_SBO, C::P_BYTES, C::P_SBO, C::P_SWIZZLE), idesc_o,
                   s > 0);
        umma_commit(&o_full[bb]);
      };
      // Event-driven issue: S^T of tile k once its K tile is converted and
      // softmax(k-2) has read S^T buffer k&1; O^T of tile k once softmax(k)
      // has written P^T and O^T buffer k&1 has been read back (tile k-2).
      int s_issued = 0, o_issued = 0;
      bool ok = true;
      const long long start = clock64();
      long long last = start;
      while (o_issued < ntiles) {
        bool progress = false;
        if (s_issued < ntiles && s_issued < o_issued + 2) {
          const int k = s_issued;
          if (mbar_test(&kv_ready[k & 1], (k >> 1) & 1) &&
              (k < 2 || mbar_test(&p_ready[k & 1], ((k - 2) >> 1) & 1))) {
            tmem_fence_after();
            issue_s(k);
            ++s_issued;
            progress = true;
          }
        }
        if (o_issued < s_issued) {
          const int k = o_issued;
          if (mbar_test(&p_ready[k & 1], (k >> 1) & 1) &&
              (k < 2 || mbar_test(&o_free[k & 1], ((k - 2) >> 1) & 1))) {
            tmem_fence_after();
            issue_o(k);
            ++o_issued;
            progress = true;
          }
        }
        const long long now = clock64();
        if (progress) {
          last = now;
        } else if (now - last > kWaitTimeoutCycles || *abort_flag) {
          if (!*abort_flag) record_error_at(a.err, kErrTimeout);
          ok = false;
          break;
        }
      }
      if (!ok) *abort_flag = 1;
      if (*abort_flag) {
        // MMAs already issued finish before TMEM is released
        if (s_issued > 0)
          mbar_wait(&s_full[(s_issued - 1) & 1], ((s_issued - 1) >> 1) & 1, a.err,
                    kWaitTimeoutCycles / 16);
        if (o_issued > 0)
          mbar_wait(&o_full[(o_issued - 1) & 1], ((o_issued - 1) >> 1) & 1, a.err,
                    kWaitTimeoutCycles / 16);
      }
    }
    __syncwarp();
  } else {
    // ======================= softmax / accumulate (thread = TMEM lane) =====
    const int i = tid - C::CONV_WARPS * 32;  // 0..127: token of S^T, element of O^T
    const int q4 = warp & 3;                 // TMEM lane quarter of this warp
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    float* wmax = reinterpret_cast<float*>(smem + C::OFF_WMAX);
    float* sm_m = reinterpret_cast<float*>(smem + C::OFF_M);
    float* sm_alpha = reinterpret_cast<float*>(smem + C::OFF_ALPHA);
    // visible key range [lo, hi) of each row of this row tile (rows past M
    // see nothing), read on boundary tiles only
    int2* rng = reinterpret_cast<int2*>(smem + C::OFF_RANGE);
    if (i < NT) {
      const int R = R0 + i;
      int lo = 0, hi = 0;
      if (R < a.M) row_range(a, L, R / a.G, lo, hi);
      rng[i] = make_int2(lo, hi);
    }
    named_bar(2, 128);
    float m_run = -INFINITY;  // row i (i < NT) keeps the running max of row i
    float l_part[NT], acc[NT];
#pragma unroll
    for (int r = 0; r < NT; ++r) {
      l_part[r] = 0.f;
      acc[r] = 0.f;
    }
    bool ok = true;

    auto accumulate = [&](int k) -> bool {  // fold O^T of tile k into acc
      const int bb = k & 1;
      const bool ok_w = __all_sync(0xFFFFFFFFu, mbar_wait(&o_full[bb], (k >> 1) & 1, a.err));
      if (!ok_w) return false;
      tmem_fence_after();
      float o[NT];
      tmem_ld_row<NT>(tmem + lane_off + C::COL_O + bb * NT, o);
      tmem_fence_before();
      mbar_arrive(&o_free[bb]);
      const float4* al = reinterpret_cast<const float4*>(sm_alpha + bb * NT);
#pragma unroll
      for (int r4 = 0; r4 < NT / 4; ++r4) {
        const float4 x = al[r4];
        acc[4 * r4 + 0] = fmaf(acc[4 * r4 + 0], x.x, o[4 * r4 + 0]);
        acc[4 * r4 + 1] = fmaf(acc[4 * r4 + 1], x.y, o[4 * r4 + 1]);
        acc[4 * r4 + 2] = fmaf(acc[4 * r4 + 2], x.z, o[4 * r4 + 2]);
        acc[4 * r4 + 3] = fmaf(acc[4 * r4 + 3], x.w, o[4 * r4 + 3]);
      }
      return true;
    };

    bool acc_ok = true;  // did the previous accumulate succeed (this thread)
    for (int n = 0; n < ntiles; ++n) {
      const int bb = n & 1;
      bool ok_s = acc_ok && !*abort_flag;
      if (ok_s) ok_s = mbar_wait(&s_full[bb], (n >> 1) & 1, a.err);
      ok_s = __all_sync(0xFFFFFFFFu, ok_s);  // tcgen05.ld is warp-wide
      float s[NT];
      if (ok_s) {
        tmem_fence_after();
        tmem_ld_row<NT>(tmem + lane_off + C::COL_S + bb * NT, s);
      } else {
#pragma unroll
        for (int r = 0; r < NT; ++r) s[r] = -INFINITY;
      }
      const int t0 = (kfirst + n) * C::TILE;
      const int j = t0 + i;
      if (!(t0 >= lo_x && t0 + C::TILE <= hi_x)) {
#pragma unroll
        for (int r = 0; r < NT; ++r) {
          const int2 lh = rng[r];
          if (!(j >= lh.x && j < lh.y)) s[r] = -INFINITY;
        }
      }
      // row maxima: warp max per row, then over the four warps
#pragma unroll
      for (int r = 0; r < NT; ++r) {
        const float wm = redux_max(s[r]);
        if (lane == r) wmax[q4 * NT + r] = wm;
      }
      if (!named_bar_and(2, 128, ok_s)) {
        ok = false;
        break;
      }
      if (i < NT) {
        float mt = fmaxf(fmaxf(wmax[i], wmax[NT + i]), fmaxf(wmax[2 * NT + i], wmax[3 * NT + i]));
        mt = mt == -INFINITY ? -INFINITY : mt * cs;
        const float m_new = fmaxf(m_run, mt);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        sm_alpha[bb * NT + i] = fast_exp2(m_run - m_use);
        sm_m[bb * NT + i] = m_use;
        m_run = m_new;
      }
      named_bar(2, 128);
      // p = exp2(s * cs - m) as f16 P^T; running row sums of this token
      const float4* mm = reinterpret_cast<const float4*>(sm_m + bb * NT);
      const float4* al = reinterpret_cast<const float4*>(sm_alpha + bb * NT);
      float* p = s;  // probabilities overwrite the scores
#pragma unroll
      for (int r4 = 0; r4 < NT / 4; ++r4) {
        const float4 m4 = mm[r4];
        const float4 a4 = al[r4];
        const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = 4 * r4 + e;
          p[r] = fast_exp2(fmaf(s[r], cs, -mv[e]));
          l_part[r] = fmaf(l_part[r], av[e], p[r]);
        }
      }
      // token i's row of P^T: NT f16 = NT/8 chunks of 16 B, XOR-swizzled by
      // the row's position in its 8-token atom (SW64: bits 7-8 of the
      // address, i.e. row >> 1; SW32: bit 7, i.e. row >> 2)
      uint8_t* sp = smem + C::OFF_P + bb * C::P_BYTES + (i >> 3) * C::P_SBO + (i & 7) * C::P_ROW;
      const int pswz = NT == 32 ? ((i & 7) >> 1) & 3 : ((i & 7) >> 2) & 1;
#pragma unroll
      for (int g = 0; g < NT / 8; ++g) {
        uint4 w;
        w.x = pack_f16x2(p[8 * g + 0], p[8 * g + 1]);
        w.y = pack_f16x2(p[8 * g + 2], p[8 * g + 3]);
        w.z = pack_f16x2(p[8 * g + 4], p[8 * g + 5]);
        w.w = pack_f16x2(p[8 * g + 6], p[8 * g + 7]);
        *reinterpret_cast<uint4*>(sp + ((g ^ pswz) << 4)) = w;
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

    // ---- epilogue: row sums over the 128 tokens, normalise, write --------
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
      for (int r = 0; r < NT; ++r) lred[q4 * NT + r] = l_part[r];
    }
    named_bar(2, 128);
    const bool failed = !ok;
    const long long rows_total = (long long)a.B * a.Lq * a.Hq;
#pragma unroll
    for (int r = 0; r < NT; ++r) {
      const int R = R0 + r;
      if (R >= a.M) continue;
      const float lt = lred[r] + lred[NT + r] + lred[2 * NT + r] + lred[3 * NT + r];
      const float o = lt > 0.f && !failed ? acc[r] * (a.v_scale / lt) : 0.f;
      const int qi = R / a.G, h = kvh * a.G + R % a.G;
      const long long row = (long long)(b * a.Lq + qi) * a.Hq + h;
      if (a.num_splits == 1) {
        a.out[row * C::D + i] = o;
      } else {
        a.o_part[((long long)split * rows_total + row) * C::D + i] = o;
      }
    }
    if (i < NT && R0 + i < a.M) {
      const int R = R0 + i;
      const float lt = lred[i] + lred[NT + i] + lred[2 * NT + i] + lred[3 * NT + i];
      const float res =
          lt > 0.f && !failed ? (m_run + log2f(lt)) * 0.69314718055994531f : -INFINITY;
      const int qi = R / a.G, h = kvh * a.G + R % a.G;
      const long long row = (long long)(b * a.Lq + qi) * a.Hq + h;
      if (a.num_splits == 1) {
        if (a.lse) a.lse[row] = res;
      } else {
        a.lse_part[(long long)split * rows_total + row] = res;
      }
    }
  }

  pdl_launch_dependents();
  tmem_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tmem_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::TMEM_COLS)
                 : "memory");
  }
}

cudaError_t launch_split_tc(int nt, const SplitArgs& a, dim3 grid, cudaStream_t stream);

}  // namespace pda
