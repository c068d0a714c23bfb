/*
 * Plain fp64 reference for paged-KV decode attention.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the oracle that the CUDA library is
 * checked against. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load it; the product path never does. It shares no
 * code, header, table or constant with the CUDA library.
 *
 * What it computes (single-threaded, double precision, no blocking, no
 * online rescaling, no split): for every sequence b, query row i and query
 * head h, plain softmax attention over the keys the row may see, walking the
 * page table one token at a time.
 *
 * Sources, by page and section:
 *  - "AstrAI commit log, attn_paged_decode_split_kv_mma.cuh": the scalar
 *    variant resolves the page table per position when it loads K/V; the
 *    split-KV partials are later combined; causal_offset semantics
 *    (-1 = off, >= 0 = position of the first query row).
 *  - "b12x 0.30.0, Kernel inventory, Attention table, Paged attention row":
 *    bf16 and FP8-E4M3 KV caches, sliding window, GQA, split-KV or direct
 *    output, persistent merge kernel.
 *  - "sglang profiler skill, fuse-overlap catalog, vLLM-origin attention +
 *    output quant row": merge_attn_states combines attention states by their
 *    log-sum-exp.
 *
 * Readings taken where the pages are silent:
 *  R1 lse is the natural log of sum_j exp(scale * q.k_j).
 *  R2 causal_offset = -2 means bottom-right alignment: pos_i = L_b - q_len + i.
 *  R3 a window of W keys includes the query's own position:
 *     visible iff j >= pos_i - W + 1; W <= 0 is off; with causal off the
 *     window is measured from L_b - 1.
 *  R4 GQA head mapping is consecutive: kv head = h / (Hq / Hkv).
 *  R5 KV pool layout is [num_pages, Hkv, page_size, D].
 *  R6 FP8 value = decode_e4m3(byte) * kv_scale, one scale for K and V.
 *  R8 a row that sees no key has out = 0 and lse = -inf.
 *  R22 NVFP4 KV ("b12x 0.30.0, Kernel inventory": NVFP4 float4_e2m1fn with
 *      E4M3 scales per 16 elements, "BF16-to-FP4 TMA quantization" row:
 *      packed NVFP4 plus scale tiles): element d of a token row is the
 *      E2M1 nibble d % 2 (low nibble first) of byte d / 2 of the code pool
 *      [num_pages, Hkv, P, D/2]; each block of 16 consecutive elements of
 *      the row has one E4M3 scale in the scale pool [num_pages, Hkv, P,
 *      D/16]; value = e2m1(code) * e4m3(block scale) * kv_scale.
 *  R23 NVFP4 quantisation of new K/V rows (the cache producer's rule): per
 *      block of 16 elements, in single precision with nearest-even rounding
 *      and saturation, q = x / kv_scale, scale = e4m3(max |q| / 6), code =
 *      e2m1(q / scale); a block whose scale is zero stores +0 codes.
 *  R18 the attention-sink bias of query head h is a logit sink[h] (natural
 *      log units, same scale as scale * q.k) that adds exp(sink[h]) to the
 *      softmax denominator and contributes no value: out = sum_j
 *      exp(s_j - lse) v_j with lse = ln(sum_j exp(s_j) + exp(sink[h])); a row
 *      that sees no key has out = 0 and lse = sink[h].
 *
 * Pins (tests/test_oracle.py): brute-force dense attention over the unpaged
 * K/V, page-permutation invariance, split-merge invariance, closed forms
 * (equal keys -> mean of V, one key -> v, one-hot V -> probabilities),
 * e4m3/bf16 decode against torch's independent float8/bfloat16 casts,
 * e2m1 decode and encode against ml_dtypes' float4_e2m1fn (another
 * independent implementation) and hand-worked codes, and hand-derived
 * golden fixtures.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -fPIC -shared oracle.c -o liboracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Status codes returned by the oracle. */
#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_BAD_PAGE 2
#define ORACLE_NO_MEMORY 3

#define ORACLE_KV_BF16 0
#define ORACLE_KV_FP8_E4M3 1
#define ORACLE_KV_NVFP4 2

#define ORACLE_CAUSAL_OFF (-1)
#define ORACLE_CAUSAL_BOTTOM_RIGHT (-2)

/* bf16 is the upper half of an IEEE binary32: widen by a 16-bit shift. */
double oracle_bf16_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* FP8 E4M3 ("fn" variant, no infinities) from its fields:
 * sign bit, 4 exponent bits with bias 7, 3 mantissa bits.
 * exponent 0 is subnormal: m/8 * 2^(1-7); S.1111.111 is NaN;
 * every other code is (1 + m/8) * 2^(e-7). Largest finite value 448. */
double oracle_e4m3_to_double(uint8_t code) {
  int s = (code >> 7) & 1;
  int e = (code >> 3) & 0xF;
  int m = code & 0x7;
  double mag;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0)
    mag = ldexp((double)m / 8.0, 1 - 7);
  else
    mag = ldexp(1.0 + (double)m / 8.0, e - 7);
  return s ? -mag : mag;
}

/* FP4 E2M1 from its fields: sign bit, 2 exponent bits with bias 1, 1
 * mantissa bit. exponent 0 is subnormal: m/2 * 2^(1-1); every other code is
 * (1 + m/2) * 2^(e-1). No infinities or NaN; largest magnitude 6. */
double oracle_e2m1_to_double(uint8_t code) {
  int s = (code >> 3) & 1;
  int e = (code >> 1) & 0x3;
  int m = code & 0x1;
  double mag;
  if (e == 0)
    mag = (double)m / 2.0;
  else
    mag = ldexp(1.0 + (double)m / 2.0, e - 1);
  return s ? -mag : mag;
}

/* One K or V element of the pool, decoded to double. `index` counts
 * elements of [num_pages, Hkv, P, D]; for NVFP4 (reading R22) the codes sit
 * two per byte and `scales` holds one E4M3 code per 16 elements. */
static double kv_elem(const void* pool, const void* scales, int kv_dtype,
                      double kv_scale, int64_t index) {
  if (kv_dtype == ORACLE_KV_BF16)
    return oracle_bf16_to_double(((const uint16_t*)pool)[index]);
  if (kv_dtype == ORACLE_KV_FP8_E4M3)
    return oracle_e4m3_to_double(((const uint8_t*)pool)[index]) * kv_scale;
  const uint8_t byte = ((const uint8_t*)pool)[index / 2];
  const uint8_t code = (index % 2) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
  const double block = oracle_e4m3_to_double(((const uint8_t*)scales)[index / 16]);
  return oracle_e2m1_to_double(code) * block * kv_scale;
}

/* Position of query row i of sequence b (reading R2/R3). */
static int64_t row_position(int causal_offset, int64_t kv_len, int q_len,
                            int i) {
  if (causal_offset >= 0) return (int64_t)causal_offset + i;
  if (causal_offset == ORACLE_CAUSAL_BOTTOM_RIGHT)
    return kv_len - (int64_t)q_len + i;
  return kv_len - 1; /* causal off: only the window uses it */
}

/* Is logical key j visible to a query row at position pos? */
static int key_visible(int64_t j, int64_t kv_len, int causal, int64_t pos,
                       int window) {
  if (j < 0 || j >= kv_len) return 0;
  if (causal && j > pos) return 0;
  if (window > 0 && j < pos - (int64_t)window + 1) return 0;
  return 1;
}

/* Shared argument checks of the two entry points below. */
static int check_args(const int32_t* kv_lens, int B, int q_len, int Hq, int Hkv,
                      int D, int page_size, int max_pages, int num_pages,
                      int causal_offset, int kv_dtype, int64_t* max_len) {
  if (B < 0 || q_len < 1 || Hq < 1 || Hkv < 1 || D < 1 || page_size < 1 ||
      max_pages < 0 || num_pages < 0 || Hq % Hkv != 0)
    return ORACLE_BAD_ARG;
  if (kv_dtype != ORACLE_KV_BF16 && kv_dtype != ORACLE_KV_FP8_E4M3 &&
      kv_dtype != ORACLE_KV_NVFP4)
    return ORACLE_BAD_ARG;
  if (kv_dtype == ORACLE_KV_NVFP4 && D % 16 != 0) return ORACLE_BAD_ARG;
  if (causal_offset < ORACLE_CAUSAL_BOTTOM_RIGHT) return ORACLE_BAD_ARG;
  *max_len = 0;
  for (int b = 0; b < B; ++b) {
    if (kv_lens[b] < 0) return ORACLE_BAD_ARG;
    if (kv_lens[b] > (int64_t)max_pages * page_size) return ORACLE_BAD_ARG;
    if (kv_lens[b] > *max_len) *max_len = kv_lens[b];
  }
  return ORACLE_OK;
}

/*
 * One output row: out[b, i, h, :] and lse[b, i, h], restricted to keys in
 * [tok_lo, tok_hi) (tok_hi < 0 means no restriction). `s` is scratch for
 * kv_lens[b] scores. `sink` (natural-log units, -inf for none) is the row's
 * attention-sink logit: one more exp(sink) term in the softmax denominator
 * with no value vector (reading R18).
 */
static int oracle_row(const uint16_t* q, const void* k_pages, const void* v_pages,
                      const void* k_scales, const void* v_scales,
                      const int32_t* page_table, const int32_t* kv_lens, int q_len,
                      int Hq, int Hkv, int D, int page_size, int max_pages,
                      int num_pages, float scale, int causal_offset, int window,
                      int kv_dtype, float kv_scale, int64_t tok_lo, int64_t tok_hi,
                      double sink, int b, int i, int h, double* s, double* out,
                      double* lse) {
  const int G = Hq / Hkv;
  const int causal = causal_offset != ORACLE_CAUSAL_OFF;
  const double dscale = (double)scale;
  const double dkv_scale = (double)kv_scale;
  const int64_t L = kv_lens[b];
  const int64_t pos = row_position(causal_offset, L, q_len, i);
  const int g = h / G; /* reading R4 */
  const uint16_t* qrow = q + (((int64_t)b * q_len + i) * Hq + h) * D;
  double* orow = out + (((int64_t)b * q_len + i) * Hq + h) * D;
  double* lrow = lse + ((int64_t)b * q_len + i) * Hq + h;

  /* Pass 1: scores of the visible keys, walking the page table. */
  double m = -INFINITY;
  int64_t nvis = 0;
  for (int64_t j = 0; j < L; ++j) {
    int vis = key_visible(j, L, causal, pos, window);
    if (vis && tok_hi >= 0 && (j < tok_lo || j >= tok_hi)) vis = 0;
    if (!vis) {
      s[j] = -INFINITY;
      continue;
    }
    const int32_t page = page_table[(int64_t)b * max_pages + j / page_size];
    if (page < 0 || page >= num_pages) return ORACLE_BAD_PAGE;
    const int64_t row = j % page_size;
    const int64_t base = (((int64_t)page * Hkv + g) * page_size + row) * D;
    double dot = 0.0;
    for (int d = 0; d < D; ++d)
      dot += oracle_bf16_to_double(qrow[d]) *
             kv_elem(k_pages, k_scales, kv_dtype, dkv_scale, base + d);
    s[j] = dscale * dot;
    if (s[j] > m) m = s[j];
    ++nvis;
  }

  if (nvis == 0) { /* reading R8; with a sink the denominator is exp(sink) alone */
    for (int d = 0; d < D; ++d) orow[d] = 0.0;
    *lrow = sink;
    return ORACLE_OK;
  }

  /* lse = m + ln (sum_j exp(s_j - m) + exp(sink - m))  (readings R1, R18) */
  if (sink > m) m = sink;
  double sum = 0.0;
  for (int64_t j = 0; j < L; ++j)
    if (s[j] != -INFINITY) sum += exp(s[j] - m);
  if (sink != -INFINITY) sum += exp(sink - m);
  const double row_lse = m + log(sum);
  *lrow = row_lse;

  /* Pass 2: out = sum_j exp(s_j - lse) * v_j. */
  for (int d = 0; d < D; ++d) orow[d] = 0.0;
  for (int64_t j = 0; j < L; ++j) {
    if (s[j] == -INFINITY) continue;
    const double p = exp(s[j] - row_lse);
    const int32_t page = page_table[(int64_t)b * max_pages + j / page_size];
    const int64_t row = j % page_size;
    const int64_t base = (((int64_t)page * Hkv + g) * page_size + row) * D;
    for (int d = 0; d < D; ++d)
      orow[d] += p * kv_elem(v_pages, v_scales, kv_dtype, dkv_scale, base + d);
  }
  return ORACLE_OK;
}

/*
 * out[b, i, h, :] and lse[b, i, h] for every row, restricted to keys in
 * [tok_lo, tok_hi) (tok_hi < 0 means no restriction). The restriction lets
 * the tests build split partials from the same definition.
 *
 * q          bf16 bits  [B, q_len, Hq, D]
 * k/v_pages  bf16 bits or e4m3 bytes  [num_pages, Hkv, page_size, D], or
 *            NVFP4 code bytes [num_pages, Hkv, page_size, D/2]
 * k/v_scales NVFP4 only: e4m3 block scales [num_pages, Hkv, page_size, D/16]
 *            (NULL otherwise)
 * page_table int32 [B, max_pages]; kv_lens int32 [B]
 * sinks      float [Hq] attention-sink logits, or NULL for none
 * out        double [B, q_len, Hq, D]; lse double [B, q_len, Hq]
 */
int oracle_paged_decode_attn(const uint16_t* q, const void* k_pages,
                             const void* v_pages, const void* k_scales,
                             const void* v_scales, const int32_t* page_table,
                             const int32_t* kv_lens, int B, int q_len, int Hq,
                             int Hkv, int D, int page_size, int max_pages,
                             int num_pages, float scale, int causal_offset,
                             int window, int kv_dtype, float kv_scale,
                             const float* sinks, int64_t tok_lo, int64_t tok_hi,
                             double* out, double* lse) {
  int64_t max_len;
  int st = check_args(kv_lens, B, q_len, Hq, Hkv, D, page_size, max_pages, num_pages,
                      causal_offset, kv_dtype, &max_len);
  if (st != ORACLE_OK) return st;
  double* s = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
  if (!s) return ORACLE_NO_MEMORY;
  for (int b = 0; b < B; ++b)
    for (int i = 0; i < q_len; ++i)
      for (int h = 0; h < Hq; ++h) {
        st = oracle_row(q, k_pages, v_pages, k_scales, v_scales, page_table, kv_lens,
                        q_len, Hq, Hkv, D,
                        page_size, max_pages, num_pages, scale, causal_offset, window,
                        kv_dtype, kv_scale, tok_lo, tok_hi,
                        sinks ? (double)sinks[h] : -INFINITY, b, i, h, s, out, lse);
        if (st != ORACLE_OK) {
          free(s);
          return st;
        }
      }
  free(s);
  return ORACLE_OK;
}

/*
 * The same rows computed by `threads` OpenMP threads (one row per task; a
 * row's arithmetic is exactly that of the single-threaded entry point, so
 * the results are bit-identical). Used to time the oracle on all host cores.
 * Without OpenMP support at build time it runs single-threaded.
 */
int oracle_paged_decode_attn_mt(const uint16_t* q, const void* k_pages,
                                const void* v_pages, const void* k_scales,
                                const void* v_scales, const int32_t* page_table,
                                const int32_t* kv_lens, int B, int q_len, int Hq,
                                int Hkv, int D, int page_size, int max_pages,
                                int num_pages, float scale, int causal_offset,
                                int window, int kv_dtype, float kv_scale,
                                const float* sinks, double* out, double* lse,
                                int threads) {
  int64_t max_len;
  int st = check_args(kv_lens, B, q_len, Hq, Hkv, D, page_size, max_pages, num_pages,
                      causal_offset, kv_dtype, &max_len);
  if (st != ORACLE_OK) return st;
  const int64_t rows = (int64_t)B * q_len * Hq;
  int status = ORACLE_OK;
  if (threads < 1) threads = 1;
#pragma omp parallel num_threads(threads)
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
    int local = s ? ORACLE_OK : ORACLE_NO_MEMORY;
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
      if (local != ORACLE_OK) continue;
      const int h = (int)(r % Hq);
      const int i = (int)((r / Hq) % q_len);
      const int b = (int)(r / ((int64_t)Hq * q_len));
      local = oracle_row(q, k_pages, v_pages, k_scales, v_scales, page_table, kv_lens,
                         q_len, Hq, Hkv, D,
                         page_size, max_pages, num_pages, scale, causal_offset, window,
                         kv_dtype, kv_scale, 0, -1, sinks ? (double)sinks[h] : -INFINITY,
                         b, i, h, s, out, lse);
    }
#pragma omp critical
    if (local != ORACLE_OK) status = local;
    free(s);
  }
  return status;
}

/* Number of threads an OpenMP parallel region would use (1 without OpenMP). */
int oracle_max_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * E4M3 encoding of a float, from the format's definition: the finite code
 * whose value is nearest to x, ties to the code with an even mantissa (even
 * code), magnitudes of 448 and above (and infinities) saturating to +-448,
 * NaN to 0x7F. Walks all 127 non-negative codes; no table, no bit tricks.
 */
uint8_t oracle_e4m3_encode(float x) {
  if (isnan(x)) return 0x7F;
  const int neg = signbit(x) ? 1 : 0;
  const double a = fabs((double)x);
  int best = 0;
  if (a >= 448.0) {
    best = 0x7E;
  } else {
    double best_err = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
      const double err = fabs(a - oracle_e4m3_to_double((uint8_t)c));
      if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
        best_err = err;
        best = c;
      }
    }
  }
  return (uint8_t)(best | (neg << 7));
}

/*
 * E2M1 encoding of a float, from the format's definition: the code whose
 * value is nearest to x, ties to the code with an even mantissa bit,
 * magnitudes of 6 and above (and infinities) saturating to +-6; the sign
 * bit follows x (so -0.0 and small negatives that round to zero give the
 * negative zero code 0x8). NaN gives 0x7 (+6; the format has no NaN, and
 * the library leaves NaN inputs unspecified). Walks all 8 non-negative codes.
 */
uint8_t oracle_e2m1_encode(float x) {
  if (isnan(x)) return 0x7;
  const int neg = signbit(x) ? 1 : 0;
  const double a = fabs((double)x);
  int best = 0;
  if (a >= 6.0) {
    best = 0x7;
  } else {
    double best_err = INFINITY;
    for (int c = 0; c <= 0x7; ++c) {
      const double err = fabs(a - oracle_e2m1_to_double((uint8_t)c));
      if (err < best_err || (err == best_err && (best & 1) == 1 && (c & 1) == 0)) {
        best_err = err;
        best = c;
      }
    }
  }
  return (uint8_t)(best | (neg << 3));
}

/*
 * NVFP4 encoding of one block of 16 bf16 values (reading R23, the KV-cache
 * producer's quantiser), every step in single precision:
 *   q_d   = x_d / kv_scale                      (IEEE division)
 *   amax  = max_d |q_d|
 *   scale = e4m3(amax / 6)                      (nearest even, saturating)
 *   code_d = e2m1(q_d / decode(scale))          (nearest even, saturating)
 * A block whose scale decodes to zero stores every code as +0.
 * codes[d] receives the 4-bit code of element d (one per byte here).
 */
void oracle_nvfp4_encode_block(const uint16_t* x, float kv_scale, uint8_t* codes,
                               uint8_t* scale_code) {
  float q[16];
  float amax = 0.f;
  for (int d = 0; d < 16; ++d) {
    q[d] = (float)oracle_bf16_to_double(x[d]) / kv_scale;
    const float a = fabsf(q[d]);
    if (a > amax) amax = a;
  }
  *scale_code = oracle_e4m3_encode(amax / 6.0f);
  const float sd = (float)oracle_e4m3_to_double(*scale_code);
  for (int d = 0; d < 16; ++d) codes[d] = sd > 0.f ? oracle_e2m1_encode(q[d] / sd) : 0;
}

/*
 * Q as "native FP8 QK" uses it: each row of D bf16 values becomes
 * e4m3(q * 2^e) * 2^-e with 2^e the power of two that puts max|q| of the row
 * in [128, 256) (e = 7 - floor(log2 max|q|)); an all-zero row stays zero.
 * The product q * 2^e is exact in single precision, so the quantised code is
 * decided as the kernel decides it. The result is exactly representable in
 * bf16 (3 mantissa bits), so it is returned as bf16 bits and the attention
 * routine runs on it unchanged.
 */
int oracle_quantize_q_e4m3(const uint16_t* q, int64_t rows, int D, uint16_t* q_out) {
  if (rows < 0 || D < 1) return ORACLE_BAD_ARG;
  for (int64_t r = 0; r < rows; ++r) {
    double mx = 0.0;
    for (int d = 0; d < D; ++d) {
      const double v = fabs(oracle_bf16_to_double(q[r * D + d]));
      if (v > mx) mx = v;
    }
    const int e = mx > 0.0 ? 7 - ilogb(mx) : 0;
    for (int d = 0; d < D; ++d) {
      const float x = (float)ldexp(oracle_bf16_to_double(q[r * D + d]), e);
      const double v = ldexp(oracle_e4m3_to_double(oracle_e4m3_encode(x)), -e);
      const float f = (float)v;  /* exact */
      uint32_t bits;
      memcpy(&bits, &f, sizeof bits);
      q_out[r * D + d] = (uint16_t)(bits >> 16);  /* low half is zero */
    }
  }
  return ORACLE_OK;
}

/*
 * Paged KV append (the KV-cache producer): new row t of sequence b goes to
 * logical position pos = kv_lens[b] + t, i.e. page page_table[b][pos / P],
 * slot pos % P, for every kv head. bf16 pools receive the bits unchanged;
 * FP8 pools receive oracle_e4m3_encode(x / kv_scale), the quotient taken in
 * single precision (the precision in which the quantised code is decided).
 *
 * k_new, v_new  bf16 bits [B, num_new, Hkv, D]
 * k/v_pages     bf16 bits or e4m3 bytes [num_pages, Hkv, P, D], or NVFP4
 *               code bytes [num_pages, Hkv, P, D/2], updated in place
 * k/v_scales    NVFP4 only: e4m3 block scales [num_pages, Hkv, P, D/16],
 *               updated in place (oracle_nvfp4_encode_block per 16 elements);
 *               NULL otherwise
 * Returns ORACLE_BAD_PAGE (writing nothing more) at the first position past
 * the page table or page id out of range.
 */
int oracle_paged_kv_append(const uint16_t* k_new, const uint16_t* v_new,
                           const int32_t* page_table, const int32_t* kv_lens, int B,
                           int num_new, int Hkv, int D, int page_size, int max_pages,
                           int num_pages, int kv_dtype, float kv_scale, void* k_pages,
                           void* v_pages, void* k_scales, void* v_scales) {
  if (B < 0 || num_new < 1 || Hkv < 1 || D < 1 || page_size < 1 || max_pages < 1 ||
      num_pages < 1)
    return ORACLE_BAD_ARG;
  if (kv_dtype != ORACLE_KV_BF16 && kv_dtype != ORACLE_KV_FP8_E4M3 &&
      kv_dtype != ORACLE_KV_NVFP4)
    return ORACLE_BAD_ARG;
  if (kv_dtype == ORACLE_KV_NVFP4 && (D % 16 != 0 || !k_scales || !v_scales))
    return ORACLE_BAD_ARG;
  for (int b = 0; b < B; ++b) {
    for (int t = 0; t < num_new; ++t) {
      const int64_t pos = (int64_t)kv_lens[b] + t;
      if (kv_lens[b] < 0 || pos >= (int64_t)max_pages * page_size) return ORACLE_BAD_PAGE;
      const int32_t page = page_table[(int64_t)b * max_pages + pos / page_size];
      if (page < 0 || page >= num_pages) return ORACLE_BAD_PAGE;
      for (int h = 0; h < Hkv; ++h) {
        const int64_t src = (((int64_t)b * num_new + t) * Hkv + h) * D;
        const int64_t dst = (((int64_t)page * Hkv + h) * page_size + pos % page_size) * D;
        if (kv_dtype == ORACLE_KV_NVFP4) {
          for (int blk = 0; blk < D / 16; ++blk) {
            for (int which = 0; which < 2; ++which) {
              const uint16_t* x = (which ? v_new : k_new) + src + 16 * blk;
              uint8_t* codes = (uint8_t*)(which ? v_pages : k_pages);
              uint8_t* scales = (uint8_t*)(which ? v_scales : k_scales);
              uint8_t c[16];
              oracle_nvfp4_encode_block(x, kv_scale, c, &scales[dst / 16 + blk]);
              for (int d = 0; d < 16; d += 2)
                codes[(dst + 16 * blk + d) / 2] = (uint8_t)(c[d] | (c[d + 1] << 4));
            }
          }
          continue;
        }
        for (int d = 0; d < D; ++d) {
          if (kv_dtype == ORACLE_KV_BF16) {
            ((uint16_t*)k_pages)[dst + d] = k_new[src + d];
            ((uint16_t*)v_pages)[dst + d] = v_new[src + d];
          } else {
            const float kx = (float)oracle_bf16_to_double(k_new[src + d]);
            const float vx = (float)oracle_bf16_to_double(v_new[src + d]);
            ((uint8_t*)k_pages)[dst + d] = oracle_e4m3_encode(kx / kv_scale);
            ((uint8_t*)v_pages)[dst + d] = oracle_e4m3_encode(vx / kv_scale);
          }
        }
      }
    }
  }
  return ORACLE_OK;
}

/*
 * Log-sum-exp merge of n attention states over disjoint key sets
 * (merge_attn_states / PagedPersistentMergeKernel):
 *   lse = m* + ln sum_s exp(lse_s - m*),  m* = max_s lse_s
 *   out = sum_s exp(lse_s - lse) * out_s
 * All states empty (every lse_s = -inf): out = 0, lse = -inf.
 *
 * o_parts [n, rows, D], lse_parts [n, rows]; out [rows, D], lse [rows].
 */
int oracle_merge_states(const double* o_parts, const double* lse_parts, int n,
                        int64_t rows, int D, double* out, double* lse) {
  if (n < 1 || rows < 0 || D < 1) return ORACLE_BAD_ARG;
  for (int64_t r = 0; r < rows; ++r) {
    double m = -INFINITY;
    for (int s = 0; s < n; ++s)
      if (lse_parts[(int64_t)s * rows + r] > m) m = lse_parts[(int64_t)s * rows + r];
    double* orow = out + r * D;
    if (m == -INFINITY) {
      for (int d = 0; d < D; ++d) orow[d] = 0.0;
      lse[r] = -INFINITY;
      continue;
    }
    double sum = 0.0;
    for (int s = 0; s < n; ++s) {
      const double ls = lse_parts[(int64_t)s * rows + r];
      if (ls != -INFINITY) sum += exp(ls - m);
    }
    const double total = m + log(sum);
    lse[r] = total;
    for (int d = 0; d < D; ++d) orow[d] = 0.0;
    for (int s = 0; s < n; ++s) {
      const double ls = lse_parts[(int64_t)s * rows + r];
      if (ls == -INFINITY) continue;
      const double w = exp(ls - total);
      const double* op = o_parts + ((int64_t)s * rows + r) * D;
      for (int d = 0; d < D; ++d) orow[d] += w * op[d];
    }
  }
  return ORACLE_OK;
}
