/*
 * Plain CPU oracle for paged-KV decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (the CUDA library) never calls it, and the two share no code.
 *
 * What it computes, and where the pages define it:
 *
 *  - KV-cache size.  "LLM推理显存优化KV Cache管理3大策略" (mlqm.cn), §1: bytes =
 *    2 x layers x hidden x seq x sizeof(dtype); "生产级 LLM 推理的 KV 缓存优化"
 *    (GPUYard), §2: bytes = 2 x batch x seq x layers x kv_heads x head_dim x
 *    precision bytes.  hidden = kv_heads x head_dim makes the two the same.
 *
 *  - Append.  "大模型推理加速实战：KV Cache内存优化与PagedAttention分页管理方案"
 *    (yunthe.com), KV-cache overhead section: each new token's K/V is written
 *    to the cache.  mlqm.cn §2 (the Block class): a block holds block_size
 *    token rows of hidden values.  A token bound for slot s goes to
 *    physical block s / block_size, row s % block_size.
 *
 *  - INT8 quantisation.  mlqm.cn §4 (quantize_tensor): scale = 127 / max|x|
 *    over the last axis (head_dim), code = clamp(round(x * scale), -128, 127),
 *    evaluated in fp32 with round-half-to-even and no fused multiply-add
 *    (this file is built with -ffp-contract=off).  An all-zero row has no
 *    defined scale on the page; the reading taken is codes 0, scale 1.
 *    Dequantisation is code / scale (the page's dequant_matmul multiplies by
 *    the scales, which would be off by scale^2 given the definition above).
 *
 *  - FP8 (E4M3) quantisation.  GPUYard, serving flags (--kv-cache-dtype fp8
 *    halves the per-token cache) and yunthe.com, KV quantisation section
 *    (FP8/INT8 KV).  The pages give no rule; the reading taken mirrors the
 *    INT8 one: per token per head, scale = 448 / max|x| (448 = largest finite
 *    E4M3 value), code = E4M3(x * scale) rounded to nearest-even and saturated
 *    to +-448, all in fp32; dequantised value = E4M3 value / scale.  E4M3 is the
 *    OCP 8-bit format: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, no
 *    infinities, S.1111.111 = NaN; subnormals 2^-6 * m/8.
 *
 *  - Decode attention.  yunthe.com, PagedAttention section: the kernel looks
 *    up physical blocks through the block table, stitches the scattered K/V
 *    back together and runs standard attention.  mlqm.cn §3 (GQA example,
 *    the Q.view(batch, seq, n_heads // group, group, dim) grouping): q head
 *    h reads K/V head h / group, group = n_q / n_kv.  So, per sequence s and
 *    q head h, with ctx = context_lens[s]:
 *        K_s[t] = k_cache[block_table[s][t / bs]][t % bs]      (0 <= t < ctx)
 *        z_t    = softmax_scale * <q[s][h], K_s[t][h / group]>
 *        p      = softmax(z)                 (max-subtracted, fp64)
 *        out    = sum_t p_t * V_s[t][h / group]
 *    ctx = 0 gives a zero output (the pages are silent; reading taken).
 *
 * Every floating-point step of the attention is in fp64 on the stored values
 * (fp32 inputs widened exactly; bf16 values arrive already widened to fp32,
 * which is exact).  OpenMP runs independent (sequence, kv head) problems in
 * parallel; nothing inside one problem is reordered, blocked or fused.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_BLOCK (-2)
#define ORACLE_ERR_SLOT (-3)

/* ---------------------------------------------------------------- size */

/* GPUYard §2 formula, in exact integer arithmetic.  Returns bytes. */
uint64_t oracle_kv_cache_bytes(uint64_t batch, uint64_t seq_len, uint64_t num_layers,
                               uint64_t num_kv_heads, uint64_t head_dim, uint64_t dtype_bytes) {
  return 2ull * batch * seq_len * num_layers * num_kv_heads * head_dim * dtype_bytes;
}

/* ---------------------------------------------------------------- append */

/* Copy each token's row (all kv heads, row_bytes bytes) into its slot.
 * x: [num_tokens][row_bytes]; cache: [num_blocks][block_size][row_bytes].
 * A negative slot means "no write" (padding).  A slot past the pool is an
 * error and nothing further is written. */
int oracle_append_rows(const uint8_t* x, const int64_t* slot_mapping, int64_t num_tokens,
                       int64_t row_bytes, uint8_t* cache, int64_t num_blocks, int64_t block_size) {
  if (!x || !slot_mapping || !cache || num_tokens < 0 || row_bytes <= 0 || num_blocks <= 0 ||
      block_size <= 0)
    return ORACLE_ERR_ARG;
  for (int64_t t = 0; t < num_tokens; ++t) {
    int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    int64_t block = slot / block_size;
    int64_t offset = slot % block_size;
    if (block >= num_blocks) return ORACLE_ERR_SLOT;
    uint8_t* dst = cache + (block * block_size + offset) * row_bytes;
    memcpy(dst, x + t * row_bytes, (size_t)row_bytes);
  }
  return ORACLE_OK;
}

/* mlqm.cn §4 quantize_tensor on one row of n fp32 values. */
void oracle_quantize_row(const float* x, int n, int8_t* codes, float* scale_out) {
  float absmax = 0.0f;
  for (int i = 0; i < n; ++i) {
    float a = fabsf(x[i]);
    if (a > absmax) absmax = a;
  }
  if (absmax == 0.0f) { /* reading: an all-zero row stores codes 0, scale 1 */
    for (int i = 0; i < n; ++i) codes[i] = 0;
    *scale_out = 1.0f;
    return;
  }
  float scale = 127.0f / absmax;
  for (int i = 0; i < n; ++i) {
    float y = x[i] * scale;       /* one fp32 multiply, rounded */
    float r = nearbyintf(y);      /* default mode: round half to even */
    if (r > 127.0f) r = 127.0f;
    if (r < -128.0f) r = -128.0f;
    codes[i] = (int8_t)r;
  }
  *scale_out = scale;
}

/* E4M3 value of an 8-bit code (NaN codes decode to NaN). */
double oracle_e4m3_decode(uint8_t code) {
  const int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  double v = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

/* Nearest E4M3 code to y (ties to even mantissa), magnitudes above 448
 * saturated to 448.  y must not be NaN. */
uint8_t oracle_e4m3_encode(float y) {
  const int sign = y < 0.0f || (y == 0.0f && signbit(y));
  double a = fabs((double)y);
  if (a >= 448.0) return (uint8_t)((sign << 7) | (15 << 3) | 6);
  /* spacing of representable values around a: 2^(e-3) in binade [2^e, 2^(e+1)),
   * e >= -6; below 2^-6 the subnormal spacing 2^-9 */
  int ex;
  frexp(a, &ex); /* a = f * 2^ex, f in [0.5, 1) */
  int e = ex - 1;
  if (a == 0.0 || e < -6) e = -6;
  const double q = ldexp(1.0, e - 3);
  const double mi = nearbyint(a / q); /* exact quotient, rounded half to even */
  const double v = mi * q;            /* may reach 2^(e+1): still representable */
  if (v >= 448.0) return (uint8_t)((sign << 7) | (15 << 3) | 6);
  int code;
  if (v < ldexp(1.0, -6)) {
    code = (int)(v / ldexp(1.0, -9)); /* subnormal: m = v / 2^-9 */
  } else {
    int vx;
    frexp(v, &vx);
    const int ve = vx - 1;
    const int m = (int)((v / ldexp(1.0, ve) - 1.0) * 8.0);
    code = ((ve + 7) << 3) | m;
  }
  return (uint8_t)((sign << 7) | code);
}

/* FP8 quantisation of one fp32 row: scale = 448 / max|x|, codes E4M3(x*scale). */
void oracle_quantize_row_fp8(const float* x, int n, uint8_t* codes, float* scale_out) {
  float absmax = 0.0f;
  for (int i = 0; i < n; ++i) {
    float a = fabsf(x[i]);
    if (a > absmax) absmax = a;
  }
  if (absmax == 0.0f) { /* same reading as INT8: codes 0, scale 1 */
    for (int i = 0; i < n; ++i) codes[i] = 0;
    *scale_out = 1.0f;
    return;
  }
  float scale = 448.0f / absmax;
  for (int i = 0; i < n; ++i) {
    float y = x[i] * scale; /* one fp32 multiply, rounded */
    codes[i] = oracle_e4m3_encode(y);
  }
  *scale_out = scale;
}

/* FP8 quantising append; layouts as oracle_append_int8. */
int oracle_append_fp8(const float* x, const int64_t* slot_mapping, int64_t num_tokens,
                      int num_kv_heads, int head_dim, uint8_t* codes, float* scale,
                      int64_t num_blocks, int64_t block_size) {
  if (!x || !slot_mapping || !codes || !scale || num_tokens < 0 || num_kv_heads <= 0 ||
      head_dim <= 0 || num_blocks <= 0 || block_size <= 0)
    return ORACLE_ERR_ARG;
  for (int64_t t = 0; t < num_tokens; ++t) {
    int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    int64_t block = slot / block_size;
    int64_t offset = slot % block_size;
    if (block >= num_blocks) return ORACLE_ERR_SLOT;
    for (int h = 0; h < num_kv_heads; ++h) {
      const float* row = x + (t * num_kv_heads + h) * (int64_t)head_dim;
      uint8_t* dst = codes + ((block * block_size + offset) * num_kv_heads + h) * (int64_t)head_dim;
      float* s = scale + (block * num_kv_heads + h) * block_size + offset;
      oracle_quantize_row_fp8(row, head_dim, dst, s);
    }
  }
  return ORACLE_OK;
}

/* Quantising append: x fp32 [num_tokens][num_kv_heads][head_dim].
 * codes: [num_blocks][block_size][num_kv_heads][head_dim] int8.
 * scale: [num_blocks][num_kv_heads][block_size] fp32 (one per token per head). */
int oracle_append_int8(const float* x, const int64_t* slot_mapping, int64_t num_tokens,
                       int num_kv_heads, int head_dim, int8_t* codes, float* scale,
                       int64_t num_blocks, int64_t block_size) {
  if (!x || !slot_mapping || !codes || !scale || num_tokens < 0 || num_kv_heads <= 0 ||
      head_dim <= 0 || num_blocks <= 0 || block_size <= 0)
    return ORACLE_ERR_ARG;
  for (int64_t t = 0; t < num_tokens; ++t) {
    int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    int64_t block = slot / block_size;
    int64_t offset = slot % block_size;
    if (block >= num_blocks) return ORACLE_ERR_SLOT;
    for (int h = 0; h < num_kv_heads; ++h) {
      const float* row = x + (t * num_kv_heads + h) * (int64_t)head_dim;
      int8_t* dst = codes + ((block * block_size + offset) * num_kv_heads + h) * (int64_t)head_dim;
      float* s = scale + (block * num_kv_heads + h) * block_size + offset;
      oracle_quantize_row(row, head_dim, dst, s);
    }
  }
  return ORACLE_OK;
}

/* Whole-block copy between pools (copy-on-write, swap): block pairs[2i] of src
 * to block pairs[2i+1] of dst, block_bytes each.  Out-of-range ids are an error
 * and nothing further is copied. */
int oracle_copy_blocks(uint8_t* dst, const uint8_t* src, int64_t block_bytes, int dst_blocks,
                       int src_blocks, const int32_t* pairs, int num_pairs) {
  if (!dst || !src || !pairs || block_bytes <= 0 || num_pairs < 0) return ORACLE_ERR_ARG;
  for (int i = 0; i < num_pairs; ++i) {
    const int32_t s = pairs[2 * i], d = pairs[2 * i + 1];
    if (s < 0 || s >= src_blocks || d < 0 || d >= dst_blocks) return ORACLE_ERR_BLOCK;
    memcpy(dst + (int64_t)d * block_bytes, src + (int64_t)s * block_bytes, (size_t)block_bytes);
  }
  return ORACLE_OK;
}

/* ---------------------------------------------------------------- gather */

/* Gather kv head kvh of sequence s's first ctx tokens into contiguous fp64
 * rows dst[t][head_dim], walking the block table. */
static int gather_f32(double* dst, const float* cache, const int32_t* table_row, int ctx,
                      int num_kv_heads, int kvh, int head_dim, int block_size, int num_blocks) {
  const int64_t row = (int64_t)num_kv_heads * head_dim;
  for (int t = 0; t < ctx; ++t) {
    int32_t phys = table_row[t / block_size];
    if (phys < 0 || phys >= num_blocks) return ORACLE_ERR_BLOCK;
    const float* src = cache + ((int64_t)phys * block_size + t % block_size) * row +
                       (int64_t)kvh * head_dim;
    for (int i = 0; i < head_dim; ++i) dst[(int64_t)t * head_dim + i] = (double)src[i];
  }
  return ORACLE_OK;
}

/* Same walk for a quantised cache, dequantising each value as value(code) /
 * scale, value(code) = the signed byte (INT8) or its E4M3 value (FP8). */
static int gather_codes(double* dst, const uint8_t* codes, const float* scale,
                        const int32_t* table_row, int ctx, int num_kv_heads, int kvh, int head_dim,
                        int block_size, int num_blocks, int fp8) {
  const int64_t row = (int64_t)num_kv_heads * head_dim;
  for (int t = 0; t < ctx; ++t) {
    int32_t phys = table_row[t / block_size];
    if (phys < 0 || phys >= num_blocks) return ORACLE_ERR_BLOCK;
    int off = t % block_size;
    const uint8_t* src = codes + ((int64_t)phys * block_size + off) * row + (int64_t)kvh * head_dim;
    double s = (double)scale[((int64_t)phys * num_kv_heads + kvh) * block_size + off];
    for (int i = 0; i < head_dim; ++i) {
      double v = fp8 ? oracle_e4m3_decode(src[i]) : (double)(int8_t)src[i];
      dst[(int64_t)t * head_dim + i] = v / s;
    }
  }
  return ORACLE_OK;
}

/* Exposed for the block-table worked example: gathers one sequence, all heads,
 * into dst[t][num_kv_heads][head_dim]. */
int oracle_gather_f32(double* dst, const float* cache, const int32_t* table_row, int ctx,
                      int num_kv_heads, int head_dim, int block_size, int num_blocks) {
  if (!dst || !cache || !table_row || ctx < 0) return ORACLE_ERR_ARG;
  double* one = (double*)malloc(sizeof(double) * (size_t)(ctx > 0 ? ctx : 1) * head_dim);
  int rc = ORACLE_OK;
  for (int h = 0; h < num_kv_heads && rc == ORACLE_OK; ++h) {
    rc = gather_f32(one, cache, table_row, ctx, num_kv_heads, h, head_dim, block_size, num_blocks);
    for (int t = 0; rc == ORACLE_OK && t < ctx; ++t)
      for (int i = 0; i < head_dim; ++i)
        dst[((int64_t)t * num_kv_heads + h) * head_dim + i] = one[(int64_t)t * head_dim + i];
  }
  free(one);
  return rc;
}

/* ---------------------------------------------------------------- attention */

/* Standard attention of one q head over contiguous K/V rows (fp64).
 * q: [head_dim]; K,V: [ctx][head_dim]. */
static void attend_one(double* out, const float* q, const double* K, const double* V, int ctx,
                       int head_dim, double softmax_scale, double* z) {
  for (int i = 0; i < head_dim; ++i) out[i] = 0.0;
  if (ctx == 0) return;
  double zmax = -INFINITY;
  for (int t = 0; t < ctx; ++t) {
    const double* k = K + (int64_t)t * head_dim;
    double dot = 0.0;
    for (int i = 0; i < head_dim; ++i) dot += (double)q[i] * k[i];
    z[t] = softmax_scale * dot;
    if (z[t] > zmax) zmax = z[t];
  }
  double denom = 0.0;
  for (int t = 0; t < ctx; ++t) {
    z[t] = exp(z[t] - zmax);
    denom += z[t];
  }
  for (int t = 0; t < ctx; ++t) {
    const double* v = V + (int64_t)t * head_dim;
    double p = z[t] / denom;
    for (int i = 0; i < head_dim; ++i) out[i] += p * v[i];
  }
}

static int check_shapes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                        int block_size, int num_blocks, int max_blocks_per_seq,
                        const int32_t* context_lens) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_blocks <= 0 || max_blocks_per_seq < 0 || num_q_heads % num_kv_heads != 0)
    return ORACLE_ERR_ARG;
  for (int s = 0; s < num_seqs; ++s) {
    if (context_lens[s] < 0) return ORACLE_ERR_ARG;
    if ((int64_t)context_lens[s] > (int64_t)max_blocks_per_seq * block_size) return ORACLE_ERR_ARG;
  }
  return ORACLE_OK;
}

/* One (sequence, kv head) problem: gather that head's K/V rows of the
 * sequence, then attend for each q head h with h / group == kvh. */
static int decode_problem(double* out, const float* q, const float* k_cache, const float* v_cache,
                          const uint8_t* k_codes, const uint8_t* v_codes, int fp8, const float* k_scale,
                          const float* v_scale, const int32_t* block_tables,
                          int max_blocks_per_seq, const int32_t* context_lens, int s, int kvh,
                          int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                          int num_blocks, double softmax_scale) {
  const int ctx = context_lens[s];
  const int group = num_q_heads / num_kv_heads;
  const size_t n = (size_t)(ctx > 0 ? ctx : 1);
  double* K = (double*)malloc(sizeof(double) * n * head_dim);
  double* V = (double*)malloc(sizeof(double) * n * head_dim);
  double* z = (double*)malloc(sizeof(double) * n);
  const int32_t* trow = block_tables + (int64_t)s * max_blocks_per_seq;
  int e;
  if (k_codes) {
    e = gather_codes(K, k_codes, k_scale, trow, ctx, num_kv_heads, kvh, head_dim, block_size,
                     num_blocks, fp8);
    if (!e)
      e = gather_codes(V, v_codes, v_scale, trow, ctx, num_kv_heads, kvh, head_dim, block_size,
                       num_blocks, fp8);
  } else {
    e = gather_f32(K, k_cache, trow, ctx, num_kv_heads, kvh, head_dim, block_size, num_blocks);
    if (!e)
      e = gather_f32(V, v_cache, trow, ctx, num_kv_heads, kvh, head_dim, block_size, num_blocks);
  }
  if (!e) {
    for (int h = 0; h < num_q_heads; ++h) {
      if (h / group != kvh) continue;
      const int64_t r = ((int64_t)s * num_q_heads + h) * head_dim;
      attend_one(out + r, q + r, K, V, ctx, head_dim, softmax_scale, z);
    }
  }
  free(K);
  free(V);
  free(z);
  return e;
}

static int decode_all(double* out, const float* q, const float* k_cache, const float* v_cache,
                      const uint8_t* k_codes, const uint8_t* v_codes, int fp8, const float* k_scale,
                      const float* v_scale, const int32_t* block_tables, int max_blocks_per_seq,
                      const int32_t* context_lens, int num_seqs, int num_q_heads,
                      int num_kv_heads, int head_dim, int block_size, int num_blocks,
                      double softmax_scale, int num_threads) {
  int rc = check_shapes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                        max_blocks_per_seq, context_lens);
  if (rc) return rc;
  int err = ORACLE_OK;
  const int64_t problems = (int64_t)num_seqs * num_kv_heads;
#ifdef _OPENMP
  if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int64_t i = 0; i < problems; ++i) {
    int e = decode_problem(out, q, k_cache, v_cache, k_codes, v_codes, fp8, k_scale, v_scale,
                           block_tables, max_blocks_per_seq, context_lens, (int)(i / num_kv_heads),
                           (int)(i % num_kv_heads), num_q_heads, num_kv_heads, head_dim,
                           block_size, num_blocks, softmax_scale);
    if (e) {
#ifdef _OPENMP
#pragma omp critical
#endif
      err = e;
    }
  }
  return err;
}

/* Paged decode over an fp32-valued cache (bf16 caches are passed widened).
 * out: [num_seqs][num_q_heads][head_dim] fp64; q: same shape, fp32-valued.
 * k_cache, v_cache: [num_blocks][block_size][num_kv_heads][head_dim].
 * block_tables: [num_seqs][max_blocks_per_seq]; context_lens: [num_seqs]. */
int oracle_paged_decode_f32(double* out, const float* q, const float* k_cache,
                            const float* v_cache, const int32_t* block_tables,
                            int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                            int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                            int num_blocks, double softmax_scale, int num_threads) {
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return ORACLE_ERR_ARG;
  return decode_all(out, q, k_cache, v_cache, NULL, NULL, 0, NULL, NULL, block_tables,
                    max_blocks_per_seq, context_lens, num_seqs, num_q_heads, num_kv_heads,
                    head_dim, block_size, num_blocks, softmax_scale, num_threads);
}

/* Paged decode over an INT8 cache: codes [num_blocks][block_size][num_kv_heads]
 * [head_dim], scales [num_blocks][num_kv_heads][block_size]; values are
 * dequantised as code / scale before the fp64 attention above. */
int oracle_paged_decode_i8(double* out, const float* q, const int8_t* k_codes,
                           const int8_t* v_codes, const float* k_scale, const float* v_scale,
                           const int32_t* block_tables, int max_blocks_per_seq,
                           const int32_t* context_lens, int num_seqs, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size, int num_blocks,
                           double softmax_scale, int num_threads) {
  if (!out || !q || !k_codes || !v_codes || !k_scale || !v_scale || !block_tables || !context_lens)
    return ORACLE_ERR_ARG;
  return decode_all(out, q, NULL, NULL, (const uint8_t*)k_codes, (const uint8_t*)v_codes, 0,
                    k_scale, v_scale, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                    num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, softmax_scale,
                    num_threads);
}

/* Paged decode over an FP8 (E4M3) cache: codes and scales laid out as for
 * INT8; values are dequantised as E4M3(code) / scale. */
int oracle_paged_decode_fp8(double* out, const float* q, const uint8_t* k_codes,
                            const uint8_t* v_codes, const float* k_scale, const float* v_scale,
                            const int32_t* block_tables, int max_blocks_per_seq,
                            const int32_t* context_lens, int num_seqs, int num_q_heads,
                            int num_kv_heads, int head_dim, int block_size, int num_blocks,
                            double softmax_scale, int num_threads) {
  if (!out || !q || !k_codes || !v_codes || !k_scale || !v_scale || !block_tables || !context_lens)
    return ORACLE_ERR_ARG;
  return decode_all(out, q, NULL, NULL, k_codes, v_codes, 1, k_scale, v_scale, block_tables,
                    max_blocks_per_seq, context_lens, num_seqs, num_q_heads, num_kv_heads,
                    head_dim, block_size, num_blocks, softmax_scale, num_threads);
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
