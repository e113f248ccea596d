/*
 * pkv_oracle.c -- plain fp64 CPU oracle for paged KV append and paged decode
 * attention.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the bench's CPU
 * baseline leg load this library.  It shares no code, header, table or helper
 * with the CUDA library and is deliberately slow and obvious: it gathers each
 * sequence's blocks into a contiguous fp64 K and V and then evaluates the
 * textbook definition of single-query attention.
 *
 * What it follows:
 *   - attention of the new token over all cached tokens: dot Q with every K,
 *     softmax, weighted sum of V ("KV Cache and PagedAttention" (gyaansetu),
 *     section "attention computation", steps 1-4; "PagedAttention: KV cache
 *     memory management" (yfxerp) §3.2, Q K^T / sqrt(d) -> softmax -> V);
 *   - the per-layer cache K, V in R^{B x h_kv x T x d_h} with GQA, h_kv < h_q
 *     ("Transformer anatomy" ch. 15 §15.2);
 *   - blocks of 16 tokens reached through a per-sequence block table whose
 *     entry i names the physical block of logical block i; a new token is
 *     written into the current block ("Transformer anatomy" ch. 15 §15.5;
 *     "LLM Primer VI" ch. 8 §8.1).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - q head h reads kv head h / (n_q / n_kv) (contiguous GQA groups);
 *   - within a physical block the layout is [n_kv][block_size][head_dim];
 *   - slot s names physical block s / block_size, offset s % block_size; a
 *     negative slot is padding and is skipped;
 *   - the per-page softmax of the yfxerp pseudocode is read as one softmax
 *     over every token of the context;
 *   - context length 0 yields an all-zero output row.
 *
 * Precision: every element is widened exactly to double (the conversions are
 * written out below from the IEEE 754 binary16 and bfloat16 definitions) and
 * all arithmetic is done in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_F16 = 1, ORC_BF16 = 2 };

enum {
  ORC_OK = 0,
  ORC_EINVAL = -1,     /* bad sizes, dtype or head counts */
  ORC_ESLOT = -2,      /* slot beyond the pool */
  ORC_EBLOCK = -3,     /* block table entry outside [0, num_blocks) */
  ORC_ECTX = -4,       /* context length negative or beyond the table */
  ORC_ENOMEM = -5
};

static int elem_bytes(int dtype) {
  switch (dtype) {
    case ORC_F32: return 4;
    case ORC_F16: return 2;
    case ORC_BF16: return 2;
    default: return 0;
  }
}

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double f16_bits_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int expo = (h >> 10) & 0x1f;
  int frac = h & 0x3ff;
  double mag;
  if (expo == 0) {
    mag = ldexp((double)frac, -24);                   /* subnormal: frac * 2^-24 */
  } else if (expo == 31) {
    mag = frac ? NAN : INFINITY;
  } else {
    mag = ldexp((double)(1024 + frac), expo - 25);    /* (1.frac) * 2^(expo-15) */
  }
  return sign ? -mag : mag;
}

/* bfloat16 is the upper half of an IEEE binary32. */
static double bf16_bits_to_double(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double load_elem(const void* base, size_t idx, int dtype) {
  if (dtype == ORC_F32) {
    float f;
    memcpy(&f, (const char*)base + idx * 4, 4);
    return (double)f;
  }
  uint16_t h;
  memcpy(&h, (const char*)base + idx * 2, 2);
  return dtype == ORC_F16 ? f16_bits_to_double(h) : bf16_bits_to_double(h);
}

/* Widen a buffer of n elements of `dtype` to double. */
int oracle_widen(const void* src, int dtype, int64_t n, double* dst) {
  if (!elem_bytes(dtype) || n < 0) return ORC_EINVAL;
  for (int64_t i = 0; i < n; ++i) dst[i] = load_elem(src, (size_t)i, dtype);
  return ORC_OK;
}

/*
 * Cache append: for every token i with slot s = slot_mapping[i] >= 0, copy
 * k[i][h][:] to k_cache[s / block_size][h][s % block_size][:] for every kv
 * head h, and likewise v.  Byte copies: the result is bit-exact by definition.
 */
int oracle_kv_append(const void* k, const void* v, const int64_t* slot_mapping,
                     int32_t num_tokens, void* k_cache, void* v_cache,
                     int32_t num_blocks, int32_t block_size, int32_t n_kv_heads,
                     int32_t head_dim, int32_t dtype) {
  int es = elem_bytes(dtype);
  if (!es || num_tokens < 0 || num_blocks <= 0 || block_size <= 0 ||
      n_kv_heads <= 0 || head_dim <= 0)
    return ORC_EINVAL;
  size_t row = (size_t)head_dim * es;
  int64_t n_slots = (int64_t)num_blocks * block_size;
  for (int32_t i = 0; i < num_tokens; ++i) {
    int64_t s = slot_mapping[i];
    if (s < 0) continue;
    if (s >= n_slots) return ORC_ESLOT;
    int64_t blk = s / block_size, off = s % block_size;
    for (int32_t h = 0; h < n_kv_heads; ++h) {
      size_t src = ((size_t)i * n_kv_heads + h) * row;
      size_t dst = (((size_t)blk * n_kv_heads + h) * block_size + off) * row;
      memcpy((char*)k_cache + dst, (const char*)k + src, row);
      memcpy((char*)v_cache + dst, (const char*)v + src, row);
    }
  }
  return ORC_OK;
}

/*
 * One output row: sequence b, query head h.
 *   kv = h / (n_q / n_kv)
 *   K[j], V[j] = cache rows of logical token j (0 <= j < ctx), gathered
 *                through block_tables[b][j / block_size]
 *   s_j  = scale * sum_e q[b][h][e] * K[j][e]
 *   m    = max_j s_j,   w_j = exp(s_j - m)
 *   out[e] = sum_j w_j V[j][e] / sum_j w_j
 */
static int decode_row(const void* q, const void* k_cache, const void* v_cache, int dtype,
                      const int32_t* block_tables, int32_t max_blocks_per_seq,
                      const int32_t* context_lens, int32_t num_blocks, double scale,
                      int32_t n_q, int32_t n_kv, int32_t d, int32_t bs,
                      int32_t b, int32_t h, double* out_row) {
  int32_t group = n_q / n_kv;
  int32_t kvh = h / group;
  int32_t ctx = context_lens[b];
  if (ctx < 0 || (int64_t)ctx > (int64_t)max_blocks_per_seq * bs) return ORC_ECTX;
  for (int32_t e = 0; e < d; ++e) out_row[e] = 0.0;
  if (ctx == 0) return ORC_OK;

  double* K = (double*)malloc(sizeof(double) * (size_t)ctx * d);
  double* V = (double*)malloc(sizeof(double) * (size_t)ctx * d);
  double* s = (double*)malloc(sizeof(double) * (size_t)ctx);
  double* qv = (double*)malloc(sizeof(double) * (size_t)d);
  if (!K || !V || !s || !qv) {
    free(K); free(V); free(s); free(qv);
    return ORC_ENOMEM;
  }

  /* Gather: logical token j lives in physical block table[j / bs], slot j % bs. */
  for (int32_t j = 0; j < ctx; ++j) {
    int32_t phys = block_tables[(size_t)b * max_blocks_per_seq + j / bs];
    if (phys < 0 || phys >= num_blocks) {
      free(K); free(V); free(s); free(qv);
      return ORC_EBLOCK;
    }
    size_t base = (((size_t)phys * n_kv + kvh) * bs + (j % bs)) * (size_t)d;
    for (int32_t e = 0; e < d; ++e) {
      K[(size_t)j * d + e] = load_elem(k_cache, base + e, dtype);
      V[(size_t)j * d + e] = load_elem(v_cache, base + e, dtype);
    }
  }
  for (int32_t e = 0; e < d; ++e) qv[e] = load_elem(q, ((size_t)b * n_q + h) * d + e, dtype);

  /* Scores. */
  for (int32_t j = 0; j < ctx; ++j) {
    double acc = 0.0;
    for (int32_t e = 0; e < d; ++e) acc += qv[e] * K[(size_t)j * d + e];
    s[j] = scale * acc;
  }
  /* Softmax with the maximum subtracted. */
  double m = s[0];
  for (int32_t j = 1; j < ctx; ++j)
    if (s[j] > m) m = s[j];
  double denom = 0.0;
  for (int32_t j = 0; j < ctx; ++j) {
    s[j] = exp(s[j] - m);
    denom += s[j];
  }
  /* Weighted sum of V. */
  for (int32_t j = 0; j < ctx; ++j)
    for (int32_t e = 0; e < d; ++e) out_row[e] += s[j] * V[(size_t)j * d + e];
  for (int32_t e = 0; e < d; ++e) out_row[e] /= denom;

  free(K); free(V); free(s); free(qv);
  return ORC_OK;
}

/*
 * Paged decode attention.  `out` is fp64 [batch][n_q][head_dim].  When `rows`
 * is non-NULL only the n_rows pairs rows[2r] = b, rows[2r+1] = h are computed
 * (the others are left untouched).  n_threads <= 0 uses the OpenMP default.
 */
int oracle_paged_decode(const void* q, const void* k_cache, const void* v_cache, int32_t dtype,
                        const int32_t* block_tables, int32_t max_blocks_per_seq,
                        const int32_t* context_lens, int32_t batch, int32_t num_blocks,
                        double scale, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                        int32_t block_size, double* out, const int32_t* rows, int32_t n_rows,
                        int32_t n_threads) {
  if (!elem_bytes(dtype) || batch < 0 || n_q_heads <= 0 || n_kv_heads <= 0 ||
      n_q_heads % n_kv_heads != 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0 ||
      max_blocks_per_seq <= 0)
    return ORC_EINVAL;
  int64_t total = rows ? (int64_t)n_rows : (int64_t)batch * n_q_heads;
  int status = ORC_OK;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < total; ++r) {
    int32_t b = rows ? rows[2 * r] : (int32_t)(r / n_q_heads);
    int32_t h = rows ? rows[2 * r + 1] : (int32_t)(r % n_q_heads);
    int rc;
    if (b < 0 || b >= batch || h < 0 || h >= n_q_heads) {
      rc = ORC_EINVAL;
    } else {
      rc = decode_row(q, k_cache, v_cache, dtype, block_tables, max_blocks_per_seq,
                      context_lens, num_blocks, scale, n_q_heads, n_kv_heads, head_dim,
                      block_size, b, h, out + ((size_t)b * n_q_heads + h) * head_dim);
    }
    if (rc != ORC_OK) {
#pragma omp critical
      status = rc;
    }
  }
  return status;
}

/*
 * Multi-query decode (several new tokens per sequence: a draft to verify,
 * "LLM Primer VI" ch. 8, speculative decoding; or a prefill chunk).  q and
 * out are [batch][q_len][n_q][head_dim]; the q_len new tokens are the last
 * q_len of the sequence's context (already in the cache), and query i sees
 * the cache up to and including its own position:
 *   ctx_i = context_lens[b] - q_len + i + 1.
 * Each row is the single-query attention above over that prefix (causal
 * among the new tokens).  context_lens[b] < q_len is an error.
 */
int oracle_paged_decode_mq(const void* q, const void* k_cache, const void* v_cache, int32_t dtype,
                           const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                           int32_t batch, int32_t num_blocks, double scale, int32_t n_q_heads,
                           int32_t n_kv_heads, int32_t head_dim, int32_t block_size, int32_t q_len, double* out,
                           int32_t n_threads) {
  int es = elem_bytes(dtype);
  if (!es || batch < 0 || q_len <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads != 0 ||
      head_dim <= 0 || block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0)
    return ORC_EINVAL;
  int64_t total = (int64_t)batch * q_len * n_q_heads;
  int status = ORC_OK;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < total; ++r) {
    int32_t h = (int32_t)(r % n_q_heads);
    int32_t i = (int32_t)((r / n_q_heads) % q_len);
    int32_t b = (int32_t)(r / ((int64_t)n_q_heads * q_len));
    int32_t ctx_i = context_lens[b] - q_len + i + 1;
    int rc;
    if (context_lens[b] < q_len) {
      rc = ORC_ECTX;
    } else {
      /* Query i of sequence b as a one-sequence single-query problem. */
      const char* q_row = (const char*)q + ((size_t)b * q_len + i) * n_q_heads * head_dim * es;
      rc = decode_row(q_row, k_cache, v_cache, dtype, block_tables + (size_t)b * max_blocks_per_seq,
                      max_blocks_per_seq, &ctx_i, num_blocks, scale, n_q_heads, n_kv_heads, head_dim,
                      block_size, 0, h, out + (size_t)r * head_dim);
    }
    if (rc != ORC_OK) {
#pragma omp critical
      status = rc;
    }
  }
  return status;
}

/*
 * ---------------------------------------------------------------------------
 * INT8 paged KV cache (quantised KV: "Transformer anatomy" ch. 15 §15.7, INT8
 * KV quantisation trades a small accuracy loss for half the bytes).
 *
 * Format (a reading: the pages fix neither granularity nor layout).  The
 * cache is one byte array [num_blocks][n_kv][R], R = 32 * d + 128 for block
 * size 16 and head dim d; the record of (block, kv head) holds
 *   bytes [0, 16 d)        K codes: row j (block offset j) of d bytes, whose
 *                          16-byte chunk c sits at chunk position c ^ (j % 8)
 *                          (c ^ (j % 4) for d = 64);
 *   bytes [16 d, 32 d)     V codes transposed: row e (dim e) of 16 bytes, the
 *                          token at block offset j at byte vpos(j) =
 *                          4 * ((j % 8) / 2) + 2 * (j / 8) + (j % 2);
 *   bytes [32 d, 32 d + 64)       16 fp32 K scales (block offset order);
 *   bytes [32 d + 64, 32 d + 128) 16 fp32 V scales.
 * Each (token, kv head) row x of K or V is quantised symmetrically:
 *   amax = max_e |x_e|, scale = amax / 127 (binary32 division),
 *   code_e = clamp(rint(x_e / scale), -127, 127) (binary32 division, rounding
 *   half to even; all codes 0 when amax = 0),
 * and read back as scale * code.  The binary32 steps are what decide the
 * integer codes, so they are done here in binary32 exactly as stated.
 * ---------------------------------------------------------------------------
 */
static int vpos(int j) { return 4 * ((j % 8) / 2) + 2 * (j / 8) + (j % 2); }

static size_t rec_bytes(int32_t d) { return (size_t)32 * d + 128; }

/* Byte of K code (offset j, dim e) inside a record. */
static size_t kpos(int j, int e, int32_t d) {
  int chunks = d / 16;
  int c = e / 16;
  return (size_t)j * d + (size_t)((c ^ (j % (chunks < 8 ? chunks : 8))) * 16 + e % 16);
}

static void quantise_row(const void* src, size_t idx0, int dtype, int32_t d, int8_t* codes, float* scale_out) {
  float amax = 0.0f;
  for (int32_t e = 0; e < d; ++e) {
    float x = (float)load_elem(src, idx0 + e, dtype); /* exact: 16-bit values widen exactly */
    float a = fabsf(x);
    if (a > amax) amax = a;
  }
  float scale = amax / 127.0f;
  for (int32_t e = 0; e < d; ++e) {
    float x = (float)load_elem(src, idx0 + e, dtype);
    float c = amax == 0.0f ? 0.0f : rintf(x / scale);
    if (c > 127.0f) c = 127.0f;
    if (c < -127.0f) c = -127.0f;
    codes[e] = (int8_t)c;
  }
  *scale_out = scale;
}

/* Append into the INT8 cache (block size 16, head dim 64 or 128). */
int oracle_kv_append_int8(const void* k, const void* v, int32_t dtype, const int64_t* slot_mapping,
                          int32_t num_tokens, uint8_t* cache, int32_t num_blocks, int32_t block_size,
                          int32_t n_kv_heads, int32_t head_dim) {
  if (!elem_bytes(dtype) || num_tokens < 0 || num_blocks <= 0 || block_size != 16 || n_kv_heads <= 0 ||
      (head_dim != 64 && head_dim != 128))
    return ORC_EINVAL;
  int8_t* codes = (int8_t*)malloc((size_t)head_dim);
  if (!codes) return ORC_ENOMEM;
  int64_t n_slots = (int64_t)num_blocks * block_size;
  for (int32_t i = 0; i < num_tokens; ++i) {
    int64_t s = slot_mapping[i];
    if (s < 0) continue;
    if (s >= n_slots) {
      free(codes);
      return ORC_ESLOT;
    }
    int64_t blk = s / block_size;
    int off = (int)(s % block_size);
    for (int32_t h = 0; h < n_kv_heads; ++h) {
      size_t src = ((size_t)i * n_kv_heads + h) * head_dim;
      uint8_t* rec = cache + ((size_t)blk * n_kv_heads + h) * rec_bytes(head_dim);
      float sc;
      quantise_row(k, src, dtype, head_dim, codes, &sc);
      for (int32_t e = 0; e < head_dim; ++e) rec[kpos(off, e, head_dim)] = (uint8_t)codes[e];
      memcpy(rec + (size_t)32 * head_dim + 4 * off, &sc, 4);
      quantise_row(v, src, dtype, head_dim, codes, &sc);
      for (int32_t e = 0; e < head_dim; ++e) rec[(size_t)16 * head_dim + (size_t)e * 16 + vpos(off)] = (uint8_t)codes[e];
      memcpy(rec + (size_t)32 * head_dim + 64 + 4 * off, &sc, 4);
    }
  }
  free(codes);
  return ORC_OK;
}

/* The same single-query attention as decode_row, over the dequantised INT8
 * cache (every value scale * code, exact in double). */
static int decode_row_int8(const void* q, int dtype, const uint8_t* cache, const int32_t* block_tables,
                           int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t num_blocks,
                           double scale, int32_t n_q, int32_t n_kv, int32_t d, int32_t bs, int32_t b, int32_t h,
                           double* out_row) {
  int32_t kvh = h / (n_q / n_kv);
  const int32_t ctx = *(context_lens + b);
  if (ctx < 0 || (int64_t)ctx > (int64_t)max_blocks_per_seq * bs) return ORC_ECTX;
  for (int32_t e = 0; e < d; ++e) out_row[e] = 0.0;
  if (ctx == 0) return ORC_OK;
  double* K = (double*)malloc(sizeof(double) * (size_t)ctx * d);
  double* V = (double*)malloc(sizeof(double) * (size_t)ctx * d);
  double* w = (double*)malloc(sizeof(double) * (size_t)ctx);
  double* qv = (double*)malloc(sizeof(double) * (size_t)d);
  if (!K || !V || !w || !qv) {
    free(K); free(V); free(w); free(qv);
    return ORC_ENOMEM;
  }
  for (int32_t j = 0; j < ctx; ++j) {
    int32_t phys = block_tables[(size_t)b * max_blocks_per_seq + (size_t)(j / bs)];
    if (phys < 0 || phys >= num_blocks) {
      free(K); free(V); free(w); free(qv);
      return ORC_EBLOCK;
    }
    const uint8_t* rec = cache + ((size_t)phys * n_kv + kvh) * rec_bytes(d);
    int off = j % bs;
    float ksf, vsf;
    memcpy(&ksf, rec + (size_t)32 * d + 4 * off, 4);
    memcpy(&vsf, rec + (size_t)32 * d + 64 + 4 * off, 4);
    for (int32_t e = 0; e < d; ++e) {
      K[(size_t)j * d + e] = (double)ksf * (double)(int8_t)rec[kpos(off, e, d)];
      V[(size_t)j * d + e] = (double)vsf * (double)(int8_t)rec[(size_t)16 * d + (size_t)e * 16 + vpos(off)];
    }
  }
  for (int32_t e = 0; e < d; ++e) qv[e] = load_elem(q, (size_t)(b * n_q + h) * d + e, dtype);
  /* Scores, softmax with the maximum subtracted, weighted sum of V. */
  for (int32_t j = 0; j < ctx; ++j) {
    double dot = 0.0;
    for (int32_t e = 0; e < d; ++e) dot += qv[e] * K[(size_t)j * d + e];
    w[j] = dot * scale;
  }
  double wmax = w[0];
  for (int32_t j = 1; j < ctx; ++j) wmax = w[j] > wmax ? w[j] : wmax;
  double total = 0.0;
  for (int32_t j = 0; j < ctx; ++j) {
    w[j] = exp(w[j] - wmax);
    total += w[j];
  }
  for (int32_t j = 0; j < ctx; ++j)
    for (int32_t e = 0; e < d; ++e) out_row[e] += w[j] * V[(size_t)j * d + e];
  for (int32_t e = 0; e < d; ++e) out_row[e] = out_row[e] / total;
  free(K); free(V); free(w); free(qv);
  return ORC_OK;
}

int oracle_paged_decode_int8(const void* q, int32_t dtype, const uint8_t* cache, const int32_t* block_tables,
                             int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t batch,
                             int32_t num_blocks, double scale, int32_t n_q_heads, int32_t n_kv_heads,
                             int32_t head_dim, int32_t block_size, double* out, const int32_t* rows,
                             int32_t n_rows, int32_t n_threads) {
  if (!elem_bytes(dtype) || batch < 0 || n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads != 0 ||
      (head_dim != 64 && head_dim != 128) || block_size != 16 || num_blocks <= 0 || max_blocks_per_seq <= 0)
    return ORC_EINVAL;
  int64_t total = rows ? (int64_t)n_rows : (int64_t)batch * n_q_heads;
  int status = ORC_OK;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < total; ++r) {
    int32_t b = rows ? rows[2 * r] : (int32_t)(r / n_q_heads);
    int32_t h = rows ? rows[2 * r + 1] : (int32_t)(r % n_q_heads);
    int rc;
    if (b < 0 || b >= batch || h < 0 || h >= n_q_heads) {
      rc = ORC_EINVAL;
    } else {
      rc = decode_row_int8(q, dtype, cache, block_tables, max_blocks_per_seq, context_lens, num_blocks, scale,
                           n_q_heads, n_kv_heads, head_dim, block_size, b, h,
                           out + ((size_t)b * n_q_heads + h) * head_dim);
    }
    if (rc != ORC_OK) {
#pragma omp critical
      status = rc;
    }
  }
  return status;
}

/* Number of threads an OpenMP region would use (for reporting). */
int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
