/*
 * oracle.c — plain, slow, CPU fp64 reference of paged decode attention and of
 * the reshape_and_cache scatter.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may include, link or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline use it. It shares no code, header, table or constant with the CUDA
 * library; it reads the same raw host bytes the GPU is given.
 *
 * Sources (web pages, cited by title and section):
 *   [P1] "vLLM框架中的KV cache优化与PagedAttention机制详解" (trdm.cn)
 *   [P2] "vLLM推理引擎架构：PagedAttention机制与高吞吐推理" (maplevalley.com.cn)
 *   [P3] "Paged KVCache：大模型推理显存管理优化方案" (intelliparadigm.com)
 *   [P4] "大模型推理KV Cache内存管理与PagedAttention分页显存实战" (yunthe.com)
 *
 * Everything is written from the definitions: the number formats from the
 * IEEE 754 binary16 layout, the bfloat16 layout (top half of binary32) and
 * the OCP 8-bit floating point specification (E4M3: bias 7, no infinities,
 * S.1111.111 is NaN, max finite 448); the attention from softmax(scale q K^T) V.
 * No blocking, fusion or reordering: sums run in ascending index order.
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared oracle.c -o liborc.so -lm
 * (no fused multiply-add contraction, no fast-math: plain IEEE arithmetic).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_F16 = 0, ORC_BF16 = 1, ORC_E4M3 = 2 };

/* ---------------------------------------------------------------- formats */

/* binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double orc_decode_f16(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 0x1f, m = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24);                 /* subnormal: m * 2^-14 * 2^-10 */
  } else if (e == 31) {
    v = (m == 0) ? INFINITY : NAN;
  } else {
    v = ldexp((double)(1024 + m), e - 25);     /* (1 + m/2^10) * 2^(e-15) */
  }
  return s ? -v : v;
}

/* bfloat16: 1 sign, 8 exponent (bias 127), 7 fraction bits. */
double orc_decode_bf16(uint16_t b) {
  int s = (b >> 15) & 1, e = (b >> 7) & 0xff, m = b & 0x7f;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -133);                /* m * 2^-126 * 2^-7 */
  } else if (e == 255) {
    v = (m == 0) ? INFINITY : NAN;
  } else {
    v = ldexp((double)(128 + m), e - 134);     /* (1 + m/2^7) * 2^(e-127) */
  }
  return s ? -v : v;
}

/* OCP E4M3: 1 sign, 4 exponent (bias 7), 3 fraction bits; S.1111.111 is NaN. */
double orc_decode_e4m3(uint8_t c) {
  int s = (c >> 7) & 1, e = (c >> 3) & 0xf, m = c & 0x7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) {
    v = ldexp((double)m, -9);                  /* m/8 * 2^(1-7) */
  } else {
    v = ldexp((double)(8 + m), e - 10);        /* (1 + m/8) * 2^(e-7) */
  }
  return s ? -v : v;
}

/* Round a non-negative real q to the nearest integer, ties to even. */
static double round_half_even(double q) {
  double f = floor(q);
  double r = q - f;
  if (r > 0.5) return f + 1.0;
  if (r < 0.5) return f;
  return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/*
 * Nearest binary-format value with `mbits` fraction bits, exponent bias `bias`
 * and largest exponent field `emax_field` (finite); ties to even. Returns the
 * magnitude code (exponent field << mbits | fraction), or -1 on overflow.
 * `a` must be finite and >= 0.
 */
static long encode_magnitude(double a, int mbits, int bias, int emax_field) {
  int emin = 1 - bias;                         /* exponent of the smallest normal */
  if (a == 0.0) return 0;
  int e2;
  frexp(a, &e2);                               /* a = f * 2^e2, f in [0.5, 1) */
  int e = e2 - 1;                              /* a in [2^e, 2^(e+1)) */
  if (e < emin) {
    /* subnormal range: uniform quantum 2^(emin - mbits); code = multiple of it */
    double q = round_half_even(ldexp(a, mbits - emin));
    return (long)q;                            /* q == 2^mbits lands on the min normal */
  }
  double q = round_half_even(ldexp(a, mbits - e));  /* in [2^mbits, 2^(mbits+1)] */
  if (q == ldexp(1.0, mbits + 1)) {
    q = ldexp(1.0, mbits);
    e += 1;
  }
  long efield = e + bias;
  if (efield > emax_field) return -1;
  return (efield << mbits) | ((long)q - (1L << mbits));
}

/* fp32 -> E4M3, round to nearest even, saturating to +-448 (no infinities);
 * NaN -> 0x7F. */
uint8_t orc_encode_e4m3_rne_satfinite(float x) {
  if (isnan(x)) return 0x7f;
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs((double)x);
  if (a >= 448.0) return sign | 0x7e;          /* satfinite: |x| >= max finite -> max finite */
  long code = encode_magnitude(a, 3, 7, 15);
  if (code < 0 || code > 0x7e) code = 0x7e;    /* 480 would be the NaN code: saturate */
  return (uint8_t)(sign | code);
}

/* double -> binary16, round to nearest even, overflow to infinity. */
uint16_t orc_encode_f16(double x) {
  if (isnan(x)) return 0x7e00;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (isinf(a)) return sign | 0x7c00;
  long code = encode_magnitude(a, 10, 15, 30);
  if (code < 0) return sign | 0x7c00;
  return (uint16_t)(sign | code);
}

/* double -> bfloat16, round to nearest even, overflow to infinity. */
uint16_t orc_encode_bf16(double x) {
  if (isnan(x)) return 0x7fc0;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (isinf(a)) return sign | 0x7f80;
  long code = encode_magnitude(a, 7, 127, 254);
  if (code < 0) return sign | 0x7f80;
  return (uint16_t)(sign | code);
}

/* One IEEE binary32 division (the FP8 quantiser divides by the scale in fp32). */
float orc_div_f32(float a, float b) {
  volatile float q = a / b;
  return q;
}

static double load_elem(const void* base, size_t idx, int dt) {
  if (dt == ORC_E4M3) return orc_decode_e4m3(((const uint8_t*)base)[idx]);
  uint16_t v = ((const uint16_t*)base)[idx];
  return dt == ORC_F16 ? orc_decode_f16(v) : orc_decode_bf16(v);
}

/* ------------------------------------------------------------ addressing */

/*
 * Address translation of [P3] §2.3 "地址转换流程" with the page size counted in
 * tokens ([P4]: a block holds 16 tokens): the logical position `pos` of
 * sequence `seq` lives in logical block pos / block_size at offset
 * pos % block_size; the block table maps the logical block to a physical one,
 * and the physical slot is physical_block * block_size + offset.
 * pos < 0 -> -1. Returns 0, or -1 if a table entry is missing/negative.
 */
int orc_slot_mapping(const int32_t* block_tables, int32_t num_seqs, int32_t max_blocks_per_seq,
                     const int32_t* seq_ids, const int32_t* positions, int32_t num_tokens,
                     int32_t block_size, int32_t* slots_out) {
  for (int32_t i = 0; i < num_tokens; ++i) {
    int32_t seq = seq_ids ? seq_ids[i] : i;
    int32_t pos = positions[i];
    if (pos < 0) { slots_out[i] = -1; continue; }
    if (seq < 0 || seq >= num_seqs) return -1;
    int32_t logical_block = pos / block_size;
    int32_t offset = pos % block_size;
    if (logical_block >= max_blocks_per_seq) return -1;
    int64_t physical_block = block_tables[(int64_t)seq * max_blocks_per_seq + logical_block];
    if (physical_block < 0) return -1;
    int64_t slot = physical_block * block_size + offset;
    if (slot > INT32_MAX) return -1;
    slots_out[i] = (int32_t)slot;
  }
  return 0;
}

/* --------------------------------------------------------- reshape_and_cache */

/*
 * Write token n's K/V rows ([num_tokens, num_kv_heads, head_dim]) into the
 * cache ([num_blocks, block_size, num_kv_heads, head_dim], the layout of [P2]
 * §2.2) at slot_mapping[n]; negative slots are skipped. Same dtype: the bytes
 * are copied. FP8 cache ([P4] "FP8 KV Cache量化", 16 -> 8 bit): the element is
 * decoded to fp32, divided by the head's fp32 scale in fp32, and rounded once
 * to E4M3 (nearest even, saturating).
 * Returns 0; -1 on a slot outside the pool, -2 on duplicate slots,
 * -3 on an unsupported dtype pair.
 */
int orc_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                          const int32_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
                          int32_t head_dim, int32_t block_size, int64_t num_blocks,
                          int kv_dtype, int cache_dtype, const float* k_scale,
                          const float* v_scale) {
  if (kv_dtype == ORC_E4M3) return -3;
  if (cache_dtype != kv_dtype && cache_dtype != ORC_E4M3) return -3;
  int64_t pool_slots = num_blocks * block_size;
  /* Slots are physical addresses: two tokens may not share one. */
  for (int32_t n = 0; n < num_tokens; ++n) {
    if (slot_mapping[n] < 0) continue;
    if (slot_mapping[n] >= pool_slots) return -1;
    for (int32_t m = 0; m < n; ++m)
      if (slot_mapping[m] == slot_mapping[n]) return -2;
  }
  size_t row = (size_t)num_kv_heads * head_dim;
  for (int32_t n = 0; n < num_tokens; ++n) {
    int64_t slot = slot_mapping[n];
    if (slot < 0) continue;
    int64_t blk = slot / block_size;
    int64_t off = slot % block_size;
    for (int32_t h = 0; h < num_kv_heads; ++h) {
      for (int32_t d = 0; d < head_dim; ++d) {
        size_t src = (size_t)n * row + (size_t)h * head_dim + d;
        size_t dst = (((size_t)blk * block_size + off) * num_kv_heads + h) * head_dim + d;
        if (cache_dtype == kv_dtype) {
          ((uint16_t*)key_cache)[dst] = ((const uint16_t*)key)[src];
          ((uint16_t*)value_cache)[dst] = ((const uint16_t*)value)[src];
        } else {
          float kx = (float)load_elem(key, src, kv_dtype);   /* exact: 16-bit -> fp32 */
          float vx = (float)load_elem(value, src, kv_dtype);
          ((uint8_t*)key_cache)[dst] = orc_encode_e4m3_rne_satfinite(orc_div_f32(kx, k_scale[h]));
          ((uint8_t*)value_cache)[dst] = orc_encode_e4m3_rne_satfinite(orc_div_f32(vx, v_scale[h]));
        }
      }
    }
  }
  return 0;
}

/* ------------------------------------------------------------------ decode */

/*
 * Step 1 (logical -> physical translation, [P1] §5.1; [P3] §2.3): copy the
 * first n tokens of sequence s, kv-head kvh, out of the block pool into a
 * contiguous fp64 matrix dst[n][head_dim], dequantising FP8 codes with the
 * head's scale. Returns -1 on a table entry outside [0, num_blocks).
 */
static int gather_sequence(const void* cache, int dt, double scale_kvh, const int32_t* table_row,
                           int32_t n, int32_t kvh, int32_t num_kv_heads, int32_t head_dim,
                           int32_t block_size, int64_t num_blocks, double* dst) {
  for (int32_t t = 0; t < n; ++t) {
    int64_t blk = table_row[t / block_size];
    int64_t off = t % block_size;
    if (blk < 0 || blk >= num_blocks) return -1;
    for (int32_t d = 0; d < head_dim; ++d) {
      size_t idx = ((size_t)(blk * block_size + off) * num_kv_heads + kvh) * head_dim + d;
      dst[(size_t)t * head_dim + d] = load_elem(cache, idx, dt) * scale_kvh;
    }
  }
  return 0;
}

/*
 * Textbook attention of one query row over contiguous K, V (n x head_dim):
 * s_t = scale * q.K[t]; m = max_t s_t; p_t = exp(s_t - m);
 * out = sum_t p_t V[t] / sum_t p_t. n == 0 -> zeros. Tokens in [t0, t1) only;
 * returns (m, l = sum p_t) for the partition combine below.
 */
static void attend_rows(const double* q, const double* K, const double* V, int32_t t0, int32_t t1,
                        int32_t head_dim, double scale, double* out, double* m_out,
                        double* l_out) {
  for (int32_t d = 0; d < head_dim; ++d) out[d] = 0.0;
  if (t1 <= t0) { *m_out = -INFINITY; *l_out = 0.0; return; }
  int32_t n = t1 - t0;
  double* s = (double*)malloc(sizeof(double) * (size_t)n);
  double m = -INFINITY;
  for (int32_t t = t0; t < t1; ++t) {
    double dot = 0.0;
    for (int32_t d = 0; d < head_dim; ++d) dot += q[d] * K[(size_t)t * head_dim + d];
    s[t - t0] = scale * dot;
    if (s[t - t0] > m) m = s[t - t0];
  }
  double l = 0.0;
  for (int32_t t = t0; t < t1; ++t) {
    double p = exp(s[t - t0] - m);
    l += p;
    for (int32_t d = 0; d < head_dim; ++d) out[d] += p * V[(size_t)t * head_dim + d];
  }
  for (int32_t d = 0; d < head_dim; ++d) out[d] /= l;
  free(s);
  *m_out = m;
  *l_out = l;
}

/*
 * Paged decode ([P2] §2.3 "PagedAttention Kernel", interface
 * (output, query, key_cache, value_cache, block_tables, context_lens, block_size)):
 * out[s][h][:] = attention of query[s][h] over the context_lens[s] tokens of
 * sequence s, found through block_tables. Query head h reads kv-head
 * h / (num_heads / num_kv_heads). out is fp64 [num_seqs, num_heads, head_dim].
 *
 * partition_tokens <= 0: one pass over the whole context (the definition).
 * partition_tokens > 0: the context is cut into partitions of that many tokens,
 * each attended separately giving (m_p, l_p, o_p), then combined as
 * M = max m_p, w_p = l_p e^(m_p - M), out = sum_p w_p o_p / sum_p w_p — an
 * algebraic identity with the one-pass result (used to pin that identity).
 * Returns 0; -1 on a bad table entry; -2 on bad sizes.
 */
int orc_decode(double* out, const void* query, const void* key_cache, const void* value_cache,
               const int32_t* block_tables, int32_t max_blocks_per_seq,
               const int32_t* context_lens, int32_t num_seqs, int32_t num_heads,
               int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int64_t num_blocks,
               float scale, int q_dtype, int cache_dtype, const float* k_scale,
               const float* v_scale, int32_t partition_tokens) {
  if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0)
    return -2;
  int32_t group = num_heads / num_kv_heads;
  for (int32_t s = 0; s < num_seqs; ++s) {
    int32_t n = context_lens[s];
    if (n < 0 || (n + block_size - 1) / block_size > max_blocks_per_seq) return -2;
    const int32_t* row = block_tables + (size_t)s * max_blocks_per_seq;
    double* K = (double*)malloc(sizeof(double) * ((size_t)n * head_dim + 1));
    double* V = (double*)malloc(sizeof(double) * ((size_t)n * head_dim + 1));
    double* q = (double*)malloc(sizeof(double) * (size_t)head_dim);
    int rc = 0;
    for (int32_t kvh = 0; kvh < num_kv_heads && rc == 0; ++kvh) {
      double ks = (cache_dtype == ORC_E4M3) ? (double)k_scale[kvh] : 1.0;
      double vs = (cache_dtype == ORC_E4M3) ? (double)v_scale[kvh] : 1.0;
      rc = gather_sequence(key_cache, cache_dtype, ks, row, n, kvh, num_kv_heads, head_dim,
                           block_size, num_blocks, K);
      if (rc == 0)
        rc = gather_sequence(value_cache, cache_dtype, vs, row, n, kvh, num_kv_heads, head_dim,
                             block_size, num_blocks, V);
      if (rc != 0) break;
      for (int32_t j = 0; j < group; ++j) {
        int32_t h = kvh * group + j;
        size_t qoff = ((size_t)s * num_heads + h) * head_dim;
        for (int32_t d = 0; d < head_dim; ++d) q[d] = load_elem(query, qoff + d, q_dtype);
        double* o = out + qoff;
        double m, l;
        if (partition_tokens <= 0 || n <= partition_tokens) {
          attend_rows(q, K, V, 0, n, head_dim, (double)scale, o, &m, &l);
          continue;
        }
        /* partitioned: combine (m_p, l_p, o_p) */
        int32_t np = (n + partition_tokens - 1) / partition_tokens;
        double M = -INFINITY;
        double* mp = (double*)malloc(sizeof(double) * (size_t)np);
        double* lp = (double*)malloc(sizeof(double) * (size_t)np);
        double* op = (double*)malloc(sizeof(double) * (size_t)np * head_dim);
        for (int32_t p = 0; p < np; ++p) {
          int32_t t0 = p * partition_tokens;
          int32_t t1 = t0 + partition_tokens < n ? t0 + partition_tokens : n;
          attend_rows(q, K, V, t0, t1, head_dim, (double)scale, op + (size_t)p * head_dim,
                      &mp[p], &lp[p]);
          if (mp[p] > M) M = mp[p];
        }
        double L = 0.0;
        for (int32_t p = 0; p < np; ++p) L += lp[p] * exp(mp[p] - M);
        for (int32_t d = 0; d < head_dim; ++d) {
          double acc = 0.0;
          for (int32_t p = 0; p < np; ++p)
            acc += lp[p] * exp(mp[p] - M) * op[(size_t)p * head_dim + d];
          o[d] = acc / L;
        }
        free(mp); free(lp); free(op);
      }
    }
    free(K); free(V); free(q);
    if (rc != 0) return rc;
  }
  return 0;
}

/*
 * Multi-token query over the paged cache (chunked prefill, verification of
 * several draft tokens). [P2] §2.3's interface takes a query tensor; here it
 * has more rows than sequences: the q_len_s = cu_q[s+1] - cu_q[s] rows
 * query[cu_q[s] ..] are the last q_len_s positions of sequence s,
 * p_i = context_lens[s] - q_len_s + i, whose keys and values are already in
 * the cache. Row i attends to the tokens t <= p_i of its sequence (the
 * causal rule of autoregressive attention: a token sees itself and its
 * past), through block_tables as in orc_decode. out is fp64
 * [num_tokens, num_heads, head_dim]. Returns 0; -1 on a bad table entry;
 * -2 on bad sizes; -3 when q_len_s > context_lens[s].
 */
int orc_chunked_prefill(double* out, const void* query, const int32_t* cu_q, int32_t num_tokens,
                        const void* key_cache, const void* value_cache,
                        const int32_t* block_tables, int32_t max_blocks_per_seq,
                        const int32_t* context_lens, int32_t num_seqs, int32_t num_heads,
                        int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                        int64_t num_blocks, float scale, int q_dtype, int cache_dtype,
                        const float* k_scale, const float* v_scale) {
  if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0 ||
      cu_q[0] != 0 || cu_q[num_seqs] != num_tokens)
    return -2;
  int32_t group = num_heads / num_kv_heads;
  for (int32_t s = 0; s < num_seqs; ++s) {
    int32_t n = context_lens[s];
    int32_t qlen = cu_q[s + 1] - cu_q[s];
    if (n < 0 || qlen < 0 || (n + block_size - 1) / block_size > max_blocks_per_seq) return -2;
    if (qlen > n) return -3;
    const int32_t* row = block_tables + (size_t)s * max_blocks_per_seq;
    double* K = (double*)malloc(sizeof(double) * ((size_t)n * head_dim + 1));
    double* V = (double*)malloc(sizeof(double) * ((size_t)n * head_dim + 1));
    double* q = (double*)malloc(sizeof(double) * (size_t)head_dim);
    int rc = 0;
    for (int32_t kvh = 0; kvh < num_kv_heads && rc == 0; ++kvh) {
      double ks = (cache_dtype == ORC_E4M3) ? (double)k_scale[kvh] : 1.0;
      double vs = (cache_dtype == ORC_E4M3) ? (double)v_scale[kvh] : 1.0;
      rc = gather_sequence(key_cache, cache_dtype, ks, row, n, kvh, num_kv_heads, head_dim,
                           block_size, num_blocks, K);
      if (rc == 0)
        rc = gather_sequence(value_cache, cache_dtype, vs, row, n, kvh, num_kv_heads, head_dim,
                             block_size, num_blocks, V);
      if (rc != 0) break;
      for (int32_t i = 0; i < qlen; ++i) {
        int32_t pos = n - qlen + i;
        for (int32_t j = 0; j < group; ++j) {
          int32_t h = kvh * group + j;
          size_t qoff = ((size_t)(cu_q[s] + i) * num_heads + h) * head_dim;
          for (int32_t d = 0; d < head_dim; ++d) q[d] = load_elem(query, qoff + d, q_dtype);
          double m, l;
          attend_rows(q, K, V, 0, pos + 1, head_dim, (double)scale, out + qoff, &m, &l);
        }
      }
    }
    free(K); free(V); free(q);
    if (rc != 0) return rc;
  }
  return 0;
}
