/*
 * Float64 CPU oracle for paged-attention decode, KV append and block copy.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls
 * this file: only the tests, the package's smoke check and the bench's CPU
 * baseline leg use it. It shares no code, header, table or constant with the
 * CUDA library; it is written directly from the pages that define the method:
 *
 *  [KVA] "KV cache" article, ainews.alishangtian.com, sections
 *        "生成一个字，为什么要背一整本账" (why a cache; KV-bytes formula),
 *        "显存账本" (GQA: several query heads share one KV head),
 *        "PagedAttention：把操作系统的老智慧搬进推理引擎" (fixed-size blocks,
 *        block table, shared prefix, copy-on-write),
 *        "再往后：压 KV 的三条路线" (FP8 KV with per-channel scaling factors).
 *  [PAX] "AI 陪读顶会论文（三）：KV Cache 显存占用计算与 PagedAttention 原理拆解",
 *        section "为什么自回归解码必须使用 KV Cache？" (decode attention equation;
 *        append the new k_t, v_t to the cache), section "PagedAttention 的破局哲学"
 *        (logical blocks -> physical blocks diagram; three innovations).
 *
 * Every routine is the plain definition: no blocking, no fusion, no online
 * softmax, no reordering. Floating point is float64 except where a reading
 * fixes a narrower type (the FP8 quantiser multiplies in fp32, once).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - cache layout [num_blocks][block_size][num_kv_heads][head_dim];
 *  - query head i reads KV head i / (Hq / Hkv) (contiguous groups);
 *  - FP8 is OCP E4M3 "FN" (bias 7, no infinities, S.1111.111 is NaN,
 *    largest finite 448), quantised as e4m3(fp32(x) * inv_scale) with
 *    round-to-nearest-even and saturation to +-448;
 *  - dequantised value = e4m3_value(byte) * scale[h][c];
 *  - a sequence with context length 0 produces an all-zero output row.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_F16 0
#define OR_BF16 1
#define OR_E4M3 2

#define OR_OK 0
#define OR_ERR_ARG 1
#define OR_ERR_BOUNDS 5

/* ---- scalar codecs, each from its format definition ---------------------- */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24); /* subnormal: m * 2^(1-15-10) */
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp(1.0 + (double)m / 1024.0, e - 15);
  return sign ? -v : v;
}

/* bfloat16: the upper half of an IEEE binary32: 8 exponent bits (bias 127),
 * 7 fraction bits. */
double oracle_bf16_to_double(uint16_t b) {
  int sign = (b >> 15) & 1;
  int e = (b >> 7) & 0xff;
  int m = b & 0x7f;
  double v;
  if (e == 0)
    v = ldexp((double)m, -133); /* subnormal: m * 2^(1-127-7) */
  else if (e == 255)
    v = m ? NAN : INFINITY;
  else
    v = ldexp(1.0 + (double)m / 128.0, e - 127);
  return sign ? -v : v;
}

/* OCP FP8 E4M3 ("FN" variant): 1 sign, 4 exponent bits (bias 7), 3 fraction
 * bits, no infinities; exponent 1111 with fraction 111 is NaN. */
double oracle_e4m3_to_double(uint8_t c) {
  int sign = (c >> 7) & 1;
  int e = (c >> 3) & 0xf;
  int m = c & 0x7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9); /* subnormal: m * 2^(1-7-3) */
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

/* Nearest E4M3 code to x, ties to the even fraction, magnitudes above the
 * largest finite value (448) saturate to it; NaN maps to S.1111.111. */
uint8_t oracle_e4m3_from_float(float xf) {
  double x = (double)xf;
  uint8_t s = signbit(x) ? 0x80 : 0x00;
  double a = fabs(x);
  if (isnan(x)) return (uint8_t)(s | 0x7f);
  if (a >= 448.0) return (uint8_t)(s | 0x7e); /* satfinite (inf included) */
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: spacing 2^-9; rint() rounds half to even */
    double r = rint(a / ldexp(1.0, -9));
    if (r >= 8.0) return (uint8_t)(s | 0x08); /* rounds up to 2^-6 */
    return (uint8_t)(s | (uint8_t)r);
  }
  int ex; /* a = f * 2^ex with f in [0.5, 1) */
  (void)frexp(a, &ex);
  int e = ex - 1;                        /* a in [2^e, 2^(e+1)), e in [-6, 8] */
  double r = rint(a / ldexp(1.0, e - 3)); /* significand * 8, in [8, 16] */
  if (r >= 16.0) {
    r = 8.0;
    e += 1;
  }
  int biased = e + 7;
  int frac = (int)r - 8;
  if (biased > 15 || (biased == 15 && frac == 7)) return (uint8_t)(s | 0x7e);
  return (uint8_t)(s | (uint8_t)(biased << 3) | (uint8_t)frac);
}

/* element of a 16-bit or 8-bit storage array, widened to double */
static double load_elem(const void* base, int64_t idx, int dtype) {
  if (dtype == OR_F16) return oracle_f16_to_double(((const uint16_t*)base)[idx]);
  if (dtype == OR_BF16) return oracle_bf16_to_double(((const uint16_t*)base)[idx]);
  return oracle_e4m3_to_double(((const uint8_t*)base)[idx]);
}

static int elem_bytes(int dtype) { return dtype == OR_E4M3 ? 1 : 2; }

/* ---- KV-bytes formula --------------------------------------------------- */

/* [KVA] section "生成一个字，为什么要背一整本账": bytes of a KV cache =
 * 2 (K and V) x layers x KV heads x head_dim x sequence length x batch x
 * bytes per element. */
int64_t oracle_kv_cache_bytes(int64_t layers, int64_t kv_heads, int64_t head_dim,
                              int64_t seq_len, int64_t batch, int64_t elem_bytes_) {
  return 2 * layers * kv_heads * head_dim * seq_len * batch * elem_bytes_;
}

/* ---- append ------------------------------------------------------------- */

/* [PAX] section "为什么自回归解码必须使用 KV Cache？": each step computes only
 * the new token's k_t, v_t and appends them to the cache; [KVA] section
 * "PagedAttention": the cache is made of fixed-size blocks, so token slot s
 * lives in block s / block_size at row s % block_size.
 *
 * k, v: [T][Hkv][D] in in_dtype (F16 or BF16). slot_mapping[t] < 0 skips
 * token t. A 16-bit cache must have the input's dtype and receives the bit
 * pattern unchanged; an E4M3 cache receives e4m3(fp32(x) * inv_scale[h][c]). */
int oracle_append_kv(const void* k, const void* v, int in_dtype, int64_t num_tokens,
                     const int64_t* slot_mapping, void* k_cache, void* v_cache,
                     int cache_dtype, int64_t num_blocks, int block_size, int num_kv_heads,
                     int head_dim, const float* k_inv_scale, const float* v_inv_scale) {
  if (in_dtype != OR_F16 && in_dtype != OR_BF16) return OR_ERR_ARG;
  if (cache_dtype != OR_E4M3 && cache_dtype != in_dtype) return OR_ERR_ARG;
  if (cache_dtype == OR_E4M3 && (!k_inv_scale || !v_inv_scale)) return OR_ERR_ARG;
  const int64_t row = (int64_t)num_kv_heads * head_dim;
  for (int64_t t = 0; t < num_tokens; ++t) {
    int64_t s = slot_mapping[t];
    if (s < 0) continue;
    if (s >= num_blocks * block_size) return OR_ERR_BOUNDS;
    int64_t blk = s / block_size, r = s % block_size;
    for (int h = 0; h < num_kv_heads; ++h) {
      for (int c = 0; c < head_dim; ++c) {
        int64_t src = t * row + (int64_t)h * head_dim + c;
        int64_t dst = ((blk * block_size + r) * num_kv_heads + h) * head_dim + c;
        if (cache_dtype == OR_E4M3) {
          float xk = (float)load_elem(k, src, in_dtype);
          float xv = (float)load_elem(v, src, in_dtype);
          float yk = xk * k_inv_scale[h * head_dim + c]; /* one fp32 multiply, RN */
          float yv = xv * v_inv_scale[h * head_dim + c];
          ((uint8_t*)k_cache)[dst] = oracle_e4m3_from_float(yk);
          ((uint8_t*)v_cache)[dst] = oracle_e4m3_from_float(yv);
        } else {
          ((uint16_t*)k_cache)[dst] = ((const uint16_t*)k)[src];
          ((uint16_t*)v_cache)[dst] = ((const uint16_t*)v)[src];
        }
      }
    }
  }
  return OR_OK;
}

/* ---- copy-on-write block copy ------------------------------------------- */

/* [KVA] section "PagedAttention" and [PAX] section "PagedAttention 的破局哲学"
 * (third innovation): branches share prompt blocks and a block is copied only
 * where the branches diverge. pairs[2p] is the source block, pairs[2p+1] the
 * destination; each copy moves the whole K block and the whole V block. */
int oracle_copy_blocks(const int32_t* pairs, int32_t num_pairs, void* k_cache, void* v_cache,
                       int cache_dtype, int64_t num_blocks, int block_size, int num_kv_heads,
                       int head_dim) {
  const int64_t block_bytes =
      (int64_t)block_size * num_kv_heads * head_dim * elem_bytes(cache_dtype);
  for (int32_t p = 0; p < num_pairs; ++p) {
    int64_t s = pairs[2 * p], d = pairs[2 * p + 1];
    if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) return OR_ERR_BOUNDS;
    memcpy((char*)k_cache + d * block_bytes, (const char*)k_cache + s * block_bytes,
           (size_t)block_bytes);
    memcpy((char*)v_cache + d * block_bytes, (const char*)v_cache + s * block_bytes,
           (size_t)block_bytes);
  }
  return OR_OK;
}

/* ---- decode attention ---------------------------------------------------- */

/* [PAX] section "为什么自回归解码必须使用 KV Cache？", attention equation: one
 * query q_t per sequence attends to all cached keys K_{1:t} (its own included):
 * o = softmax(q_t K^T / sqrt(d)) V. The caller passes the 1/sqrt(d) factor as
 * `scale` (fp32), used here widened to double.
 *
 * Step by step, for sequence b, query head i (KV head h = i / (Hq/Hkv)),
 * L = context_lens[b]:
 *  1. gather logical token j < L from physical block block_tables[b][j / BS],
 *     row j % BS ([KVA] "PagedAttention": a block table maps the logical
 *     blocks of a request to scattered physical blocks), into contiguous
 *     double arrays Kc[L][D], Vc[L][D]; E4M3 values are multiplied by the
 *     per-(kv_head, channel) scales;
 *  2. s_j = scale * sum_c q[c] * Kc[j][c];
 *  3. m = max_j s_j, w_j = exp(s_j - m) (subtracting m leaves the softmax
 *     unchanged), o = sum_j w_j Vc[j] / sum_j w_j.
 * Sliding window ([KVA] section "再往后：压 KV 的三条路线", second route: each
 * token attends only to the most recent window of tokens): with window > 0
 * the sums run over j in [max(0, L - window), L) -- the window counts the
 * new token itself -- and window == 0 means the whole history.
 * out: [B][Hq][D] doubles. */
int oracle_decode(const void* q, int q_dtype, int32_t batch, int32_t num_q_heads,
                  const void* k_cache, const void* v_cache, int cache_dtype, int64_t num_blocks,
                  int block_size, int num_kv_heads, int head_dim, const float* k_scale,
                  const float* v_scale, const int32_t* block_tables,
                  int32_t max_blocks_per_seq, const int32_t* context_lens, float scale,
                  int32_t window, double* out) {
  if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return OR_ERR_ARG;
  if (cache_dtype == OR_E4M3 && (!k_scale || !v_scale)) return OR_ERR_ARG;
  const int group = num_q_heads / num_kv_heads;
  const int D = head_dim;
  /* validate every table entry that will be read, before any work */
  for (int32_t b = 0; b < batch; ++b) {
    int32_t L = context_lens[b];
    if (L < 0) return OR_ERR_ARG;
    int64_t nblk = ((int64_t)L + block_size - 1) / block_size;
    if (nblk > max_blocks_per_seq) return OR_ERR_BOUNDS;
    for (int64_t n = 0; n < nblk; ++n) {
      int32_t blk = block_tables[(int64_t)b * max_blocks_per_seq + n];
      if (blk < 0 || blk >= num_blocks) return OR_ERR_BOUNDS;
    }
  }
  int err = OR_OK;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int32_t b = 0; b < batch; ++b) {
    for (int32_t i = 0; i < num_q_heads; ++i) {
      const int h = i / group;
      const int32_t L = context_lens[b];
      /* attended tokens: [j0, L), n of them */
      const int32_t j0 = (window > 0 && L > window) ? L - window : 0;
      const int32_t n = L - j0;
      double* o = out + ((int64_t)b * num_q_heads + i) * D;
      for (int c = 0; c < D; ++c) o[c] = 0.0;
      if (n == 0) continue;
      double* Kc = (double*)malloc(sizeof(double) * (size_t)n * D);
      double* Vc = (double*)malloc(sizeof(double) * (size_t)n * D);
      double* s = (double*)malloc(sizeof(double) * (size_t)n);
      double* qd = (double*)malloc(sizeof(double) * (size_t)D);
      if (!Kc || !Vc || !s || !qd) {
#pragma omp atomic write
        err = OR_ERR_ARG;
        free(Kc);
        free(Vc);
        free(s);
        free(qd);
        continue;
      }
      /* step 1: gather through the block table */
      for (int32_t k = 0; k < n; ++k) {
        const int32_t j = j0 + k;
        int64_t blk = block_tables[(int64_t)b * max_blocks_per_seq + j / block_size];
        int64_t r = j % block_size;
        int64_t base = ((blk * block_size + r) * num_kv_heads + h) * D;
        for (int c = 0; c < D; ++c) {
          double kv = load_elem(k_cache, base + c, cache_dtype);
          double vv = load_elem(v_cache, base + c, cache_dtype);
          if (cache_dtype == OR_E4M3) {
            kv *= (double)k_scale[h * D + c];
            vv *= (double)v_scale[h * D + c];
          }
          Kc[(int64_t)k * D + c] = kv;
          Vc[(int64_t)k * D + c] = vv;
        }
      }
      for (int c = 0; c < D; ++c)
        qd[c] = load_elem(q, ((int64_t)b * num_q_heads + i) * D + c, q_dtype);
      /* step 2: scores */
      for (int32_t k = 0; k < n; ++k) {
        double dot = 0.0;
        for (int c = 0; c < D; ++c) dot += qd[c] * Kc[(int64_t)k * D + c];
        s[k] = (double)scale * dot;
      }
      /* step 3: softmax-weighted sum of values */
      double m = s[0];
      for (int32_t k = 1; k < n; ++k)
        if (s[k] > m) m = s[k];
      double denom = 0.0;
      for (int32_t k = 0; k < n; ++k) {
        s[k] = exp(s[k] - m);
        denom += s[k];
      }
      for (int32_t k = 0; k < n; ++k)
        for (int c = 0; c < D; ++c) o[c] += s[k] * Vc[(int64_t)k * D + c];
      for (int c = 0; c < D; ++c) o[c] /= denom;
      free(Kc);
      free(Vc);
      free(s);
      free(qd);
    }
  }
  return err;
}

/* number of host threads the oracle's parallel loop uses */
int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
