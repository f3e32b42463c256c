/*
 * pa_oracle.c -- plain, slow, fp64 CPU oracle for the paged KV-cache decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker, not the product: only the
 * test suite, the smoke check and the CPU-baseline leg of the benchmark may load
 * it.  It shares no code, header, table or helper with the CUDA library under
 * paged_kv_cache_443_b200/; neither side includes or links the other.
 *
 * What it follows (sources are the three pages on vLLM / PagedAttention):
 *   - "자기회귀 생성과 KV 캐시" (supersilo.blog vLLM summary): the query of the
 *     current position attends to the keys of all valid past positions with
 *     scores q.k_j / sqrt(d_k), softmax-normalised over those positions, and the
 *     result is the score-weighted sum of the values.
 *   - "PagedAttention의 설계" (same page): K/V live in fixed-size blocks; a block
 *     table maps a sequence's logical blocks to physical blocks; the kernel reads
 *     K/V through that table in logical order and normalises the softmax over
 *     all valid tokens jointly (not per-block softmaxes added up).  The last
 *     block may hold unused slots, which carry no token.
 *   - "블록 공유" (same page) and "3. vLLM: KV cache를 블록 단위로 관리하기"
 *     (blog.aqudi.me): sequences may point at the same physical blocks; a block is
 *     copied only when one side must modify it (copy-on-write).
 *   - "1. KV 캐시란" (hjr-study-book Day 3): every decode step appends the new
 *     token's K and V to the cache.
 *
 * Nothing here is blocked, fused or reordered: attention rebuilds each
 * sequence's K and V contiguously from the block table, then evaluates the
 * softmax definition in two plain passes, in double precision.  Inputs are read
 * from their stored bit patterns (fp32 / fp16 / bf16) by the decoders below,
 * which do exponent/mantissa arithmetic, so the oracle sees exactly the values
 * the GPU sees.  OpenMP only spreads independent (sequence, head) rows over
 * threads; it does not change any row's arithmetic.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - grouped-query heads: query head h reads kv head floor(h / G), G = Hq / Hkv
 *     (contiguous groups);
 *   - cache layout [num_blocks][Hkv][block_size][D]; token j of a sequence sits in
 *     physical block block_tables[b][j / block_size] at offset j % block_size;
 *   - a sequence with context length 0 produces an all-zero output row;
 *   - copy-on-write pairs are applied in the given order;
 *   - a lower-precision KV cache ("quantization" in "4. 이 밖의 기법들",
 *     blog.aqudi.me, which names no format): 8-bit OCP E4M3 codes with one
 *     scale per cache (k_scale, v_scale); the stored code of x is
 *     E4M3(fp32(x) / fp32(scale)), the quotient rounded once in fp32, then to
 *     the nearest E4M3 value (ties to an even fraction), magnitudes above 448
 *     saturating to 448; a code stands for decode(code) * scale.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_F16 = 1, OR_BF16 = 2, OR_E4M3 = 3 };

/* ---- element decoders (IEEE 754 binary16 and bfloat16 by field arithmetic) ---- */

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double or_f16_to_f64(uint16_t bits) {
  int sign = (bits >> 15) & 1;
  int e = (bits >> 10) & 0x1f;
  int f = bits & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)f, -24); /* subnormal: f * 2^(1-15-10) */
  } else if (e == 31) {
    v = f ? NAN : INFINITY;
  } else {
    v = ldexp((double)(f + 1024), e - 25); /* (1 + f/2^10) * 2^(e-15) */
  }
  return sign ? -v : v;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double or_bf16_to_f64(uint16_t bits) {
  int sign = (bits >> 15) & 1;
  int e = (bits >> 7) & 0xff;
  int f = bits & 0x7f;
  double v;
  if (e == 0) {
    v = ldexp((double)f, -133); /* subnormal: f * 2^(1-127-7) */
  } else if (e == 255) {
    v = f ? NAN : INFINITY;
  } else {
    v = ldexp((double)(f + 128), e - 134); /* (1 + f/2^7) * 2^(e-127) */
  }
  return sign ? -v : v;
}

/* OCP 8-bit floating point, E4M3: 1 sign bit, 4 exponent bits (bias 7), 3
 * fraction bits; exponent field 0 is subnormal (f * 2^-9); there are no
 * infinities and S.1111.111 is NaN, so the largest finite value is
 * 1.75 * 2^8 = 448. */
double or_e4m3_to_f64(uint8_t bits) {
  int sign = (bits >> 7) & 1;
  int e = (bits >> 3) & 0xf;
  int f = bits & 0x7;
  double v;
  if (e == 15 && f == 7) {
    v = NAN;
  } else if (e == 0) {
    v = ldexp((double)f, -9); /* f/8 * 2^(1-7) */
  } else {
    v = ldexp((double)(f + 8), e - 10); /* (1 + f/8) * 2^(e-7) */
  }
  return sign ? -v : v;
}

/* Nearest E4M3 code to v (ties to an even fraction field), |v| > 448 and
 * infinities saturating to +-448, NaN to 0x7f.  Works on the exact value: the
 * spacing of E4M3 values around v is a power of two, so v / spacing is exact
 * in double and only the final rounding to an integer decides. */
uint8_t or_f64_to_e4m3(double v) {
  if (isnan(v)) return 0x7f;
  const uint8_t sign = signbit(v) ? 0x80 : 0x00;
  double a = fabs(v);
  if (a >= 448.0) return sign | 0x7e;
  int e; /* a = m * 2^e with m in [0.5, 1) */
  frexp(a, &e);
  int unbiased = e - 1; /* a in [2^unbiased, 2^(unbiased+1)) */
  if (a == 0.0 || unbiased < -6) unbiased = -6; /* subnormal range: spacing 2^-9 */
  const double spacing = ldexp(1.0, unbiased - 3);
  const double q = a / spacing; /* exact */
  double n = floor(q);
  const double rest = q - n;
  if (rest > 0.5 || (rest == 0.5 && fmod(n, 2.0) != 0.0)) n += 1.0;
  /* n counts spacings: in the normal range 8..16 (16 carries into the next
   * binade), in the subnormal range 0..8 (8 is the smallest normal) */
  const double r = n * spacing;
  if (r >= 448.0) return sign | 0x7e; /* cannot exceed: 448 is on the grid */
  if (r < ldexp(1.0, -6)) return sign | (uint8_t)n; /* subnormal code = fraction */
  int re;
  frexp(r, &re);
  const int be = re - 1 + 7; /* biased exponent */
  const int frac = (int)(ldexp(r, -(re - 1)) * 8.0) - 8;
  return sign | (uint8_t)((be << 3) | frac);
}

int or_elem_size(int dtype) {
  switch (dtype) {
    case OR_F32: return 4;
    case OR_F16: return 2;
    case OR_BF16: return 2;
    case OR_E4M3: return 1;
    default: return 0;
  }
}

/* Value of element idx of an array of the given storage type (an E4M3 code
 * without its scale). */
static double load_elem(const void* base, int dtype, size_t idx) {
  if (dtype == OR_E4M3) return or_e4m3_to_f64(((const uint8_t*)base)[idx]);
  if (dtype == OR_F32) {
    float x;
    memcpy(&x, (const char*)base + 4 * idx, 4);
    return (double)x;
  }
  uint16_t bits;
  memcpy(&bits, (const char*)base + 2 * idx, 2);
  return dtype == OR_F16 ? or_f16_to_f64(bits) : or_bf16_to_f64(bits);
}

/* Decode n elements (test helper: lets the tests pin the decoders directly). */
void or_decode(double* out, const void* src, int dtype, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = load_elem(src, dtype, (size_t)i);
}

/* Encode n values as E4M3 codes (test helper for the encoder pins). */
void or_encode_e4m3(uint8_t* out, const double* src, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = or_f64_to_e4m3(src[i]);
}

/* ---- attention over the paged cache ----
 * Follows the score and softmax definition of "자기회귀 생성과 KV 캐시" and the
 * block-table gather with one joint normaliser of "PagedAttention의 설계"
 * (supersilo.blog vLLM summary). */

/*
 * out[r][d] for each requested row r = (b, h) in rows[2r], rows[2r+1]; rows may
 * be NULL, meaning every (b, h) in order b-major (r = b * Hq + h).
 *
 * q:        [B][Hq][D]                     (dtype)
 * k_cache:  [num_blocks][Hkv][block_size][D] (dtype), v_cache the same
 * block_tables: [B][max_blocks] int32, context_lens: [B] int32
 *
 * Returns 0, or -1 if an input is out of range (a table entry outside
 * [0, num_blocks), a context length < 0 or beyond max_blocks * block_size, a
 * head count that does not divide, a row outside [0,B) x [0,Hq)).
 */
int or_paged_attention_kv(double* out, const int64_t* rows, int64_t nrows, const void* q,
                          const void* k_cache, const void* v_cache, int dtype, int kv_dtype,
                          double k_scale, double v_scale, const int32_t* block_tables,
                          int max_blocks, const int32_t* context_lens, int B, int Hq, int Hkv,
                          int D, int block_size, int num_blocks, double scale, int nthreads) {
  if (Hkv <= 0 || Hq % Hkv != 0 || or_elem_size(dtype) == 0 || or_elem_size(kv_dtype) == 0 ||
      dtype == OR_E4M3 || block_size <= 0 || D <= 0)
    return -1;
  const int G = Hq / Hkv;
  if (rows == NULL) nrows = (int64_t)B * Hq;
  int bad = 0;
  if (nthreads < 1) nthreads = 1;

#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1) reduction(| : bad)
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t b = rows ? rows[2 * r] : r / Hq;
    const int64_t h = rows ? rows[2 * r + 1] : r % Hq;
    double* o = out + r * D;
    if (b < 0 || b >= B || h < 0 || h >= Hq) {
      bad = 1;
      continue;
    }
    const int64_t g = h / G; /* kv head of this query head */
    const int64_t L = context_lens[b];
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (L < 0 || L > (int64_t)max_blocks * block_size) {
      bad = 1;
      continue;
    }
    if (L == 0) continue;

    /* 1. Rebuild this sequence's K and V contiguously, in logical order. */
    double* K = (double*)malloc(sizeof(double) * (size_t)L * D);
    double* V = (double*)malloc(sizeof(double) * (size_t)L * D);
    double* s = (double*)malloc(sizeof(double) * (size_t)L);
    int row_bad = 0;
    for (int64_t j = 0; j < L && !row_bad; ++j) {
      const int64_t phys = block_tables[b * max_blocks + j / block_size];
      const int64_t off = j % block_size;
      if (phys < 0 || phys >= num_blocks) {
        row_bad = 1;
        break;
      }
      const size_t base = (size_t)(((phys * Hkv + g) * block_size + off) * D);
      for (int d = 0; d < D; ++d) {
        K[j * D + d] = load_elem(k_cache, kv_dtype, base + d) * k_scale;
        V[j * D + d] = load_elem(v_cache, kv_dtype, base + d) * v_scale;
      }
    }
    if (!row_bad) {
      /* 2. Scores s_j = scale * q . K_j over the valid positions j < L. */
      const size_t qbase = (size_t)((b * Hq + h) * D);
      for (int64_t j = 0; j < L; ++j) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += load_elem(q, dtype, qbase + d) * K[j * D + d];
        s[j] = scale * acc;
      }
      /* 3. Softmax over all L positions at once (one normaliser for the whole
       *    sequence), then the weighted sum of V. */
      double mx = s[0];
      for (int64_t j = 1; j < L; ++j)
        if (s[j] > mx) mx = s[j];
      double Z = 0.0;
      for (int64_t j = 0; j < L; ++j) {
        s[j] = exp(s[j] - mx);
        Z += s[j];
      }
      for (int64_t j = 0; j < L; ++j) {
        const double w = s[j] / Z;
        for (int d = 0; d < D; ++d) o[d] += w * V[j * D + d];
      }
    } else {
      bad = 1;
    }
    free(K);
    free(V);
    free(s);
  }
  return bad ? -1 : 0;
}

/* The same with a cache of the query's own type and unit scales. */
int or_paged_attention(double* out, const int64_t* rows, int64_t nrows, const void* q,
                       const void* k_cache, const void* v_cache, int dtype,
                       const int32_t* block_tables, int max_blocks, const int32_t* context_lens,
                       int B, int Hq, int Hkv, int D, int block_size, int num_blocks,
                       double scale, int nthreads) {
  return or_paged_attention_kv(out, rows, nrows, q, k_cache, v_cache, dtype, dtype, 1.0, 1.0,
                               block_tables, max_blocks, context_lens, B, Hq, Hkv, D, block_size,
                               num_blocks, scale, nthreads);
}

/* ---- several new query tokens per sequence ----
 * Chunked prefill and speculative verification ("4. 이 밖의 기법들",
 * blog.aqudi.me: a long prefill cut into chunks between decode steps; several
 * proposed tokens checked by the large model at once).  The pages give no
 * formula beyond the attention of "자기회귀 생성과 KV 캐시" (supersilo.blog), so
 * the reading is: sequence b's last Q_b = query_start[b+1] - query_start[b]
 * context tokens are its new query tokens, and query token i (0 <= i < Q_b)
 * sits at position L_b - Q_b + i and attends to positions 0 .. L_b - Q_b + i
 * (its own included, none after it).
 *
 * q / out: [total_q][Hq][D] with total_q = query_start[B]; the cache, tables
 * and context lengths as above.  Each (query token, head) is the single-query
 * attention of or_paged_attention over its own number of positions.  Returns
 * -1 on an input out of range (query_start not non-decreasing from 0, Q_b >
 * L_b, and the cases of or_paged_attention).
 */
int or_paged_attention_mq(double* out, const void* q, const void* k_cache, const void* v_cache,
                          int dtype, const int32_t* block_tables, int max_blocks,
                          const int32_t* context_lens, const int32_t* query_start, int B, int Hq,
                          int Hkv, int D, int block_size, int num_blocks, double scale,
                          int nthreads) {
  if (B < 0 || Hq <= 0 || query_start[0] != 0) return -1;
  for (int b = 0; b < B; ++b)
    if (query_start[b + 1] < query_start[b] ||
        query_start[b + 1] - query_start[b] > context_lens[b])
      return -1;
  const int64_t total = query_start[B];
  const size_t es = (size_t)or_elem_size(dtype);
  if (es == 0) return -1;
  /* one row at a time through the single-query definition: a one-sequence
   * batch whose context ends at the query token's own position */
  int bad = 0;
  for (int b = 0; b < B && !bad; ++b) {
    const int Qb = query_start[b + 1] - query_start[b];
    for (int i = 0; i < Qb && !bad; ++i) {
      const int64_t t = query_start[b] + i;
      const int32_t len = context_lens[b] - Qb + i + 1;
      if (or_paged_attention(out + t * Hq * D, NULL, 0, (const char*)q + (size_t)t * Hq * D * es,
                             k_cache, v_cache, dtype, block_tables + (int64_t)b * max_blocks,
                             max_blocks, &len, 1, Hq, Hkv, D, block_size, num_blocks, scale,
                             nthreads) != 0)
        bad = 1;
    }
  }
  (void)total;
  return bad ? -1 : 0;
}

/* ---- appending the new tokens' K and V ----
 * Follows "1. KV 캐시란" (hjr-study-book Day 3: each step stores the new K, V
 * pair) and the slot arithmetic of the block-table example in "4.2
 * PagedAttention의 접근" (16-token blocks, logical block -> physical block). */

/*
 * For every t < N with slot = slot_mapping[t] >= 0:
 *   k_cache[slot / block_size][h][slot % block_size][:] = key[t][h][:]   (all h)
 *   v_cache[...]                                        = value[t][h][:]
 * A negative slot means "no token to store" and is skipped.  Elements are moved
 * as raw bytes.  Returns -1 (after writing nothing further) on a slot beyond the
 * cache.
 */
int or_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                         const int64_t* slot_mapping, int64_t N, int Hkv, int D, int block_size,
                         int64_t num_blocks, int dtype) {
  const size_t es = (size_t)or_elem_size(dtype);
  if (es == 0) return -1;
  for (int64_t t = 0; t < N; ++t) {
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= num_blocks * block_size) return -1;
    const int64_t blk = slot / block_size;
    const int64_t off = slot % block_size;
    for (int64_t h = 0; h < Hkv; ++h) {
      const size_t dst = (size_t)(((blk * Hkv + h) * block_size + off) * D) * es;
      const size_t src = (size_t)((t * Hkv + h) * D) * es;
      memcpy((char*)k_cache + dst, (const char*)key + src, (size_t)D * es);
      memcpy((char*)v_cache + dst, (const char*)value + src, (size_t)D * es);
    }
  }
  return 0;
}

/*
 * The append into an E4M3 cache: for every t < N with slot = slot_mapping[t] >= 0
 * and every h, d: k_cache[...][d] = E4M3(fp32(key[t][h][d]) / k_scale), the
 * quotient rounded once in fp32 (the cache reading in the header); value alike
 * with v_scale.  key/value are f32 / f16 / bf16 (dtype).  Returns -1 on a slot
 * beyond the cache or a bad dtype / scale.
 */
int or_reshape_and_cache_e4m3(const void* key, const void* value, uint8_t* k_cache,
                              uint8_t* v_cache, const int64_t* slot_mapping, int64_t N, int Hkv,
                              int D, int block_size, int64_t num_blocks, int dtype,
                              float k_scale, float v_scale) {
  if (or_elem_size(dtype) == 0 || dtype == OR_E4M3) return -1;
  if (!(k_scale > 0.0f) || !(v_scale > 0.0f) || isinf(k_scale) || isinf(v_scale)) return -1;
  for (int64_t t = 0; t < N; ++t) {
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= num_blocks * block_size) return -1;
    const int64_t blk = slot / block_size;
    const int64_t off = slot % block_size;
    for (int64_t h = 0; h < Hkv; ++h) {
      const size_t dst = (size_t)(((blk * Hkv + h) * block_size + off) * D);
      const size_t src = (size_t)((t * Hkv + h) * D);
      for (int d = 0; d < D; ++d) {
        const float kq = (float)load_elem(key, dtype, src + d) / k_scale;
        const float vq = (float)load_elem(value, dtype, src + d) / v_scale;
        k_cache[dst + d] = or_f64_to_e4m3((double)kq);
        v_cache[dst + d] = or_f64_to_e4m3((double)vq);
      }
    }
  }
  return 0;
}

/* ---- copy-on-write block copies ----
 * Follows "블록 공유" (supersilo.blog) and the copy-on-write bullet of "3. vLLM:
 * KV cache를 블록 단위로 관리하기" (blog.aqudi.me): a shared block is duplicated
 * before one of its sharers modifies it. */

/*
 * For each pair p in order: physical block pairs[2p+1] of both caches becomes a
 * copy of physical block pairs[2p] (all kv heads, all slots).  Returns -1 on an
 * id outside [0, num_blocks).
 */
int or_copy_blocks(void* k_cache, void* v_cache, const int64_t* pairs, int64_t P, int Hkv, int D,
                   int block_size, int64_t num_blocks, int dtype) {
  const size_t es = (size_t)or_elem_size(dtype);
  if (es == 0) return -1;
  const size_t block_bytes = (size_t)Hkv * block_size * D * es;
  for (int64_t p = 0; p < P; ++p) {
    const int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return -1;
    for (size_t i = 0; i < block_bytes; ++i) {
      ((char*)k_cache)[dst * block_bytes + i] = ((const char*)k_cache)[src * block_bytes + i];
      ((char*)v_cache)[dst * block_bytes + i] = ((const char*)v_cache)[src * block_bytes + i];
    }
  }
  return 0;
}

/* ---- swapping blocks between two caches ----
 * Follows "적용 범위와 관련 연구" (supersilo.blog): when GPU memory runs short, a
 * sequence's KV blocks move to CPU memory and come back later.  For each pair p
 * in order, block pairs[2p+1] of the destination caches becomes a byte copy of
 * block pairs[2p] of the source caches (all kv heads, all slots).  Returns -1 on
 * an id outside the source or destination pool. */
int or_swap_blocks(void* dst_k, void* dst_v, int64_t dst_num_blocks, const void* src_k,
                   const void* src_v, int64_t src_num_blocks, const int64_t* pairs, int64_t P,
                   int Hkv, int D, int block_size, int dtype) {
  const size_t es = (size_t)or_elem_size(dtype);
  if (es == 0) return -1;
  const size_t block_bytes = (size_t)Hkv * block_size * D * es;
  for (int64_t p = 0; p < P; ++p) {
    const int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
    if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) return -1;
    memcpy((char*)dst_k + dst * block_bytes, (const char*)src_k + src * block_bytes, block_bytes);
    memcpy((char*)dst_v + dst * block_bytes, (const char*)src_v + src * block_bytes, block_bytes);
  }
  return 0;
}

int or_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
