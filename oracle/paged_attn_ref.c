/*
 * Oracle for paged decode attention — TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may load
 * this file's library. It shares no code with the CUDA path.
 *
 * What it computes: Eq. 1 of "KV-Cache Optimization Techniques", section
 * "PagedAttention (vLLM)": for one query token, attention is the softmax of
 * q times the concatenation of the key pages (transposed) over sqrt(d_k),
 * applied to the concatenation of the value pages. The pages that make up a
 * sequence are found through its page table (same section, "Architecture":
 * a per-request table maps logical KV positions to physical pages of P tokens).
 *
 * The oracle writes this definition out with no blocking or reordering:
 *   1. gather K_c[t] and V_c[t] for t < ctx from pool[table[t / P]][h][t % P]
 *      into contiguous fp64 arrays (bf16 widened exactly; INT8 rows dequantised
 *      in fp64 as s*code + z, the right-hand side of Eq. 3 in section
 *      "KV-Cache Quantization");
 *   2. s_t = scale * (q . K_c[t]) in fp64;
 *   3. textbook two-pass softmax: m = max s, e_t = exp(s_t - m), l = sum e_t;
 *   4. out = sum_t (e_t / l) V_c[t];  lse = m + log(l).
 * Query head hq reads KV head hq / G with G = Hq / Hkv (section "Multi-Query
 * and Grouped-Query Caching", Eq. 7: groups of query heads share one K/V).
 * An empty token range gives out = 0 and lse = -inf.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_BAD_ARG 1
#define ORC_BAD_TABLE 5

static double bf16_bits_to_f64(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

double oracle_e4m3_value(uint8_t c); /* quant_ref.c: E4M3 code -> value */

/* One element of a cached row, widened to fp64.  kind 0: bf16 bits;
 * kind 1: uint8 code with the row's fp32 (scale, zero), value s*code + z;
 * kind 2: E4M3 code with the row's fp32 scale, value s*E4M3(code);
 * kind 3: 4-bit code (two per byte, element 2i in the low nibble of byte i)
 *         with the row's fp32 (scale, zero), value s*code + z. */
static double kv_elem(int kind, const void *pool, const float *sz, int64_t row,
                      int d, int j) {
  if (kind == 0) {
    const uint16_t *p = (const uint16_t *)pool;
    return bf16_bits_to_f64(p[row * d + j]);
  }
  const uint8_t *p = (const uint8_t *)pool;
  const double s = (double)sz[2 * row + 0];
  const double z = (double)sz[2 * row + 1];
  if (kind == 1) return s * (double)p[row * d + j] + z;
  if (kind == 2) return s * oracle_e4m3_value(p[row * d + j]) + z;
  const uint8_t byte = p[row * (d / 2) + j / 2];
  const int code = (j % 2 == 0) ? (byte & 15) : (byte >> 4);
  return s * (double)code + z;
}

/*
 * Attention for a list of (sequence, query head) pairs over the token range
 * [t_begin, t_end) of each sequence (t_end < 0 means "up to ctx").
 *
 * k_pool, v_pool: [num_pages][hkv][page_size][d], bf16 bits or uint8 codes.
 * k_sz, v_sz:     [num_pages][hkv][page_size][2] fp32 (scale, zero); INT8 only.
 * q:              [B][hq][d] bf16 bits.
 * block_tables:   [B][max_pages] int32; ctx: [B] int32.
 * pairs:          [n_pairs][2] (b, hq); NULL means every (b, hq) in order.
 * out:            [n_pairs][d] fp64;  lse: [n_pairs] fp64 (may be NULL).
 * Returns ORC_BAD_TABLE if a page the range needs is outside the pool.
 */
int oracle_paged_attention(int kind, const void *k_pool, const void *v_pool,
                           const float *k_sz, const float *v_sz, int num_pages,
                           int page_size, int hkv, int d, const uint16_t *q,
                           int B, int hq, const int32_t *block_tables,
                           int max_pages, const int32_t *ctx, double scale,
                           int t_begin, int t_end, const int32_t *pairs,
                           int n_pairs, double *out, double *lse) {
  if (hkv <= 0 || hq % hkv != 0 || d <= 0 || page_size <= 0 || B < 0)
    return ORC_BAD_ARG;
  if (kind != 0 && (k_sz == NULL || v_sz == NULL)) return ORC_BAD_ARG;
  const int G = hq / hkv;
  const int n_items = pairs ? n_pairs : B * hq;
  int status = ORC_OK;

#pragma omp parallel for schedule(dynamic, 1)
  for (int it = 0; it < n_items; ++it) {
    const int b = pairs ? pairs[2 * it] : it / hq;
    const int qh = pairs ? pairs[2 * it + 1] : it % hq;
    const int h = qh / G;
    int t0 = t_begin < 0 ? 0 : t_begin;
    int t1 = (t_end < 0 || t_end > ctx[b]) ? ctx[b] : t_end;
    if (t1 < t0) t1 = t0;
    const int n = t1 - t0;
    double *o = out + (int64_t)it * d;
    for (int j = 0; j < d; ++j) o[j] = 0.0;
    if (lse) lse[it] = -INFINITY;
    if (n == 0) continue;

    /* 1. gather the pages of this sequence into contiguous K_c, V_c */
    double *Kc = (double *)malloc(sizeof(double) * (size_t)n * d);
    double *Vc = (double *)malloc(sizeof(double) * (size_t)n * d);
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    int bad = 0;
    for (int i = 0; i < n && !bad; ++i) {
      const int t = t0 + i;
      const int lp = t / page_size;
      if (lp >= max_pages) { bad = 1; break; }
      const int32_t page = block_tables[(int64_t)b * max_pages + lp];
      if (page < 0 || page >= num_pages) { bad = 1; break; }
      const int64_t row = ((int64_t)page * hkv + h) * page_size + t % page_size;
      for (int j = 0; j < d; ++j) {
        Kc[(int64_t)i * d + j] = kv_elem(kind, k_pool, k_sz, row, d, j);
        Vc[(int64_t)i * d + j] = kv_elem(kind, v_pool, v_sz, row, d, j);
      }
    }
    if (bad) {
#pragma omp atomic write
      status = ORC_BAD_TABLE;
      free(Kc); free(Vc); free(s);
      continue;
    }

    /* 2. scores */
    const uint16_t *qv = q + ((int64_t)b * hq + qh) * d;
    for (int i = 0; i < n; ++i) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j) acc += bf16_bits_to_f64(qv[j]) * Kc[(int64_t)i * d + j];
      s[i] = scale * acc;
    }
    /* 3. two-pass softmax */
    double m = s[0];
    for (int i = 1; i < n; ++i) if (s[i] > m) m = s[i];
    double l = 0.0;
    for (int i = 0; i < n; ++i) { s[i] = exp(s[i] - m); l += s[i]; }
    /* 4. weighted sum of V */
    for (int i = 0; i < n; ++i) {
      const double w = s[i] / l;
      for (int j = 0; j < d; ++j) o[j] += w * Vc[(int64_t)i * d + j];
    }
    if (lse) lse[it] = m + log(l);
    free(Kc); free(Vc); free(s);
  }
  return status;
}

/*
 * Eq. 5 and Eq. 6 of "KV-Cache Optimization Techniques" (sections "Token
 * Eviction Strategies", StreamingLLM, and "Sliding Window Cache"): attention
 * over the cached token set {first `sinks` tokens} U {last `window` tokens}
 * of each sequence (window = 0 means no window: the whole context; sinks = 0
 * is the plain sliding window of Eq. 6). The set is gathered in increasing
 * token order, each token once, then the same textbook softmax as above.
 * pairs/out/lse as for oracle_paged_attention.
 */
int oracle_paged_attention_window(int kind, const void *k_pool, const void *v_pool,
                                  const float *k_sz, const float *v_sz, int num_pages,
                                  int page_size, int hkv, int d, const uint16_t *q, int B,
                                  int hq, const int32_t *block_tables, int max_pages,
                                  const int32_t *ctx, double scale, int sinks, int window,
                                  const int32_t *pairs, int n_pairs, double *out,
                                  double *lse) {
  if (hkv <= 0 || hq % hkv != 0 || d <= 0 || page_size <= 0 || B < 0 || sinks < 0 ||
      window < 0)
    return ORC_BAD_ARG;
  if (kind != 0 && (k_sz == NULL || v_sz == NULL)) return ORC_BAD_ARG;
  const int G = hq / hkv;
  const int n_items = pairs ? n_pairs : B * hq;
  int status = ORC_OK;

#pragma omp parallel for schedule(dynamic, 1)
  for (int it = 0; it < n_items; ++it) {
    const int b = pairs ? pairs[2 * it] : it / hq;
    const int qh = pairs ? pairs[2 * it + 1] : it % hq;
    const int h = qh / G;
    const int n_ctx = ctx[b];
    double *o = out + (int64_t)it * d;
    for (int j = 0; j < d; ++j) o[j] = 0.0;
    if (lse) lse[it] = -INFINITY;
    /* the token set, in increasing order */
    int *tok = (int *)malloc(sizeof(int) * (size_t)(n_ctx > 0 ? n_ctx : 1));
    int n = 0;
    for (int t = 0; t < n_ctx; ++t) {
      const int in_sinks = t < sinks;
      const int in_window = window == 0 || t >= n_ctx - window;
      if (in_sinks || in_window) tok[n++] = t;
    }
    if (n == 0) { free(tok); continue; }
    double *Kc = (double *)malloc(sizeof(double) * (size_t)n * d);
    double *Vc = (double *)malloc(sizeof(double) * (size_t)n * d);
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    int bad = 0;
    for (int i = 0; i < n && !bad; ++i) {
      const int t = tok[i];
      const int lp = t / page_size;
      if (lp >= max_pages) { bad = 1; break; }
      const int32_t page = block_tables[(int64_t)b * max_pages + lp];
      if (page < 0 || page >= num_pages) { bad = 1; break; }
      const int64_t row = ((int64_t)page * hkv + h) * page_size + t % page_size;
      for (int j = 0; j < d; ++j) {
        Kc[(int64_t)i * d + j] = kv_elem(kind, k_pool, k_sz, row, d, j);
        Vc[(int64_t)i * d + j] = kv_elem(kind, v_pool, v_sz, row, d, j);
      }
    }
    if (!bad) {
      const uint16_t *qv = q + ((int64_t)b * hq + qh) * d;
      for (int i = 0; i < n; ++i) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += bf16_bits_to_f64(qv[j]) * Kc[(int64_t)i * d + j];
        s[i] = scale * acc;
      }
      double m = s[0];
      for (int i = 1; i < n; ++i) if (s[i] > m) m = s[i];
      double l = 0.0;
      for (int i = 0; i < n; ++i) { s[i] = exp(s[i] - m); l += s[i]; }
      for (int i = 0; i < n; ++i) {
        const double w = s[i] / l;
        for (int j = 0; j < d; ++j) o[j] += w * Vc[(int64_t)i * d + j];
      }
      if (lse) lse[it] = m + log(l);
    } else {
#pragma omp atomic write
      status = ORC_BAD_TABLE;
    }
    free(Kc); free(Vc); free(s); free(tok);
  }
  return status;
}
