/*
 * gqa_oracle.c -- plain fp64 CPU oracle for masked grouped-query attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header, table or helper with
 * the CUDA library.
 *
 * What it computes (one query row at a time, straight from the definition):
 *
 *   "TPU v6e Masked GQA Kernel Optimization", sections "What You Have" and
 *   "What You Submit": attention over bf16 q (batch, num_q_heads, q_len,
 *   head_dim) and k, v (batch, num_kv_heads, kv_len, head_dim), GQA ratios
 *   1:1 to 16:1, optional causal mask, optional sliding window, optional
 *   logit softcap; output has q's shape.  "How It Is Judged": correctness is
 *   measured against an fp32 reference -- this oracle is fp64, so stricter.
 *
 *   "Independent attention product layouts", flowchart: scores QK, a softmax
 *   over the complete row, then PV and a final normalisation.
 *
 * Readings where the pages are silent (each one is a documented choice):
 *   - query row i sits at position qpos = kv_len - q_len + i (bottom-right
 *     alignment of causal and window masks);
 *   - key j is visible iff j < kv_len and (!causal or j <= qpos) and
 *     (window <= 0 or 0 <= qpos - j < window);
 *   - query head h reads kv head h / (num_q_heads / num_kv_heads);
 *   - logit x = (q.k) / sqrt(head_dim) with the logical head_dim, then, if
 *     softcap > 0, x = softcap * tanh(x / softcap); masking is applied to
 *     the capped logits (a masked key simply takes no part in the row);
 *   - a row with no visible key returns zeros.
 *
 * Arithmetic: every input element is widened exactly to double (bf16 inputs
 * by placing their 16 bits on top of a float), all sums, exp and tanh are
 * fp64 (host libm), and the result is returned unrounded in fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Element formats the oracle accepts. */
#define ORACLE_F64 0  /* IEEE double */
#define ORACLE_BF16 1 /* raw bfloat16 bits (uint16) */

/* Read element idx of an array in the given format, widened exactly. */
static double load_elem(const void *base, int64_t idx, int fmt) {
  if (fmt == ORACLE_BF16) {
    uint32_t bits = (uint32_t)((const uint16_t *)base)[idx] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  return ((const double *)base)[idx];
}

/* Is key j visible from the query at position qpos? */
static int key_visible(long j, long qpos, int kv_len, int causal, int window) {
  if (j < 0 || j >= kv_len) return 0;
  if (causal && j > qpos) return 0;
  if (window > 0 && !(qpos - j >= 0 && (qpos - j) < window)) return 0;
  return 1;
}

/*
 * One output row: batch b, query head h, query row i.  `x` is scratch of
 * kv_len doubles, `acc` scratch of head_dim doubles, `out` receives
 * head_dim doubles.
 */
static void attend_row(const void *q, const void *k, const void *v, int fmt,
                       int batch_idx, int h, int i, int q_len, int kv_len,
                       int num_q_heads, int num_kv_heads, int head_dim,
                       int causal, int window, double softcap, double *x,
                       double *acc, double *out) {
  int group = num_q_heads / num_kv_heads;
  int hk = h / group;
  long qpos = (long)kv_len - q_len + i;
  double scale = 1.0 / sqrt((double)head_dim);
  int64_t q_row = (((int64_t)batch_idx * num_q_heads + h) * q_len + i) * head_dim;
  int64_t kv_head = ((int64_t)batch_idx * num_kv_heads + hk) * kv_len;

  /* Logits of the visible keys; the maximum over them. */
  int any = 0;
  double m = -INFINITY;
  for (long j = 0; j < kv_len; ++j) {
    if (!key_visible(j, qpos, kv_len, causal, window)) continue;
    double dot = 0.0;
    for (int d = 0; d < head_dim; ++d)
      dot += load_elem(q, q_row + d, fmt) *
             load_elem(k, (kv_head + j) * head_dim + d, fmt);
    double s = dot * scale;
    if (softcap > 0.0) s = softcap * tanh(s / softcap);
    x[j] = s;
    if (!any || s > m) m = s;
    any = 1;
  }

  if (!any) { /* no visible key: the row is zero */
    for (int d = 0; d < head_dim; ++d) out[d] = 0.0;
    return;
  }

  /* Softmax weights and the weighted sum of values. */
  double denom = 0.0;
  for (int d = 0; d < head_dim; ++d) acc[d] = 0.0;
  for (long j = 0; j < kv_len; ++j) {
    if (!key_visible(j, qpos, kv_len, causal, window)) continue;
    double w = exp(x[j] - m);
    denom += w;
    for (int d = 0; d < head_dim; ++d)
      acc[d] += w * load_elem(v, (kv_head + j) * head_dim + d, fmt);
  }
  for (int d = 0; d < head_dim; ++d) out[d] = acc[d] / denom;
}

/*
 * Compute selected output rows.  rows[r] = (b * num_q_heads + h) * q_len + i;
 * out is n_rows x head_dim doubles.  When rows is NULL every row is computed
 * in natural order (out then has q's shape).  n_threads <= 0 uses the OpenMP
 * default.  Returns 0, or -1 on bad arguments / allocation failure.
 */
int oracle_gqa_attn_rows(const void *q, const void *k, const void *v, int fmt,
                         int batch, int q_len, int kv_len, int num_q_heads,
                         int num_kv_heads, int head_dim, int causal, int window,
                         double softcap, const int64_t *rows, int64_t n_rows,
                         double *out, int n_threads) {
  if (batch < 0 || q_len < 0 || kv_len < 0 || num_q_heads <= 0 ||
      num_kv_heads <= 0 || head_dim <= 0 || num_q_heads % num_kv_heads != 0 ||
      !(softcap >= 0.0) || (fmt != ORACLE_F64 && fmt != ORACLE_BF16))
    return -1;
  int64_t total = (int64_t)batch * num_q_heads * q_len;
  if (rows == NULL) n_rows = total;
  if (n_rows <= 0) return 0;
  for (int64_t r = 0; rows != NULL && r < n_rows; ++r)
    if (rows[r] < 0 || rows[r] >= total) return -1;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
  int failed = 0;
#pragma omp parallel
  {
    double *x = (double *)malloc(sizeof(double) * (size_t)(kv_len > 0 ? kv_len : 1));
    double *acc = (double *)malloc(sizeof(double) * (size_t)head_dim);
    if (!x || !acc) {
#pragma omp atomic write
      failed = 1;
    } else {
#pragma omp for schedule(dynamic, 4)
      for (int64_t r = 0; r < n_rows; ++r) {
        int64_t id = rows ? rows[r] : r;
        int i = (int)(id % q_len);
        int64_t bh = id / q_len;
        int h = (int)(bh % num_q_heads);
        int b = (int)(bh / num_q_heads);
        attend_row(q, k, v, fmt, b, h, i, q_len, kv_len, num_q_heads,
                   num_kv_heads, head_dim, causal, window, softcap, x, acc,
                   out + r * head_dim);
      }
    }
    free(x);
    free(acc);
  }
  return failed ? -1 : 0;
}

/* Threads the OpenMP runtime would use (for reporting). */
int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
