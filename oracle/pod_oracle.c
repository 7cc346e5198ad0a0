/*
 * pod_oracle.c -- plain fp64 CPU attention, the parity oracle.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg do. It shares no code, header or table with the CUDA library.
 *
 * What it computes (the plain definition; POD-Attention's fusion only moves
 * independent tiles around and leaves these values unchanged -- Silicon &
 * Systems digest of the ASPLOS'25 paper, section "Virtual CTAs and SM-aware
 * balance"): for one query row q (bf16, head h) and one KV cache (bf16,
 * [len, Hk, d]) restricted to keys [kbeg, kend):
 *
 *     g      = h / (H / Hk)                      (contiguous GQA groups)
 *     s_j    = (sum_k q_k * K[j, g, k]) / sqrt(d)      j in [kbeg, kend)
 *     m      = max_j s_j
 *     Z      = sum_j exp(s_j - m)
 *     O[:]   = sum_j exp(s_j - m) * V[j, g, :] / Z
 *     LSE    = m + ln Z
 *
 * Everything is fp64; the bf16 inputs are widened exactly in the inner loop.
 * Two passes per item (max, then weighted sums), no online rescaling. An empty
 * key range gives O = 0 and LSE = -inf.
 *
 * Parallel over items with OpenMP (one item = one (row, head, key range)).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static inline double bf16_to_f64(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/*
 * n_items items. For item i:
 *   q_rows[i]   : pointer to the bf16 query vector of that row and head (d values)
 *   kv_cache[i] : index into k_ptrs / v_ptrs
 *   kbeg[i], kend[i] : key range (kend exclusive)
 *   head_kv[i]  : KV head g used by this item
 * k_ptrs[c] / v_ptrs[c] : bf16 [len_c, Hk, d], row-major.
 * Outputs o[i*d .. i*d+d-1] and lse[i] (fp64).
 * Returns 0, or -1 if a scratch allocation failed.
 */
int pod_oracle_items(long long n_items, int Hk, int d, const uint16_t *const *q_rows,
                     const int *kv_cache, const long long *kbeg, const long long *kend,
                     const int *head_kv, const uint16_t *const *k_ptrs,
                     const uint16_t *const *v_ptrs, double *o, double *lse, int n_threads) {
  int failed = 0;
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
#pragma omp parallel
  {
    double *qv = (double *)malloc(sizeof(double) * (size_t)d);
    double *acc = (double *)malloc(sizeof(double) * (size_t)d);
    double *s = NULL;
    long long s_cap = 0;
    int mine_ok = (qv != NULL && acc != NULL);
    if (!mine_ok) {
#pragma omp atomic write
      failed = 1;
    }
#pragma omp for schedule(dynamic, 4)
    for (long long it = 0; it < n_items; ++it) {
      if (!mine_ok) continue;
      const long long a = kbeg[it], b = kend[it];
      double *out = o + it * (long long)d;
      if (b <= a) {
        for (int k = 0; k < d; ++k) out[k] = 0.0;
        lse[it] = -INFINITY;
        continue;
      }
      const long long n = b - a;
      if (n > s_cap) {
        free(s);
        s = (double *)malloc(sizeof(double) * (size_t)n);
        s_cap = s ? n : 0;
        if (!s) {
#pragma omp atomic write
          failed = 1;
          mine_ok = 0;
          continue;
        }
      }
      for (int k = 0; k < d; ++k) qv[k] = bf16_to_f64(q_rows[it][k]);
      const uint16_t *K = k_ptrs[kv_cache[it]];
      const uint16_t *V = v_ptrs[kv_cache[it]];
      const long long row_stride = (long long)Hk * d;
      const int g = head_kv[it];
      /* pass 1: scores and their maximum */
      double m = -INFINITY;
      for (long long j = 0; j < n; ++j) {
        const uint16_t *kr = K + (a + j) * row_stride + (long long)g * d;
        double dot = 0.0;
        for (int k = 0; k < d; ++k) dot += qv[k] * bf16_to_f64(kr[k]);
        s[j] = dot * inv_sqrt_d;
        if (s[j] > m) m = s[j];
      }
      /* pass 2: normaliser and weighted sum of V */
      double Z = 0.0;
      for (int k = 0; k < d; ++k) acc[k] = 0.0;
      for (long long j = 0; j < n; ++j) {
        const double w = exp(s[j] - m);
        Z += w;
        const uint16_t *vr = V + (a + j) * row_stride + (long long)g * d;
        for (int k = 0; k < d; ++k) acc[k] += w * bf16_to_f64(vr[k]);
      }
      for (int k = 0; k < d; ++k) out[k] = acc[k] / Z;
      lse[it] = m + log(Z);
    }
    free(qv);
    free(acc);
    free(s);
  }
  return failed ? -1 : 0;
}

/* Number of threads OpenMP would use (for reporting). */
int pod_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
