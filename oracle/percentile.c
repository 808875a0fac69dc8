/*
 * percentile.c -- oracle step 1: the percentile that sets the RTN scale.
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * IM-Unpack summary page, measured-effects table: the default quantiser maps the p = 95% percentile
 * of |x| to beta, and the p = 100% ablation maps the maximum.  READING: nearest-rank percentile --
 * sort |x| ascending into v_1..v_n, k = clamp(ceil(p*n), 1, n), q = v_k -- so q is an element of the
 * data and p = 1 gives the maximum exactly.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#include "oracle.h"

static int cmp_float_asc(const void *a, const void *b) {
  float x = *(const float *)a, y = *(const float *)b;
  return (x > y) - (x < y);
}

/* v: n finite values (not modified).  Returns the nearest-rank p-quantile of |v|. */
float oracle_percentile_abs(const float *v, int64_t n, double p) {
  if (n <= 0) return 0.0f;
  float *a = (float *)malloc((size_t)n * sizeof(float));
  for (int64_t i = 0; i < n; ++i) a[i] = fabsf(v[i]);
  qsort(a, (size_t)n, sizeof(float), cmp_float_asc);
  int64_t k = (int64_t)ceil(p * (double)n);
  if (k < 1) k = 1;
  if (k > n) k = n;
  float q = a[k - 1];
  free(a);
  return q;
}
