/*
 * rtn.c -- oracle step 2: round-to-nearest quantisation, without clipping (the method) or with it (the
 * comparison variant).
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * IM-Unpack summary page: "Problem" (a few heavy hitters lie far outside the low-bit range),
 * "Approach" (those entries are kept and unpacked later, not clipped), measured-effects table (beta
 * and the percentile p; clipping at 99.5% is a separate ablation).
 * READINGs: s = (float)beta / q in fp32; x_int = rint(fp32(x * s)) with ties to even (the IEEE default
 * rounding, one fp32 multiply, no fused operation); Delta = q / (float)beta is the dequantisation step;
 * q == 0 falls back to the group maximum, and to s = Delta = 1 when the maximum is 0 too.
 * Clipping variant (the measured-effects table's 99.5% row, READING: the scaled value is clamped to
 * [-beta, beta] before rounding, which equals clamping the rounded value since beta is an integer).
 * Built with -ffp-contract=off and without fast-math, so every operation is one IEEE fp32 operation.
 */
#include <math.h>
#include <stdlib.h>
#include "oracle.h"

/* Quantises one group of n values read with stride `stride` from x; writes with the same stride. */
static int quantize_group(const float *x, int64_t n, int64_t stride, double p, int beta, int clip,
                          int64_t *xint, float *delta, float *qval) {
  float *g = (float *)calloc((size_t)(n > 0 ? n : 1), sizeof(float));
  float mx = 0.0f;
  for (int64_t i = 0; i < n; ++i) {
    float v = x[i * stride];
    if (!isfinite(v)) { free(g); return OR_ERR_NONFINITE; }
    g[i] = v;
    if (fabsf(v) > mx) mx = fabsf(v);
  }
  float q = oracle_percentile_abs(g, n, p);
  free(g);
  if (q == 0.0f) q = mx;
  float s, d;
  if (q == 0.0f) {
    s = 1.0f;
    d = 1.0f;
  } else {
    s = (float)beta / q;
    d = q / (float)beta;
  }
  *delta = d;
  *qval = q;
  for (int64_t i = 0; i < n; ++i) {
    float y = x[i * stride] * s;
    if (clip) {
      if (y > (float)beta) y = (float)beta;
      if (y < -(float)beta) y = -(float)beta;
    }
    if (!(fabsf(y) < 2147483648.0f)) return OR_ERR_RANGE;
    xint[i * stride] = (int64_t)rintf(y);
  }
  return OR_OK;
}

/* x: rows x cols row-major fp32 (bf16 inputs are widened exactly by the caller).
 * gran: OR_PER_TENSOR / OR_PER_ROW / OR_PER_COL over the stored matrix.
 * delta, qval: 1 / rows / cols entries.  xint: rows x cols. */
int oracle_rtn_quantize_ex(const float *x, int64_t rows, int64_t cols, int gran, double p, int beta, int clip,
                           int64_t *xint, float *delta, float *qval) {
  if (rows < 0 || cols < 0 || !(p > 0.0 && p <= 1.0) || beta < 1) return OR_ERR_ARG;
  int rc = OR_OK;
  if (gran == OR_PER_TENSOR) {
    rc = quantize_group(x, rows * cols, 1, p, beta, clip, xint, delta, qval);
  } else if (gran == OR_PER_ROW) {
    for (int64_t r = 0; r < rows && rc == OR_OK; ++r)
      rc = quantize_group(x + r * cols, cols, 1, p, beta, clip, xint + r * cols, delta + r, qval + r);
  } else if (gran == OR_PER_COL) {
    for (int64_t c = 0; c < cols && rc == OR_OK; ++c)
      rc = quantize_group(x + c, rows, cols, p, beta, clip, xint + c, delta + c, qval + c);
  } else {
    rc = OR_ERR_ARG;
  }
  return rc;
}

int oracle_rtn_quantize(const float *x, int64_t rows, int64_t cols, int gran, double p, int beta,
                        int64_t *xint, float *delta, float *qval) {
  return oracle_rtn_quantize_ex(x, rows, cols, gran, p, beta, 0, xint, delta, qval);
}
