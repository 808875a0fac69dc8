/*
 * digits.c -- oracle: the level of an integer and its sign-magnitude base-R digits.
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * IM-Unpack summary page, "Approach": an out-of-bound integer is decomposed into several in-bound
 * b-bit integers whose bit-shifted sum is the original.  READING: radix R = 2^(b-1), in-range set
 * |v| <= R-1, digits d_l(v) = sgn(v) * ((|v| >> l(b-1)) & (R-1)), so sum_l R^l d_l(v) = v and every
 * digit carries the sign of v.
 */
#include <stdlib.h>
#include "oracle.h"

/* Number of base-R digits of |v|, at least 1. */
int oracle_level(int64_t v, int b) {
  uint64_t m = (uint64_t)(v < 0 ? -v : v);
  int n = 0;
  while (m > 0) {
    m >>= (b - 1);
    ++n;
  }
  return n > 0 ? n : 1;
}

int64_t oracle_digit(int64_t v, int l, int b) {
  int shift = l * (b - 1);
  if (shift >= 63) return 0;
  uint64_t m = (uint64_t)(v < 0 ? -v : v);
  int64_t d = (int64_t)((m >> shift) & (((uint64_t)1 << (b - 1)) - 1));
  return v < 0 ? -d : d;
}

/* Bulk forms for exhaustive checks: out[i * nl + l] = d_l(v[i]) for l < nl; lev[i] = L(v[i]). */
void oracle_digits_array(const int64_t *v, int64_t n, int b, int nl, int64_t *out, int32_t *lev) {
  for (int64_t i = 0; i < n; ++i) {
    for (int l = 0; l < nl; ++l) out[i * nl + l] = oracle_digit(v[i], l, b);
    lev[i] = oracle_level(v[i], b);
  }
}
