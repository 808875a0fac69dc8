/*
 * unpack.c -- oracle step 5: the unpacked b-bit operands, stated without a memory layout.
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * IM-Unpack summary page, "Approach": out-of-bound entries are written as several in-bound b-bit
 * integers by row or column unpacking.  With the unpacked lines and inner triples of oracle_unpack_lines
 * (a line of A is (i, l), a line of B is (j, m), an inner index is (t, lA, lB)):
 *   A'[(i, l), (t, lA, lB)] = digit l + lA of A[i, t]
 *   B'[(t, lA, lB), (j, m)] = digit m + lB of B[t, j]
 * (one of l, lA is always 0 unless A is unpacked both ways, and likewise for B).  Under the hybrid
 * strategy a row of A unpacked OUTER (dir_a has the OUTER part and the level the row carries, LrA, is
 * above 1) has all its digits on its own lines, so its entries at inner triples with lA > 0 are zero;
 * likewise a column of B unpacked OUTER (LcB above 1) at lB > 0.
 * Output: Aq is M_eff x K_eff and Bq is N_eff x K_eff (B'^T), row u / w and column p in the order of the
 * enumeration, which only names the entries.
 */
#include "oracle.h"

int oracle_unpack(const oracle_plan_t *pl, const int32_t *LrA, const int32_t *LcB,
                  const int32_t *a_lines, const int32_t *b_lines, const int32_t *pairs,
                  const int64_t *A, const int64_t *B, int8_t *Aq, int8_t *Bq) {
  const int b = pl->b;
  const int64_t K = pl->K, N = pl->N, Ke = pl->K_eff;
  const int64_t lim = ((int64_t)1 << (b - 1)) - 1;
  for (int64_t u = 0; u < pl->M_eff; ++u) {
    const int64_t i = a_lines[2 * u];
    const int l = a_lines[2 * u + 1];
    const int whole_row = (pl->dir_a & OR_DIR_OUTER) && LrA[i] > 1;
    for (int64_t p = 0; p < Ke; ++p) {
      const int64_t t = pairs[3 * p];
      const int lA = pairs[3 * p + 1];
      int64_t d = 0;
      if (!(whole_row && lA > 0)) d = oracle_digit(A[i * K + t], l + lA, b);
      if (d > lim || d < -lim) return OR_ERR_RANGE;
      Aq[u * Ke + p] = (int8_t)d;
    }
  }
  for (int64_t w = 0; w < pl->N_eff; ++w) {
    const int64_t j = b_lines[2 * w];
    const int m = b_lines[2 * w + 1];
    const int whole_col = (pl->dir_b & OR_DIR_OUTER) && LcB[j] > 1;
    for (int64_t p = 0; p < Ke; ++p) {
      const int64_t t = pairs[3 * p];
      const int lB = pairs[3 * p + 2];
      int64_t d = 0;
      if (!(whole_col && lB > 0)) d = oracle_digit(B[t * N + j], m + lB, b);
      if (d > lim || d < -lim) return OR_ERR_RANGE;
      Bq[w * Ke + p] = (int8_t)d;
    }
  }
  return OR_OK;
}
