/*
 * unpack.c -- oracle step 5: the unpacked b-bit operands A' (M_unp x K_unp) and B'^T (N_unp x K_unp).
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * IM-Unpack summary page, "Approach": out-of-bound entries are written as several in-bound b-bit
 * integers by row or column unpacking.  Entry (u, p) of A' is digit lvlA[u] + lAk[p] of
 * A[srcA[u], tK[p]]; entry (w, p) of B'^T is digit lvlB[w] + lBk[p] of B[tK[p], srcB[w]]; unused lines
 * and inner padding are zero.  One of lvlA[u], lAk[p] is always 0, and likewise for B.  Under the
 * hybrid strategy a matrix is unpacked in both directions: a source row of A that is unpacked OUTER
 * (dir_a has the OUTER part and LrA, the level the row carries, is above 1) has all its digits on its
 * own lines, so its entries in the inner segments of level lAk[p] > 0 are zero; likewise a source column
 * of B unpacked OUTER (LcB above 1) at lBk[p] > 0.
 */
#include "oracle.h"

int oracle_unpack(const oracle_plan_t *pl, const int32_t *tK, const int32_t *lAk,
                  const int32_t *lBk, const int32_t *srcA, const int32_t *lvlA,
                  const int32_t *srcB, const int32_t *lvlB, const int32_t *LrA, const int32_t *LcB,
                  const int64_t *A, const int64_t *B, int8_t *Aunp, int8_t *Bunp_t) {
  const int b = pl->b;
  const int64_t K = pl->K, N = pl->N, Ku = pl->K_unp;
  const int64_t lim = ((int64_t)1 << (b - 1)) - 1;
  for (int64_t u = 0; u < pl->M_unp; ++u)
    for (int64_t p = 0; p < Ku; ++p) {
      int64_t d = 0;
      const int whole_row = (pl->dir_a & OR_DIR_OUTER) && srcA[u] >= 0 && LrA[srcA[u]] > 1;
      if (srcA[u] >= 0 && tK[p] >= 0 && !(whole_row && lAk[p] > 0))
        d = oracle_digit(A[(int64_t)srcA[u] * K + tK[p]], lvlA[u] + lAk[p], b);
      if (d > lim || d < -lim) return OR_ERR_RANGE;
      Aunp[u * Ku + p] = (int8_t)d;
    }
  for (int64_t w = 0; w < pl->N_unp; ++w)
    for (int64_t p = 0; p < Ku; ++p) {
      int64_t d = 0;
      const int whole_col = (pl->dir_b & OR_DIR_OUTER) && srcB[w] >= 0 && LcB[srcB[w]] > 1;
      if (srcB[w] >= 0 && tK[p] >= 0 && !(whole_col && lBk[p] > 0))
        d = oracle_digit(B[(int64_t)tK[p] * N + srcB[w]], lvlB[w] + lBk[p], b);
      if (d > lim || d < -lim) return OR_ERR_RANGE;
      Bunp_t[w * Ku + p] = (int8_t)d;
    }
  return OR_OK;
}
