/*
 * gemm.c -- oracle steps 6-7: the integer product, directly and through the unpacked operands.
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * IM-Unpack summary page, "Approach" and the one-line summary: the unpacked low bit-width GEMMs,
 * followed by bit-shift scaling and accumulation, give the original integer GEMM exactly.  The
 * defining result is therefore the plain integer product, computed here in int64 by a triple loop.
 */
#include <omp.h>
#include <string.h>
#include "oracle.h"

/* C = A * B, A M x K, B K x N, row-major int64; nthreads <= 0 uses the OpenMP default. */
void oracle_gemm_i64(const int64_t *A, const int64_t *B, int64_t M, int64_t K, int64_t N,
                     int64_t *C, int nthreads) {
  const int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
#pragma omp parallel for schedule(static) num_threads(nt)
  for (int64_t i = 0; i < M; ++i) {
    int64_t *c = C + i * N;
    for (int64_t j = 0; j < N; ++j) c[j] = 0;
    for (int64_t t = 0; t < K; ++t) {
      const int64_t a = A[i * K + t];
      if (a == 0) continue;
      const int64_t *brow = B + t * N;
      for (int64_t j = 0; j < N; ++j) c[j] += a * brow[j];
    }
  }
}

/* C (M x N, overwritten) from the unpacked operands: for every pair of used lines (u, w),
 *   acc = sum over exponent groups g of R^e_g * sum_{p in g} A'[u,p] * B'^T[w,p]
 * and acc * R^(lvlA[u] + lvlB[w]) is added to C[srcA[u], srcB[w]]. */
int oracle_unpacked_gemm(const oracle_plan_t *pl, const int32_t *srcA, const int32_t *lvlA,
                         const int32_t *srcB, const int32_t *lvlB, const int8_t *Aunp,
                         const int8_t *Bunp_t, int64_t *C) {
  const int64_t N = pl->N, Ku = pl->K_unp;
  const int sh = pl->b - 1;
  memset(C, 0, (size_t)(pl->M * N) * sizeof(int64_t));
  for (int64_t u = 0; u < pl->M_unp; ++u) {
    if (srcA[u] < 0) continue;
    for (int64_t w = 0; w < pl->N_unp; ++w) {
      if (srcB[w] < 0) continue;
      int64_t acc = 0;
      for (int g = 0; g < pl->n_groups; ++g) {
        int64_t part = 0;
        for (int64_t p = pl->group_off[g]; p < pl->group_off[g] + pl->group_padded[g]; ++p)
          part += (int64_t)Aunp[u * Ku + p] * (int64_t)Bunp_t[w * Ku + p];
        acc += part * ((int64_t)1 << (pl->group_e[g] * sh));
      }
      C[(int64_t)srcA[u] * N + srcB[w]] += acc * ((int64_t)1 << ((lvlA[u] + lvlB[w]) * sh));
    }
  }
  return OR_OK;
}
