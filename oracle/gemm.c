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

/* C (M x N, overwritten) from the unpacked operands ("Approach": bit-shift scaling and accumulation):
 * for every unpacked line (i, l) of A and (j, m) of B,
 *   C[i, j] += R^(l + m) * sum over inner triples (t, lA, lB) of R^(lA + lB) * A'[(i,l),p] * B'[p,(j,m)]
 * with R = 2^(b-1).  *macs (when not NULL) gets the number of multiply-adds of unpacked entries the
 * loop executed, the count the unpack ratio describes. */
int oracle_unpacked_gemm(const oracle_plan_t *pl, const int32_t *a_lines, const int32_t *b_lines,
                         const int32_t *pairs, const int8_t *Aq, const int8_t *Bq, int64_t *C,
                         int64_t *macs) {
  const int64_t N = pl->N, Ke = pl->K_eff;
  const int sh = pl->b - 1;
  int64_t count = 0;
  memset(C, 0, (size_t)(pl->M * N) * sizeof(int64_t));
  for (int64_t u = 0; u < pl->M_eff; ++u) {
    const int64_t i = a_lines[2 * u];
    const int l = a_lines[2 * u + 1];
    for (int64_t w = 0; w < pl->N_eff; ++w) {
      const int64_t j = b_lines[2 * w];
      const int m = b_lines[2 * w + 1];
      int64_t acc = 0;
      for (int64_t p = 0; p < Ke; ++p) {
        const int e = pairs[3 * p + 1] + pairs[3 * p + 2];
        acc += (int64_t)Aq[u * Ke + p] * (int64_t)Bq[w * Ke + p] * ((int64_t)1 << (e * sh));
      }
      count += Ke;
      C[i * N + j] += acc * ((int64_t)1 << ((l + m) * sh));
    }
  }
  if (macs) *macs = count;
  return OR_OK;
}
