/*
 * dequant.c -- oracle step 8: the dequantised product.
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * IM-Unpack summary page, one-line summary and "Key results": RTN integer GEMMs stand in for the
 * floating-point GEMMs, so the integer product is mapped back by the two quantisation steps.
 * READING: Cf[i,j] = C[i,j] * (DeltaA[i] * DeltaB[j]), evaluated here in double from the fp32 steps.
 * gA: OR_PER_TENSOR (one value) or OR_PER_ROW (M values); gB: OR_PER_TENSOR or OR_PER_COL (N values).
 */
#include "oracle.h"

void oracle_dequant(const int64_t *C, int64_t M, int64_t N, const float *dA, int gA,
                    const float *dB, int gB, double *Cf) {
  for (int64_t i = 0; i < M; ++i)
    for (int64_t j = 0; j < N; ++j) {
      double a = (double)(gA == OR_PER_TENSOR ? dA[0] : dA[i]);
      double b = (double)(gB == OR_PER_TENSOR ? dB[0] : dB[j]);
      Cf[i * N + j] = (double)C[i * N + j] * (a * b);
    }
}
