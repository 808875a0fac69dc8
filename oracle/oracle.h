/*
 * oracle.h -- declarations of the CPU oracle for the IM-Unpack exact low-bit integer GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg
 * (and its --impl reference arm) may load or call this code.  It shares no code, header, table or
 * constant with the CUDA library under bit_integer_gemm_b200/, and neither side includes the other.
 *
 * Source of the method: "IM-Unpack: Training and Inference with Arbitrarily Low Precision Integers"
 * (atlas.scime.ai summary page).  Each function cites the section it follows.  Points the page leaves
 * open are marked READING and are the same readings the library documents in include/imq.h.
 *
 * Parity pins: every function here is checked by tests/test_oracle_pins.py against something other
 * than itself (sorting, brute force, closed forms, invariants, exact library arithmetic).
 */
#ifndef IMQ_ORACLE_H
#define IMQ_ORACLE_H
#include <stdint.h>

#define OR_OK 0
#define OR_ERR_ARG 1
#define OR_ERR_NONFINITE 2
#define OR_ERR_RANGE 3

#define OR_PER_TENSOR 0
#define OR_PER_ROW 1
#define OR_PER_COL 2

#define OR_MIX 0
#define OR_ROW_ROW 1
#define OR_ROW_COL 2
#define OR_COL_ROW 3
#define OR_COL_COL 4
/* Joint Mix: the (A, B) direction pair of least exact unpacked cost M_eff * N_eff * K_eff over the four
 * pairs (a reading of the page's per-matrix choice; see oracle_plan). */
#define OR_MIX_JOINT 5
/* Hybrid ("unpack both"): per matrix, the outer lines with at least tau out-of-range entries unpacked
 * OUTER and the rest INNER, tau of least unpacked size (a reading; see oracle_plan). */
#define OR_HYBRID 6

#define OR_DIR_NONE 0
#define OR_DIR_OUTER 1
#define OR_DIR_INNER 2
#define OR_DIR_BOTH 3 /* OR_DIR_OUTER | OR_DIR_INNER: the hybrid's two parts */

/* Exponents e = lA + lB of the inner pairs: at most 2 * 31 + 1 distinct values (levels are at most 32). */
#define OR_MAX_GROUPS 64

/* The plan: sizes and counts only.  The unpacked operands are stated without any memory layout: an
 * unpacked line of A is a pair (source row i, level l), an unpacked line of B a pair (source column j,
 * level m), an unpacked inner index a triple (t, lA, lB); see oracle_unpack_lines. */
typedef struct {
  int32_t b, strategy, dir_a, dir_b;
  int64_t M, K, N;
  int64_t M_eff, N_eff, K_eff;  /* numbers of unpacked lines of A, of B, and of inner triples     */
  double ratio;
  double bound;            /* sum_t max_i|A_it| * max_j|B_tj|, rounded to double          */
  int32_t bound_lt_2_31;   /* exact comparison of the bound with 2^31                     */
  int32_t n_groups;        /* distinct exponents e = lA + lB among the inner triples      */
  int32_t lmax[4];         /* A rows, A cols, B rows, B cols                              */
  int64_t suml[4];
  int64_t oor_lines[4];
  int32_t group_e[OR_MAX_GROUPS];    /* the exponents, ascending                         */
  int64_t group_len[OR_MAX_GROUPS];  /* inner triples with that exponent                 */
} oracle_plan_t;

/* percentile.c */
float oracle_percentile_abs(const float *v, int64_t n, double p);
/* rtn.c */
int oracle_rtn_quantize(const float *x, int64_t rows, int64_t cols, int gran, double p, int beta,
                        int64_t *xint, float *delta, float *qval);
/* The same with clip != 0: the clipping comparison variant (scaled values clamped to [-beta, beta]). */
int oracle_rtn_quantize_ex(const float *x, int64_t rows, int64_t cols, int gran, double p, int beta, int clip,
                           int64_t *xint, float *delta, float *qval);
/* digits.c */
int oracle_level(int64_t v, int b);
int64_t oracle_digit(int64_t v, int l, int b);
void oracle_digits_array(const int64_t *v, int64_t n, int b, int nl, int64_t *out, int32_t *lev);
/* plan.c */
int oracle_plan(const int64_t *A, const int64_t *B, int64_t M, int64_t K, int64_t N, int b,
                int strategy, int32_t *LrA, int32_t *LcA, int32_t *LrB, int32_t *LcB,
                oracle_plan_t *out);
int oracle_unpack_lines(const oracle_plan_t *pl, const int32_t *LrA, const int32_t *LcA,
                        const int32_t *LrB, const int32_t *LcB, int32_t *a_lines, int32_t *b_lines,
                        int32_t *pairs);
/* unpack.c */
int oracle_unpack(const oracle_plan_t *pl, const int32_t *LrA, const int32_t *LcB,
                  const int32_t *a_lines, const int32_t *b_lines, const int32_t *pairs,
                  const int64_t *A, const int64_t *B, int8_t *Aq, int8_t *Bq);
/* gemm.c */
void oracle_gemm_i64(const int64_t *A, const int64_t *B, int64_t M, int64_t K, int64_t N,
                     int64_t *C, int nthreads);
int oracle_unpacked_gemm(const oracle_plan_t *pl, const int32_t *a_lines, const int32_t *b_lines,
                         const int32_t *pairs, const int8_t *Aq, const int8_t *Bq, int64_t *C,
                         int64_t *macs);
/* dequant.c */
void oracle_dequant(const int64_t *C, int64_t M, int64_t N, const float *dA, int gA,
                    const float *dB, int gB, double *Cf);
#endif
