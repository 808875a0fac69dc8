/*
 * imq.h -- C ABI of the IM-Unpack exact low-bit integer GEMM for NVIDIA B200 (sm_100a).
 *
 * Source of the method: "IM-Unpack: Training and Inference with Arbitrarily Low Precision Integers"
 * (atlas.scime.ai summary page), sections "Approach", "Problem", "Key results", the measured-effects
 * table and "Limitations".  The page states the method in prose only; every point it leaves open is
 * fixed below and marked READING.
 *
 * The hot path has three stages, one entry point each:
 *   1. imq_rtn_quantize   round-to-nearest quantisation: the p-th percentile of |x| of each group maps
 *                         to the bound beta, heavy hitters are kept unclipped   ("Approach", "Problem",
 *                         measured-effects rows on beta and p)
 *   2. imq_plan           per-line outlier statistics and the per-matrix choice of row or column
 *                         unpacking ("Approach": chosen per matrix from outlier counts; the Mix row and
 *                         the four fixed-strategy rows of the measured-effects table)
 *   3. imq_unpacked_gemm  digit-split unpacking into b-bit integers, b-bit integer GEMMs on the tensor
 *                         cores, then bit-shift scaling and accumulation that give back the exact
 *                         integer product ("Approach"), plus an fp32 dequantised copy.
 *
 * Conventions shared by every call
 *   - Matrices are dense and row-major with a leading dimension (elements between consecutive rows).
 *   - Every tensor pointer is DEVICE memory owned by the caller unless a parameter says "host".
 *   - Every call is asynchronous on the given stream except imq_plan (it reads a small summary back
 *     to the host to size the unpacked operands) and the imq_plan_* query calls.
 *   - Argument errors are returned at once and launch nothing.  Errors found by a kernel (a non-finite
 *     input, an integer that leaves its type) are written to a per-device status word; the next
 *     imq_plan call or imq_device_status() returns it.  No call aborts the process.
 *   - Every wait inside a kernel is bounded; a wait that runs out sets IMQ_ERR_TIMEOUT and the kernel
 *     returns instead of hanging the device.
 *   - GEMM notation: C = A * B with A logically M x K, B logically K x N, unpack width b in [2, 8],
 *     radix R = 2^(b-1).  The b-bit in-range set is |v| <= R-1 (READING: symmetric sign-magnitude
 *     digits, so every digit of an entry has the entry's sign).
 */
#ifndef IMQ_H
#define IMQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t); NULL selects the legacy default stream. */
typedef struct CUstream_st *imq_stream_t;

typedef enum {
  IMQ_OK = 0,
  IMQ_ERR_ARG = 1,         /* null pointer, bad size, stride, dtype, b outside [2,8], p outside (0,1]   */
  IMQ_ERR_NONFINITE = 2,   /* NaN or Inf in a quantiser input                                           */
  IMQ_ERR_RANGE = 3,       /* |x*s| >= 2^31, an int16 output above 32767, or an int32 C requested while */
                           /* the plan's bound says the product may leave int32                          */
  IMQ_ERR_BUFFER = 4,      /* workspace smaller than imq_plan_info.workspace_bytes                      */
  IMQ_ERR_TIMEOUT = 5,     /* a bounded wait inside a kernel ran out                                    */
  IMQ_ERR_CUDA = 6,        /* a CUDA runtime call failed                                                 */
  IMQ_ERR_UNSUPPORTED = 7, /* legal input outside what the kernels implement (see imq_plan)             */
  IMQ_ERR_PLAN = 8,        /* imq_rtn_quantize_unpack: a quantised entry above the plan's max |A[:, t]| */
  IMQ_ERR_BOUNDS = 9       /* debug build (IMQ_DEBUG) only: a plan index outside the plan's sizes        */
} imq_status;

typedef enum { IMQ_F32 = 0, IMQ_BF16 = 1, IMQ_I16 = 2, IMQ_I32 = 3, IMQ_I64 = 4 } imq_dtype;

/* Quantisation groups, relative to the STORED matrix passed to imq_rtn_quantize. */
typedef enum { IMQ_PER_TENSOR = 0, IMQ_PER_ROW = 1, IMQ_PER_COL = 2 } imq_gran;

/* Unpack strategy: Mix decides per matrix; the fixed ones force (A direction)/(B direction), named
 * for the C = A*B convention: "row" of A = an output row (OUTER), "col" of A = an inner index (INNER),
 * "row" of B = an inner index (INNER), "col" of B = an output column (OUTER).
 * READING: the page never says whether its GEMM is A*B or A*B^T; the directions are therefore named
 * by axis (OUTER/INNER) in imq_plan_info. */
typedef enum {
  IMQ_MIX = 0, IMQ_ROW_ROW = 1, IMQ_ROW_COL = 2, IMQ_COL_ROW = 3, IMQ_COL_COL = 4,
  /* Joint Mix (READING of the per-matrix choice that weighs both matrices together): the direction pair
   * of least exact unpacked size M_eff * N_eff * K_eff (the unpack ratio's numerator) over the four
   * pairs, starting from the Mix choice and taking strict improvements in the order row/row, row/col,
   * col/row, col/col; a matrix without out-of-range entries stays not unpacked. */
  IMQ_MIX_JOINT = 5,
  /* Hybrid, "unpack both" (READING of the per-matrix choice for matrices whose heavy hitters sit in
   * some rows AND some columns, which pure row or column unpacking both handle badly): per matrix, the
   * outer lines (rows of A, columns of B) holding at least tau out-of-range entries are unpacked OUTER
   * with all their digits, the other lines INNER, the inner levels taken over those other lines only;
   * tau is the threshold of least M_eff * K_eff (A) or N_eff * K_eff (B) -- thresholds 1 and max + 1
   * are pure row and pure column unpacking, so the size is never above the smaller of the two -- the
   * smallest such tau on a tie.  The plan reads A and B twice more (out-of-range counts per line, then
   * the least count per inner index and level) and decides on the device. */
  IMQ_HYBRID = 6
} imq_strategy;

/* Direction a matrix is unpacked in, a bit set.  NONE: the matrix has no out-of-range entry (Mix and
 * the hybrid).  BOTH = OUTER | INNER: the hybrid unpacks some outer lines OUTER and the rest INNER. */
typedef enum { IMQ_DIR_NONE = 0, IMQ_DIR_OUTER = 1, IMQ_DIR_INNER = 2, IMQ_DIR_BOTH = 3 } imq_dir;

#define IMQ_MAX_GROUPS 64   /* exponent groups e = lA + lB of the inner dimension                         */
#define IMQ_INNER_PAD 128   /* each exponent group of the unpacked inner dimension is padded to this      */
#define IMQ_A_GROUP 32      /* OUTER-unpacked rows of A are packed in groups of this many unpacked rows   */
#define IMQ_B_GROUP 32      /* OUTER-unpacked columns of B are packed in groups of this many columns      */

/* ------------------------------------------------------------------------------------------------ */
/* 1. Round-to-nearest quantisation                                                                  */
/* ------------------------------------------------------------------------------------------------ */
/*
 * imq_rtn_quantize -- per group g (the whole tensor, one stored row or one stored column):
 *   q_g   = nearest-rank p-quantile of |x| over the group: sort |x| ascending into v_1..v_n,
 *           k = clamp(ceil(p*n), 1, n), q = v_k  (READING: nearest rank, so q is an element of the
 *           data and p = 1 gives the maximum, as the p=100% ablation row of the measured-effects
 *           table requires).  If q == 0 the group's maximum is used; if that is 0 too, s = Delta = 1.
 *   s_g   = (float)beta / q_g              fp32, correctly rounded
 *   x_int = rint_half_even(fp32(x * s_g))  no clipping: heavy hitters stay outside +-beta
 *           ("Problem" and "Approach"; clipping is the separate 99.5% ablation row)
 *   Delta_g = q_g / (float)beta            fp32, the dequantisation step (x ~= Delta * x_int)
 *
 * X       device, rows x cols, row-major with leading dimension ld (>= cols), dtype xt (F32 or BF16).
 * Xint    device, dtype it (I16 or I32).  trans_out = 0: rows x cols like X, leading dimension ldq
 *         (>= cols).  trans_out = 1: the transpose, cols x rows, leading dimension ldq (>= rows) -- a
 *         weight W stored K x N is quantised per output channel straight into the N x K layout that
 *         imq_plan takes as B with transB = 1.
 * delta   device, fp32, 1 / rows / cols entries for PER_TENSOR / PER_ROW / PER_COL.
 * qval    device or NULL, fp32, same length as delta: the q each scale was derived from -- the
 *         selected percentile q_g, or the group's maximum where q_g is 0 (0 when that is 0 too).
 * rowmax  device or NULL, int32[rows]: max |x_int| over each row of X (whatever trans_out is).
 * colmax  device or NULL, int32[cols]: max |x_int| over each column of X.
 * Errors: IMQ_ERR_ARG at once; IMQ_ERR_NONFINITE / IMQ_ERR_RANGE through the device status word.
 * Scratch: the per-CTA partial line maxima (and, for PER_TENSOR, the select state) come from a
 *         library-owned stream-ordered memory pool, allocated and freed on `stream`; calls on
 *         different streams therefore never share scratch and may run concurrently.
 */
imq_status imq_rtn_quantize(const void *X, imq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                            imq_gran g, double p, int32_t beta,
                            void *Xint, imq_dtype it, int64_t ldq, int32_t trans_out,
                            float *delta, float *qval, int32_t *rowmax, int32_t *colmax,
                            imq_stream_t stream);

/*
 * imq_rtn_quantize_ex -- imq_rtn_quantize with option flags (0 gives imq_rtn_quantize exactly).
 *   IMQ_RTN_CLIP  the clipping comparison variant of the measured-effects table (its 99.5% row, with
 *                 p = 0.995): the scaled value x * s_g is clamped to [-beta, beta] before rounding
 *                 (READING; equal to clamping the rounded value, beta being an integer), so no entry
 *                 leaves +-beta and nothing is left to unpack when beta <= R - 1.  The scale and Delta
 *                 are those of the unclipped rule.  The method itself keeps heavy hitters: flags = 0.
 * Errors: those of imq_rtn_quantize; IMQ_ERR_ARG for an unknown flag.
 */
#define IMQ_RTN_CLIP 1u
imq_status imq_rtn_quantize_ex(const void *X, imq_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                               imq_gran g, double p, int32_t beta,
                               void *Xint, imq_dtype it, int64_t ldq, int32_t trans_out,
                               float *delta, float *qval, int32_t *rowmax, int32_t *colmax,
                               uint32_t flags, imq_stream_t stream);

/*
 * imq_rtn_quantize_rows_noalloc -- imq_rtn_quantize with g = IMQ_PER_ROW and trans_out = 0 (the
 * per-token quantisation of an activation), with the same arguments otherwise and the same results,
 * but it allocates no device memory.  The IM-Unpack page has no counterpart to this call: it is an
 * interface convenience of this library, not a step of the method.
 *
 * Why: imq_rtn_quantize takes its per-CTA partial column maxima from a library-owned memory pool,
 * which maps more device memory whenever it has to grow.  A process whose own allocator has reserved
 * the free device memory up front (a serving engine that owns every byte of HBM) cannot let a
 * library grow a pool: the allocation fails there, or it takes memory the process had planned for.
 * This call takes its scratch from one fixed array in the library's device image instead, of
 * IMQ_NOALLOC_SCRATCH_BYTES per device, which the CUDA runtime maps when it loads the module.
 *
 * Scratch needed: 4 * cols * G bytes when colmax is requested, where G is the number of CTAs the
 * per-row kernel uses (at most 4 per SM; fewer for wide rows).  On 148 SMs any cols <= 3542 fits,
 * and a 2048 x 4096 bf16 activation takes 4.6 MiB (296 CTAs).  None when colmax is NULL.  Nothing in the
 * scratch has to start at zero: each CTA writes its whole slice before the reduction reads it.
 * Errors: those of imq_rtn_quantize, plus IMQ_ERR_UNSUPPORTED, returned at once with nothing launched,
 * when the scratch needed exceeds IMQ_NOALLOC_SCRATCH_BYTES.
 * Set-up: the first call on a device looks up the device address of the scratch array for that
 * device (cudaGetSymbolAddress, with that device current); make this first call before any stream
 * capture.  A first call on a device whose stream is capturing returns IMQ_ERR_UNSUPPORTED at once.
 * Concurrency: every call on a device uses the same scratch array, so calls whose executions overlap
 * (on different streams, or from different host threads without ordering) race on it and may return
 * wrong column maxima.  Order them on one stream or with events.
 */
#define IMQ_NOALLOC_SCRATCH_BYTES (8u << 20)
imq_status imq_rtn_quantize_rows_noalloc(const void *X, imq_dtype xt, int64_t rows, int64_t cols,
                                         int64_t ld, double p, int32_t beta, void *Xint, imq_dtype it,
                                         int64_t ldq, float *delta, float *qval, int32_t *rowmax,
                                         int32_t *colmax, imq_stream_t stream);

/* ------------------------------------------------------------------------------------------------ */
/* 2. Unpack plan                                                                                    */
/* ------------------------------------------------------------------------------------------------ */
typedef struct imq_plan imq_plan_t;   /* opaque, owned by the library, freed by imq_plan_destroy */

typedef struct {
  int32_t e;            /* scale exponent of the group: its products are weighted by R^e            */
  int32_t pad_;
  int64_t k_offset;     /* first unpacked inner index of the group (a multiple of IMQ_INNER_PAD)   */
  int64_t k_len;        /* number of real (t, lA, lB) pairs in the group                            */
  int64_t k_len_padded; /* k_len rounded up to IMQ_INNER_PAD                                          */
} imq_group;

typedef struct {
  int32_t b;                 /* unpack bit width                                                   */
  int32_t strategy;          /* imq_strategy the plan was made with                                */
  int32_t dir_a, dir_b;      /* imq_dir chosen for A and B                                         */
  int64_t M, K, N;           /* original GEMM shape                                                */
  int64_t M_unp;             /* rows of the unpacked A' (OUTER: a multiple of IMQ_A_GROUP)         */
  int64_t N_unp;             /* rows of the unpacked B'^T (OUTER: a multiple of IMQ_B_GROUP)       */
  int64_t K_unp;             /* unpacked inner length including padding                           */
  int64_t M_eff, N_eff, K_eff; /* unpadded sizes: sum of row levels, column levels, inner pairs    */
  double  ratio;             /* unpack ratio M_eff*N_eff*K_eff / (M*N*K)  (READING: executed MACs   */
                             /* over original MACs; the page names the metric without a formula)  */
  double  bound;             /* sum_t max_i|A[i,t]| * max_j|B[t,j]|: bounds |C| and every partial  */
                             /* sum of the fold-back (exact below 2^53)                            */
  int32_t acc_bits;          /* 32 when bound < 2^31 (int32 C is exact), else 64                   */
  int32_t n_groups;          /* exponent groups of the inner dimension                             */
  int32_t lmax_a_row, lmax_a_col, lmax_b_row, lmax_b_col;  /* largest level per line kind         */
  int64_t sum_l_a_row, sum_l_a_col, sum_l_b_row, sum_l_b_col; /* sums of levels per line kind       */
  int64_t oor_lines_a_row, oor_lines_a_col, oor_lines_b_row, oor_lines_b_col; /* lines with level>1 */
  size_t  workspace_bytes;   /* device bytes imq_unpacked_gemm needs for A' and B'^T               */
} imq_plan_info;

/*
 * imq_plan -- levels, outlier counts, the direction of each matrix and the unpacked layout
 * ("Approach": row or column unpacking chosen per matrix from outlier counts).
 *
 *   L(v) = 1 if |v| <= R-1, else the number of base-R digits of |v|.
 *   Level of a line = L(max |v| over the line).  A line "holds outliers" when its level is > 1.
 *   Expansion factors: A outer (row unpack) = sum_i L(A row i) / M, A inner (column unpack)
 *   = sum_t L(A col t) / K; B inner (row unpack) = sum_t L(B row t) / K, B outer (column unpack)
 *   = sum_j L(B col j) / N.
 *   Mix (READING of "chosen per matrix via outlier counts"): per matrix, the direction with the
 *   smaller factor; on a tie the one with fewer lines holding outliers; then row unpacking.  A matrix
 *   without any out-of-range entry is not unpacked (IMQ_DIR_NONE).
 *   IMQ_HYBRID: see imq_strategy.  The plan's levels (imq_plan_levels, the lmax / sum_l / oor_lines
 *   fields) are then the levels each line carries in the unpacked GEMM: 1 for an outer line that is
 *   not unpacked OUTER, and inner levels taken over those lines only.
 *
 * A       device, logical M x K.  transA = 0: stored M x K with leading dim lda; transA = 1: stored
 *         K x M (A^T row-major) with leading dim lda.   dtype it (I16 or I32), as written by
 *         imq_rtn_quantize; I32 entries must differ from -2^31 (the quantiser never writes it).
 * B       device, logical K x N.  transB = 0: stored K x N; transB = 1: stored N x K (B^T row-major).
 * a_rowmax, a_colmax, b_rowmax, b_colmax
 *         device or NULL, int32 max |v| per logical line (A rows: M, A cols: K, B rows: K, B cols: N),
 *         e.g. the rowmax/colmax side outputs of imq_rtn_quantize.  When all four are given the plan
 *         skips its own pass over A and B; when any is NULL all four are computed.
 * plan    out: a new plan object.
 * Synchronises the stream once (reads a summary of a few hundred bytes).  Returns any pending device
 * status (e.g. IMQ_ERR_NONFINITE from a preceding quantisation) before planning.
 * IMQ_ERR_UNSUPPORTED: more than IMQ_MAX_GROUPS exponent groups, more than 128 accumulation jobs
 * (groups, split along K where a raw int32 accumulator could overflow), or a bound of 2^63 or more
 * (the product itself may leave int64).
 */
imq_status imq_plan(const void *A, const void *B, imq_dtype it, int64_t M, int64_t K, int64_t N,
                    int32_t transA, int64_t lda, int32_t transB, int64_t ldb,
                    int32_t b, imq_strategy strategy,
                    const int32_t *a_rowmax, const int32_t *a_colmax,
                    const int32_t *b_rowmax, const int32_t *b_colmax,
                    imq_plan_t **plan, imq_stream_t stream);

/* Copies the plan summary to *info (host).  No device work. */
imq_status imq_plan_info_get(const imq_plan_t *plan, imq_plan_info *info);

/* Copies the per-line levels to HOST buffers (int8): a_row[M], a_col[K], b_row[K], b_col[N].
 * Any pointer may be NULL.  Synchronous. */
imq_status imq_plan_levels(const imq_plan_t *plan, int8_t *a_row, int8_t *a_col,
                           int8_t *b_row, int8_t *b_col);

/* Copies the exponent-group table (HOST, up to max_groups entries; *n_out gets the count). */
imq_status imq_plan_groups(const imq_plan_t *plan, imq_group *groups, int32_t max_groups,
                           int32_t *n_out);

/* Copies the plan's index maps of the unpacked operands to HOST buffers (the layout described under
 * imq_unpack), so that a caller can name every byte of A' and B'^T:
 *   tK[K_unp]    source inner index t of unpacked inner position p, -1 on padding
 *   lAk[K_unp]   digit level lA of A at position p;  lBk[K_unp]: digit level lB of B (0 on padding)
 *   srcA[M_unp]  source row of A of unpacked row u, -1 on an unused row;  lvlA[M_unp]: its level l
 *   srcB[N_unp]  source column of B of unpacked row w of B'^T, -1 unused;  lvlB[N_unp]: its level m
 * Byte (u, p) of A' is then digit lvlA[u] + lAk[p] of A[srcA[u], tK[p]] (zero where srcA or tK is -1,
 * and, for a row unpacked both ways by the hybrid, at lAk[p] > 0); likewise for B'^T.  Any pointer
 * may be NULL.  Synchronous; a diagnostic query, not part of the hot path. */
imq_status imq_plan_maps(const imq_plan_t *plan, int32_t *tK, int8_t *lAk, int8_t *lBk, int32_t *srcA,
                         int8_t *lvlA, int32_t *srcB, int8_t *lvlB);

/* Frees the plan and its device arrays.  Call only after work that uses it has finished. */
imq_status imq_plan_destroy(imq_plan_t *plan);

/* ------------------------------------------------------------------------------------------------ */
/* 3. Unpack and low-bit GEMM                                                                        */
/* ------------------------------------------------------------------------------------------------ */
/*
 * imq_unpack -- digit split of A and B into b-bit integers stored as int8 ("Approach": out-of-range
 * entries become several in-range entries by row or column unpacking).
 *   digit d_l(v) = sgn(v) * ((|v| >> (l*(b-1))) & (R-1)), so sum_l R^l d_l(v) = v and |d_l| <= R-1.
 * Layout (READING: the page fixes no operand order; this one is the library's):
 *   inner index p enumerates pairs (t, lA, lB) with lA < la_t, lB < lb_t (la_t = level of A column t
 *   when A is INNER else 1, lb_t = level of B row t when B is INNER else 1), ordered by exponent
 *   e = lA + lB, then lA, then t -- or, in a plan that groups the inner indices by class, by the class
 *   (la_t, lb_t) in descending order (la_t first) and then t; each exponent group padded with zeros to
 *   IMQ_INNER_PAD.  (Grouping by class makes each (lA, lB) segment a few ranges of one fixed order of
 *   the inner indices, in which the unpack kernels stage a source line, so that most 16-position blocks
 *   are runs of consecutive staged entries; the plan groups when index order would leave many blocks
 *   scattered.  imq_plan_maps gives the order a plan took.)
 *   OUTER rows of A: source rows sorted by level L (stable), floor(IMQ_A_GROUP / L) source rows per
 *   group of IMQ_A_GROUP unpacked rows, lines (source, level) consecutive, unused rows zero.
 *   OUTER columns of B: the same with IMQ_B_GROUP.
 *   IMQ_DIR_BOTH (hybrid): a source row of A unpacked OUTER (level above 1) has all its digits on its
 *   own lines and zeros at the inner pairs with lA > 0; the other rows are single lines with the
 *   digits of every pair; likewise for the columns of B with lB > 0.
 * A_unp   device int8, M_unp x K_unp row-major (K contiguous), written in full.
 * B_unp_t device int8, N_unp x K_unp row-major (K contiguous, i.e. B'^T), written in full.
 * A, B must be the matrices (same pointers and layouts) the plan was made from.  Asynchronous.
 */
imq_status imq_unpack(const imq_plan_t *plan, const void *A, const void *B,
                      int8_t *A_unp, int8_t *B_unp_t, imq_stream_t stream);

/*
 * imq_rtn_quantize_unpack -- per-row RTN of X fused with its unpacking into the A' layout of an existing
 * plan, for inference with a weight that is quantised, planned and unpacked once (B'^T kept by the
 * caller) while the activations change ("Approach" and "Key results": quantised linear layers at
 * inference; the page does not describe caching, this is the library's way of not re-unpacking a
 * static weight).  The integer activations are never written to memory: one warp per row stages the
 * row, selects its percentile, quantises it (exactly as imq_rtn_quantize with IMQ_PER_ROW and I16
 * output) in shared memory and writes the row's unpacked line.
 *   Coverage: the plan stays valid for X when every quantised entry satisfies |x_int[i,t]| <= the
 *   maximum |A[:, t]| the plan was made from (its a_colmax, or the column maxima of its A): the
 *   levels, the inner layout and the accumulator bound then all hold and imq_gemm_unpacked with the
 *   kept B'^T gives X_int * B exactly.  A larger entry sets IMQ_ERR_PLAN in the device status word;
 *   the caller then plans again.  To cover later batches, plan with widened column maxima (any values
 *   >= the true ones; the plan's levels and bound follow the maxima it is given).
 * plan    a plan whose A is INNER or not unpacked (imq_plan_info.dir_a of IMQ_DIR_INNER or
 *         IMQ_DIR_NONE; OUTER rows would depend on the new values): IMQ_ERR_ARG otherwise.  Its M x K
 *         is X's shape.
 * X       device, M x K row-major with leading dimension ld (>= K), dtype xt (F32 or BF16).
 * A_unp   device int8, M_unp (= M) x K_unp, 16-byte aligned, written in full.
 * deltaA  device fp32[M]: the dequantisation step of every row.
 * Errors: IMQ_ERR_ARG at once; IMQ_ERR_NONFINITE, IMQ_ERR_RANGE (an entry above 32767), IMQ_ERR_PLAN
 *         through the device status word.  IMQ_ERR_UNSUPPORTED when a row (input and int16 copy) does
 *         not fit in shared memory (K above about 33 000 for F32 input, 50 000 for BF16).
 *         Asynchronous; allocates nothing.
 */
imq_status imq_rtn_quantize_unpack(const imq_plan_t *plan, const void *X, imq_dtype xt, int64_t ld,
                                   double p, int32_t beta, int8_t *A_unp, float *deltaA,
                                   imq_stream_t stream);

/*
 * imq_level_cover -- out[i] = min(R^L - 1, cap), L the level of maxima[i] (its number of base-R digits,
 * R = 2^(b-1)): the largest magnitude with as many digits.  For a plan kept with an unpacked weight
 * (imq_rtn_quantize_unpack): planned with A's column maxima raised this way, the plan covers every later
 * activation whose entries need no more digits than the one it was made from, since levels, layout and
 * the bound only depend on the maxima the plan is given ("Approach": the digit count decides how many
 * lines an entry takes).  maxima, out: device int32[n] (they may alias).  cap >= 0 (32767 for int16
 * activations).  Asynchronous.
 */
imq_status imq_level_cover(const int32_t *maxima, int64_t n, int32_t b, int32_t cap, int32_t *out,
                           imq_stream_t stream);

/*
 * imq_gemm_unpacked -- the low-bit GEMM on already unpacked operands with the fold-back epilogue:
 *   C = sum over exponent groups e of R^e * (A'_e * B'_e), every OUTER line folded back with its level
 *   weight R^l ("Approach": bit-shift scaling and accumulation reproduce the integer product
 *   exactly).  s8 x s8 -> s32 products run on the tcgen05 tensor cores, one int32 tensor-memory
 *   accumulator per exponent group (the plan splits a group along K if that could overflow); the
 *   epilogue shifts each group into C.  Every partial sum is bounded by the plan's bound, so int32
 *   is exact when acc_bits == 32 and int64 otherwise.
 *   Cf[i,j] = (float)C[i,j] * (deltaA[i] * deltaB[j])  (fp32; READING: the page implies dequantised
 *   outputs but gives no formula).
 * deltaA  device fp32: 1 value (gA = IMQ_PER_TENSOR) or M values (IMQ_PER_ROW: one per row of A).
 * deltaB  device fp32: 1 value (IMQ_PER_TENSOR) or N values (IMQ_PER_COL: one per column of B).
 *         Both may be NULL when Cf is NULL.
 * Cint    device or NULL, M x N, leading dim ldc, dtype ct (I32 or I64).  I32 with
 *         plan acc_bits == 64 returns IMQ_ERR_RANGE.  When the plan has more than one exponent group
 *         the groups accumulate in Cint, so it must be given (IMQ_ERR_ARG otherwise).
 * Cf      device or NULL, fp32 M x N, leading dim ldcf.
 * Asynchronous.
 */
imq_status imq_gemm_unpacked(const imq_plan_t *plan, const int8_t *A_unp, const int8_t *B_unp_t,
                             const float *deltaA, imq_gran gA, const float *deltaB, imq_gran gB,
                             void *Cint, imq_dtype ct, int64_t ldc, float *Cf, int64_t ldcf,
                             imq_stream_t stream);

/*
 * imq_unpacked_gemm -- imq_unpack into the caller's workspace followed by imq_gemm_unpacked.
 * workspace  device, at least imq_plan_info.workspace_bytes bytes, 1024-byte aligned.
 */
imq_status imq_unpacked_gemm(const imq_plan_t *plan, const void *A, const void *B,
                             const float *deltaA, imq_gran gA, const float *deltaB, imq_gran gB,
                             void *Cint, imq_dtype ct, int64_t ldc, float *Cf, int64_t ldcf,
                             void *workspace, size_t workspace_bytes, imq_stream_t stream);

/*
 * imq_plan_unpack -- imq_plan followed, in the same host call, by imq_unpack into the caller's workspace
 * (the plan and unpack steps of "Approach" without a return to the caller in between: the unpack is
 * queued right behind the plan's last kernel).  Arguments as imq_plan, plus:
 * workspace  device, 1024-byte aligned, workspace_bytes long; A' = workspace[0 .. M_unp*K_unp) and
 *            B'^T from the next 1024-byte boundary (the layout imq_unpacked_gemm uses), so the caller
 *            passes those two pointers to imq_gemm_unpacked.
 * Errors: those of imq_plan and imq_unpack.  IMQ_ERR_BUFFER when workspace_bytes is below the plan's
 *         workspace_bytes (or workspace is NULL): *plan is then a valid plan (destroy it as usual) and
 *         nothing was unpacked; the caller may allocate imq_plan_info.workspace_bytes and call
 *         imq_unpack.  IMQ_ERR_ARG for a misaligned workspace.  Synchronises like imq_plan.
 */
imq_status imq_plan_unpack(const void *A, const void *B, imq_dtype it, int64_t M, int64_t K, int64_t N,
                           int32_t transA, int64_t lda, int32_t transB, int64_t ldb, int32_t b,
                           imq_strategy strategy, const int32_t *a_rowmax, const int32_t *a_colmax,
                           const int32_t *b_rowmax, const int32_t *b_colmax, void *workspace,
                           size_t workspace_bytes, imq_plan_t **plan, imq_stream_t stream);

/* ------------------------------------------------------------------------------------------------ */
/* 4. Batches of equal-shaped GEMMs (attention heads)                                                */
/* ------------------------------------------------------------------------------------------------ */
/*
 * The page singles out the attention GEMMs: its "Key results" quote an unpack ratio of about 3-4x for
 * attention-output GEMMs at 5 bits, and its "Limitations" name the self-attention matrix, whose outliers
 * sit on the diagonal, as the case unpacking handles worst.  One attention layer is many small GEMMs of
 * one shape (one per head), each needing its own plan: the calls below plan, unpack and multiply such a
 * batch with one host round trip for all the plans, one unpack launch per operand and one GEMM launch
 * whose tile scheduler runs the tiles of every problem (as few as the problem table allows: 64 problems
 * per launch).  Problem h reads A + h * strideA and B + h * strideB (in elements of the integer dtype)
 * with the leading dimensions lda, ldb; every problem is planned separately (its own levels, directions
 * and layout), exactly as imq_plan would plan it alone.
 */

/*
 * imq_plan_batched -- `batch` plans, plans[h] for problem h (HOST array of batch handles, each freed
 * with imq_plan_destroy).  Arguments as imq_plan; the four line-maxima vectors, when all are given,
 * hold batch consecutive vectors (problem h's a_rowmax at a_rowmax + h * M, a_colmax at + h * K,
 * b_rowmax at + h * K, b_colmax at + h * N); when any is NULL each plan computes its own.  Synchronises
 * once for the whole batch.  Every plan is made as by imq_plan.  Up to 256 plans (except with
 * IMQ_HYBRID) share their device launches: one per kind of plan kernel for the whole batch.  Larger
 * batches queue each plan's kernels in turn.  On an error no plan is returned (every entry of plans is
 * NULL).
 */
imq_status imq_plan_batched(int32_t batch, const void *A, int64_t strideA, const void *B, int64_t strideB,
                            imq_dtype it, int64_t M, int64_t K, int64_t N, int32_t transA, int64_t lda,
                            int32_t transB, int64_t ldb, int32_t b, imq_strategy strategy,
                            const int32_t *a_rowmax, const int32_t *a_colmax, const int32_t *b_rowmax,
                            const int32_t *b_colmax, imq_plan_t **plans, imq_stream_t stream);

/*
 * imq_batch_workspace -- the device workspace a batch needs (*total_bytes) and, when offsets (HOST,
 * 2 * batch entries) is given, where each operand lies in it: problem h's A' at offsets[2h] and its B'^T
 * at offsets[2h + 1], each from a 1024-byte boundary (the workspace itself 1024-byte aligned).
 */
imq_status imq_batch_workspace(int32_t batch, imq_plan_t *const *plans, size_t *offsets, size_t *total_bytes);

/* imq_unpack_batched -- imq_unpack of every problem of a batch planned by one imq_plan_batched call, into
 * the workspace layout of imq_batch_workspace.  A, B, strides: those the plans were made from.
 * IMQ_ERR_BUFFER when workspace_bytes is below the batch's need; IMQ_ERR_ARG for plans of different
 * shapes, layouts or b.  Asynchronous. */
imq_status imq_unpack_batched(int32_t batch, imq_plan_t *const *plans, const void *A, int64_t strideA,
                              const void *B, int64_t strideB, void *workspace, size_t workspace_bytes,
                              imq_stream_t stream);

/* imq_gemm_unpacked_batched -- imq_gemm_unpacked of every problem of the batch from the unpacked operands
 * in the workspace: problem h uses deltaA + h * strideDA, deltaB + h * strideDB (each NULL when Cf is
 * NULL), writes C at Cint + h * strideC and Cf at Cf + h * strideCf (strides in elements of C's dtype
 * and of fp32; leading dimensions ldc, ldcf).  Errors as imq_gemm_unpacked.  Asynchronous. */
imq_status imq_gemm_unpacked_batched(int32_t batch, imq_plan_t *const *plans, const void *workspace,
                                     size_t workspace_bytes, const float *deltaA, int64_t strideDA,
                                     imq_gran gA, const float *deltaB, int64_t strideDB, imq_gran gB,
                                     void *Cint, int64_t strideC, imq_dtype ct, int64_t ldc, float *Cf,
                                     int64_t strideCf, int64_t ldcf, imq_stream_t stream);

/* imq_unpacked_gemm_batched -- imq_unpack_batched followed by imq_gemm_unpacked_batched. */
imq_status imq_unpacked_gemm_batched(int32_t batch, imq_plan_t *const *plans, const void *A, int64_t strideA,
                                     const void *B, int64_t strideB, const float *deltaA, int64_t strideDA,
                                     imq_gran gA, const float *deltaB, int64_t strideDB, imq_gran gB,
                                     void *Cint, int64_t strideC, imq_dtype ct, int64_t ldc, float *Cf,
                                     int64_t strideCf, int64_t ldcf, void *workspace, size_t workspace_bytes,
                                     imq_stream_t stream);

/* ------------------------------------------------------------------------------------------------ */
/* Status                                                                                            */
/* ------------------------------------------------------------------------------------------------ */
/* Synchronises the stream, returns the device status word of the current device and, when clear is
 * non-zero, resets it to IMQ_OK. */
imq_status imq_device_status(imq_stream_t stream, int32_t clear);

/* Diagnostic, no counterpart on the page: launches one kernel whose bounded wait (the one every wait of
 * the GEMM goes through) waits on an mbarrier that nothing arrives at, so it gives up after timeout_ns
 * (1 us .. 1 s, else IMQ_ERR_ARG) and records IMQ_ERR_TIMEOUT in the device status word.  It shows that
 * a stalled wait ends the kernel with a status the host reads and leaves the context usable.
 * Asynchronous. */
imq_status imq_check_bounded_wait(uint64_t timeout_ns, imq_stream_t stream);

/* Static, never NULL. */
const char *imq_status_str(imq_status s);

#ifdef __cplusplus
}
#endif
#endif /* IMQ_H */
