/*
 * plan.c -- oracle step 3-4 and the unpacked layout: levels, outlier counts, the per-matrix direction
 * (the Mix strategy or a fixed one), the unpack ratio and the index maps of the unpacked operands.
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * IM-Unpack summary page:
 *   "Approach"  -- rows or columns that hold out-of-bound entries are unpacked; the choice between row
 *                  and column unpacking is made per matrix from outlier counts.
 *   measured-effects table -- the Mix strategy against fixed row/row, row/col, col/row and col/col
 *                  unpacking, compared by unpack ratio (beta = 15, b = 5).
 *   "Experimental setup" -- the unpack ratio is one of the reported metrics (no formula given).
 * READINGs (the page gives no formulas):
 *   level of a line = number of base-R digits of its largest |entry|; it "holds outliers" if > 1.
 *   expansion factor of a direction = mean level of the lines unpacked in that direction.
 *   Mix: per matrix the smaller factor; tie -> fewer lines holding outliers; tie -> row unpacking;
 *        a matrix without any out-of-range entry is not unpacked.
 *   unpack ratio = M_eff * N_eff * K_eff / (M * N * K): executed multiply-adds over original ones.
 *   Hybrid ("unpack both", for matrices whose heavy hitters sit in some rows AND some columns): per
 *        matrix, the outer lines (rows of A, columns of B) holding at least tau out-of-range entries are
 *        unpacked OUTER with all their digits, the remaining lines INNER, the inner levels taken over
 *        those remaining lines only; tau is the threshold of least M_eff * K_eff (A) or N_eff * K_eff (B),
 *        the smallest such tau on a tie; the direction is then OUTER, INNER or both (OR_DIR_BOTH).  The
 *        level vectors the plan returns are then the levels each line carries in the unpacked GEMM.
 *   the unpacked operands have no memory layout here: an unpacked line of A is a pair (row i, level l),
 *   l < the level row i carries when A is unpacked OUTER (else l = 0 only); an unpacked line of B is a
 *   pair (column j, level m) likewise; an unpacked inner index is a triple (t, lA, lB), lA < the level
 *   of A's column t when A is unpacked INNER (else 0 only), lB < the level of B's row t when B is
 *   unpacked INNER (else 0 only).  oracle_unpack_lines lists them in lexicographic order, which is a
 *   naming, not a layout: every check against a kernel matches entries by these pairs and triples.
 */
#include <stdlib.h>
#include <string.h>
#include "oracle.h"

static int64_t iabs64(int64_t v) { return v < 0 ? -v : v; }

/* Li[t] = the largest level of entry t over the outer lines with fewer than tau out-of-range entries
 * (1 when there is none); lev is n_out x n_in, row by row. */
static void inner_levels(const int8_t *lev, const int64_t *cnt, int64_t n_out, int64_t n_in, int64_t tau,
                         int32_t *Li) {
  for (int64_t t = 0; t < n_in; ++t) Li[t] = 1;
  for (int64_t o = 0; o < n_out; ++o) {
    if (cnt[o] >= tau) continue;
    for (int64_t t = 0; t < n_in; ++t)
      if (lev[o * n_in + t] > Li[t]) Li[t] = lev[o * n_in + t];
  }
}

/* The hybrid choice for one matrix seen as n_out outer lines of n_in inner entries, entry (o, t) at
 * X[o * s_out + t * s_in].  On entry Lo holds the outer lines' levels; on exit Lo and Li hold the levels
 * each line carries: Lo[o] unchanged for a line unpacked OUTER (its out-of-range count >= tau), else 1;
 * Li[t] the largest level of entry t over the lines that are not (1 when there is none). */
static int hybrid_choose(const int64_t *X, int64_t n_out, int64_t n_in, int64_t s_out, int64_t s_in, int b,
                         int32_t *Lo, int32_t *Li) {
  int8_t *lev = malloc((size_t)(n_out * n_in > 0 ? n_out * n_in : 1));
  int64_t *cnt = calloc((size_t)(n_out > 0 ? n_out : 1), sizeof(int64_t));
  char *present = calloc((size_t)(n_in + 2), 1);
  if (!lev || !cnt || !present) {
    free(lev);
    free(cnt);
    free(present);
    return OR_ERR_ARG;
  }
  int64_t cmax = 0;
  for (int64_t o = 0; o < n_out; ++o) {
    for (int64_t t = 0; t < n_in; ++t) {
      lev[o * n_in + t] = (int8_t)oracle_level(X[o * s_out + t * s_in], b);
      if (lev[o * n_in + t] > 1) cnt[o] += 1;
    }
    present[cnt[o]] = 1;
    if (cnt[o] > cmax) cmax = cnt[o];
  }
  /* every threshold at which the set of OUTER lines changes, and one above all counts (no OUTER line) */
  int64_t best_tau = 1;
  unsigned __int128 best = 0;
  int first = 1;
  for (int64_t tau = 1; tau <= cmax + 1; ++tau) {
    if (!(tau == cmax + 1 || present[tau])) continue;
    unsigned __int128 me = 0, ke = 0;
    for (int64_t o = 0; o < n_out; ++o) me += (unsigned)(cnt[o] >= tau ? Lo[o] : 1);
    inner_levels(lev, cnt, n_out, n_in, tau, Li);
    for (int64_t t = 0; t < n_in; ++t) ke += (unsigned)Li[t];
    const unsigned __int128 cost = me * ke;
    if (first || cost < best) {
      best = cost;
      best_tau = tau;
      first = 0;
    }
  }
  inner_levels(lev, cnt, n_out, n_in, best_tau, Li);
  for (int64_t o = 0; o < n_out; ++o)
    if (cnt[o] < best_tau) Lo[o] = 1;
  free(lev);
  free(cnt);
  free(present);
  return OR_OK;
}

int oracle_plan(const int64_t *A, const int64_t *B, int64_t M, int64_t K, int64_t N, int b,
                int strategy, int32_t *LrA, int32_t *LcA, int32_t *LrB, int32_t *LcB,
                oracle_plan_t *out) {
  if (b < 2 || b > 8 || M < 0 || K < 0 || N < 0 || strategy < 0 || strategy > 6) return OR_ERR_ARG;
  memset(out, 0, sizeof(*out));
  out->b = b;
  out->strategy = strategy;
  out->M = M;
  out->K = K;
  out->N = N;

  /* levels of every line */
  for (int64_t i = 0; i < M; ++i) LrA[i] = 1;
  for (int64_t t = 0; t < K; ++t) { LcA[t] = 1; LrB[t] = 1; }
  for (int64_t j = 0; j < N; ++j) LcB[j] = 1;
  for (int64_t i = 0; i < M; ++i)
    for (int64_t t = 0; t < K; ++t) {
      int l = oracle_level(A[i * K + t], b);
      if (l > LrA[i]) LrA[i] = l;
      if (l > LcA[t]) LcA[t] = l;
    }
  for (int64_t t = 0; t < K; ++t)
    for (int64_t j = 0; j < N; ++j) {
      int l = oracle_level(B[t * N + j], b);
      if (l > LrB[t]) LrB[t] = l;
      if (l > LcB[j]) LcB[j] = l;
    }
  if (strategy == OR_HYBRID) {
    /* A: rows outer, columns inner; B: columns outer (entry (j, t) at B[t * N + j]), rows inner */
    if (hybrid_choose(A, M, K, K, 1, b, LrA, LcA) != OR_OK) return OR_ERR_ARG;
    if (hybrid_choose(B, N, K, 1, N, b, LcB, LrB) != OR_OK) return OR_ERR_ARG;
  }
  const int32_t *vecs[4] = {LrA, LcA, LrB, LcB};
  const int64_t lens[4] = {M, K, K, N};
  for (int v = 0; v < 4; ++v) {
    out->lmax[v] = 1;
    for (int64_t x = 0; x < lens[v]; ++x) {
      out->suml[v] += vecs[v][x];
      if (vecs[v][x] > 1) out->oor_lines[v] += 1;
      if (vecs[v][x] > out->lmax[v]) out->lmax[v] = vecs[v][x];
    }
  }

  /* direction of each matrix */
  int da, db;
  if (strategy == OR_MIX || strategy == OR_MIX_JOINT) {
    if (out->oor_lines[0] == 0 && out->oor_lines[1] == 0) {
      da = OR_DIR_NONE;
    } else {
      /* row factor suml[0]/M against column factor suml[1]/K, compared exactly */
      int64_t row_side = out->suml[0] * K, col_side = out->suml[1] * M;
      if (row_side < col_side) da = OR_DIR_OUTER;
      else if (row_side > col_side) da = OR_DIR_INNER;
      else if (out->oor_lines[0] < out->oor_lines[1]) da = OR_DIR_OUTER;
      else if (out->oor_lines[0] > out->oor_lines[1]) da = OR_DIR_INNER;
      else da = OR_DIR_OUTER;
    }
    if (out->oor_lines[2] == 0 && out->oor_lines[3] == 0) {
      db = OR_DIR_NONE;
    } else {
      /* row factor suml[2]/K against column factor suml[3]/N */
      int64_t row_side = out->suml[2] * N, col_side = out->suml[3] * K;
      if (row_side < col_side) db = OR_DIR_INNER;
      else if (row_side > col_side) db = OR_DIR_OUTER;
      else if (out->oor_lines[2] < out->oor_lines[3]) db = OR_DIR_INNER;
      else if (out->oor_lines[2] > out->oor_lines[3]) db = OR_DIR_OUTER;
      else db = OR_DIR_INNER;
    }
  } else if (strategy == OR_HYBRID) {
    /* the levels above are already those of the hybrid choice */
    da = (out->oor_lines[0] ? OR_DIR_OUTER : 0) | (out->oor_lines[1] ? OR_DIR_INNER : 0);
    db = (out->oor_lines[3] ? OR_DIR_OUTER : 0) | (out->oor_lines[2] ? OR_DIR_INNER : 0);
  } else {
    da = (strategy == OR_ROW_ROW || strategy == OR_ROW_COL) ? OR_DIR_OUTER : OR_DIR_INNER;
    db = (strategy == OR_ROW_ROW || strategy == OR_COL_ROW) ? OR_DIR_INNER : OR_DIR_OUTER;
  }
  if (strategy == OR_MIX_JOINT) {
    /* Joint Mix: starting from the per-matrix Mix choice above, take the direction pair whose exact
     * unpacked size M_eff * N_eff * K_eff is strictly smaller, trying the pairs in the order
     * row/row, row/col, col/row, col/col (A's direction / B's).  A matrix without out-of-range entries
     * stays not unpacked (its size factors are 1 either way). */
    const int pa[4] = {OR_DIR_OUTER, OR_DIR_OUTER, OR_DIR_INNER, OR_DIR_INNER};
    const int pb[4] = {OR_DIR_INNER, OR_DIR_OUTER, OR_DIR_INNER, OR_DIR_OUTER};
    unsigned __int128 best = 0;
    for (int c = -1; c < 4; ++c) {
      const int ca = c < 0 ? da : (da == OR_DIR_NONE ? OR_DIR_NONE : pa[c]);
      const int cb = c < 0 ? db : (db == OR_DIR_NONE ? OR_DIR_NONE : pb[c]);
      unsigned __int128 me = 0, ne = 0, ke = 0;
      for (int64_t i = 0; i < M; ++i) me += (ca == OR_DIR_OUTER) ? (unsigned)LrA[i] : 1u;
      for (int64_t j = 0; j < N; ++j) ne += (cb == OR_DIR_OUTER) ? (unsigned)LcB[j] : 1u;
      for (int64_t t = 0; t < K; ++t)
        ke += (unsigned __int128)((ca == OR_DIR_INNER) ? LcA[t] : 1) * (unsigned)((cb == OR_DIR_INNER) ? LrB[t] : 1);
      const unsigned __int128 cost = me * ne * ke;
      if (c < 0 || cost < best) {
        best = cost;
        da = ca;
        db = cb;
      }
    }
  }
  out->dir_a = da;
  out->dir_b = db;

  /* levels each index carries in the unpacked GEMM */
  out->M_eff = 0;
  for (int64_t i = 0; i < M; ++i) out->M_eff += (da & OR_DIR_OUTER) ? LrA[i] : 1;
  out->N_eff = 0;
  for (int64_t j = 0; j < N; ++j) out->N_eff += (db & OR_DIR_OUTER) ? LcB[j] : 1;
  int maxla = (da & OR_DIR_INNER) ? out->lmax[1] : 1;
  int maxlb = (db & OR_DIR_INNER) ? out->lmax[2] : 1;
  out->K_eff = 0;
  for (int64_t t = 0; t < K; ++t) {
    int64_t la = (da & OR_DIR_INNER) ? LcA[t] : 1;
    int64_t lb = (db & OR_DIR_INNER) ? LrB[t] : 1;
    out->K_eff += la * lb;
  }
  if (M > 0 && N > 0 && K > 0)
    out->ratio = ((double)out->M_eff / (double)M) * ((double)out->N_eff / (double)N) *
                 ((double)out->K_eff / (double)K);
  else
    out->ratio = 1.0;

  /* exponents of the inner triples: e = lA + lB, with the number of triples carrying each */
  int ng = 0;
  for (int e = 0; e <= maxla + maxlb - 2; ++e) {
    int64_t len = 0;
    for (int64_t t = 0; t < K; ++t) {
      const int64_t a = (da & OR_DIR_INNER) ? LcA[t] : 1;
      const int64_t bb = (db & OR_DIR_INNER) ? LrB[t] : 1;
      for (int la = 0; la < a; ++la)
        if (e - la >= 0 && e - la < bb) len += 1;
    }
    if (len == 0) continue;
    if (ng >= OR_MAX_GROUPS) return OR_ERR_ARG;
    out->group_e[ng] = e;
    out->group_len[ng] = len;
    ng += 1;
  }
  out->n_groups = ng;

  /* bound on |C| and on every partial sum of the fold-back */
  __int128 bound = 0;
  for (int64_t t = 0; t < K; ++t) {
    int64_t ma = 0, mb = 0;
    for (int64_t i = 0; i < M; ++i)
      if (iabs64(A[i * K + t]) > ma) ma = iabs64(A[i * K + t]);
    for (int64_t j = 0; j < N; ++j)
      if (iabs64(B[t * N + j]) > mb) mb = iabs64(B[t * N + j]);
    bound += (__int128)ma * (__int128)mb;
  }
  out->bound = (double)bound;
  out->bound_lt_2_31 = bound < ((__int128)1 << 31);
  return OR_OK;
}

/* The unpacked lines and inner triples of a plan, in lexicographic order (see the top of this file):
 * a_lines[2u], a_lines[2u+1] = (i, l) for u < M_eff; b_lines[2w], b_lines[2w+1] = (j, m) for w < N_eff;
 * pairs[3p .. 3p+2] = (t, lA, lB) for p < K_eff.  The level vectors are those oracle_plan returned. */
int oracle_unpack_lines(const oracle_plan_t *pl, const int32_t *LrA, const int32_t *LcA,
                        const int32_t *LrB, const int32_t *LcB, int32_t *a_lines, int32_t *b_lines,
                        int32_t *pairs) {
  const int da = pl->dir_a, db = pl->dir_b;
  int64_t u = 0;
  for (int64_t i = 0; i < pl->M; ++i) {
    const int L = (da & OR_DIR_OUTER) ? LrA[i] : 1;
    for (int l = 0; l < L; ++l) {
      a_lines[2 * u] = (int32_t)i;
      a_lines[2 * u + 1] = l;
      u += 1;
    }
  }
  if (u != pl->M_eff) return OR_ERR_ARG;
  int64_t w = 0;
  for (int64_t j = 0; j < pl->N; ++j) {
    const int L = (db & OR_DIR_OUTER) ? LcB[j] : 1;
    for (int m = 0; m < L; ++m) {
      b_lines[2 * w] = (int32_t)j;
      b_lines[2 * w + 1] = m;
      w += 1;
    }
  }
  if (w != pl->N_eff) return OR_ERR_ARG;
  int64_t p = 0;
  for (int64_t t = 0; t < pl->K; ++t) {
    const int la = (da & OR_DIR_INNER) ? LcA[t] : 1;
    const int lb = (db & OR_DIR_INNER) ? LrB[t] : 1;
    for (int x = 0; x < la; ++x)
      for (int y = 0; y < lb; ++y) {
        pairs[3 * p] = (int32_t)t;
        pairs[3 * p + 1] = x;
        pairs[3 * p + 2] = y;
        p += 1;
      }
  }
  if (p != pl->K_eff) return OR_ERR_ARG;
  return OR_OK;
}
