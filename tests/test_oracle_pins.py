"""CPU pins of the oracle against facts that do not come from the oracle itself.

Each test names what fixes the expected value: sorting / counting (percentile), exact rational
arithmetic (rounding, dequantisation), the defining properties of sign-magnitude base-R digits,
brute-force integer products, closed forms of the unpack ratio, and the Mix rule re-derived from the
line levels.  Method source: "IM-Unpack: Training and Inference with Arbitrarily Low Precision
Integers" (atlas.scime.ai summary): "Approach", "Problem", measured-effects table.
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads

BF16_FINITE = None


def _all_finite_bf16():
    global BF16_FINITE
    if BF16_FINITE is None:
        bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
        exp = (bits >> 7) & 0xFF
        BF16_FINITE = bits[exp != 0xFF]
    return BF16_FINITE


# ------------------------------------------------------------------------------------------------
# percentile (measured-effects table: p = 95% default, p = 100% ablation)
# ------------------------------------------------------------------------------------------------
def _rank_by_counting(v, p):
    """Smallest |x| such that at least ceil(p*n) values are <= it (nearest-rank, by counting)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    k = oracle.nearest_rank(a.size, p)
    for c in sorted(set(a.tolist())):
        if (a <= c).sum() >= k:
            return c
    raise AssertionError


@pytest.mark.parametrize("p", [0.01, 0.5, 0.95, 0.999, 1.0])
def test_percentile_matches_counting_definition(p):
    rng = np.random.default_rng(11)
    for n in (1, 2, 3, 7, 20, 101):
        v = rng.standard_normal(n).astype(np.float32) * np.float32(rng.uniform(0.1, 100))
        assert float(oracle.percentile_abs(v, p)) == _rank_by_counting(v, p)


def test_percentile_order_invariant_bruteforce():
    rng = np.random.default_rng(12)
    for _ in range(20):
        n = int(rng.integers(1, 7))
        v = (rng.integers(-4, 5, size=n)).astype(np.float32)  # many ties
        p = float(rng.choice([0.2, 0.5, 0.95, 1.0]))
        want = _rank_by_counting(v, p)
        for perm in itertools.permutations(range(n)):
            assert float(oracle.percentile_abs(v[list(perm)], p)) == want


def test_percentile_p1_is_max_and_ranks_of_configs():
    rng = np.random.default_rng(13)
    v = rng.standard_normal(1000).astype(np.float32)
    assert oracle.percentile_abs(v, 1.0) == np.abs(v).max()
    # ranks k = ceil(0.95 n) for the group sizes of the workloads (nearest rank, double arithmetic)
    want = {128: 122, 2048: 1946, 4096: 3892, 8192: 7783, 11008: 10458,
            8388608: 7969178, 33554432: 31876711}
    for n, k in want.items():
        assert oracle.nearest_rank(n, 0.95) == k


# ------------------------------------------------------------------------------------------------
# RTN ("Problem"/"Approach": heavy hitters kept, not clipped)
# ------------------------------------------------------------------------------------------------
def _rne_int(fr: Fraction) -> int:
    """Round a rational to the nearest integer, ties to even, in exact arithmetic."""
    fl = math.floor(fr)
    rem = fr - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def test_rtn_exhaustive_bf16_against_exact_rounding():
    bits = _all_finite_bf16()
    x = oracle.bf16_bits_to_f32(bits).reshape(1, -1)
    for beta in (15, 31, 255):
        xint, delta, q = oracle.rtn_quantize(x, oracle.PER_TENSOR, 0.95, beta)
        s = np.float32(beta) / np.float32(q[0])  # IEEE fp32 division, correctly rounded
        # a bf16 value has 8 significant bits and s 24, so x*s is exact in float64; casting that
        # float64 to float32 is the single correct rounding of the fp32 product
        prod32 = (x.astype(np.float64) * np.float64(s)).astype(np.float32)
        want = np.array([_rne_int(Fraction(float(v))) for v in prod32.ravel()], dtype=np.int64)
        assert np.array_equal(xint.ravel(), want)
        assert delta[0] == np.float32(q[0]) / np.float32(beta)


def test_rtn_rank_k_maps_to_beta_and_sign_symmetry():
    g = workloads.q_proj()[0]
    X = oracle.as_f32(g.A.data[:64], "bf16")
    for beta in (15, 31):
        xint, delta, q = oracle.rtn_quantize(X, oracle.PER_ROW, 0.95, beta)
        n = X.shape[1]
        k = oracle.nearest_rank(n, 0.95)
        for r in range(X.shape[0]):
            row = X[r]
            idx = np.flatnonzero(np.abs(row) == q[r])
            assert idx.size > 0, "q must be an element of the group"
            assert np.all(np.abs(xint[r, idx]) == beta)
            assert (np.abs(xint[r]) <= beta).sum() >= k
        # heavy hitters are not clipped: the x60 channels exceed beta
        assert np.abs(xint).max() > 10 * beta
        xneg, dneg, qneg = oracle.rtn_quantize(-X, oracle.PER_ROW, 0.95, beta)
        assert np.array_equal(xneg, -xint) and np.array_equal(dneg, delta)


def test_rtn_clip_exhaustive_bf16_against_exact_rounding():
    """Clipping variant (the measured-effects table's 99.5% row): the exactly rounded fp32 product,
    clamped to [-beta, beta] (clamping before or after rounding agree since beta is an integer)."""
    bits = _all_finite_bf16()
    x = oracle.bf16_bits_to_f32(bits).reshape(1, -1)
    for beta in (15, 255):
        xint, delta, q = oracle.rtn_quantize(x, oracle.PER_TENSOR, 0.995, beta, clip=True)
        s = np.float32(beta) / np.float32(q[0])
        prod32 = (x.astype(np.float64) * np.float64(s)).astype(np.float32)
        want = np.array([max(-beta, min(beta, _rne_int(Fraction(float(v))))) for v in prod32.ravel()],
                        dtype=np.int64)
        assert np.array_equal(xint.ravel(), want)
        # the scale is the unclipped one: clipping only changes the heavy hitters
        _, d0, q0 = oracle.rtn_quantize(x, oracle.PER_TENSOR, 0.995, beta)
        assert d0[0] == delta[0] and q0[0] == q[0]


def test_rtn_variants_error_ordering():
    """The comparison the measured-effects table draws, on heavy-hitter data with an exact float64
    reference product: keeping heavy hitters (the method, p = 95 %, beta = 15) loses far less than
    clipping them at the 99.5 % point, and the unpacked product of the method is the exact product
    of its integers (so its only error is the rounding of RTN)."""
    g = workloads.q_proj()[0]
    X = oracle.as_f32(g.A.data[:96], "bf16")
    W = oracle.as_f32(g.B.data[:, :80], "bf16")
    ref = X.astype(np.float64) @ W.astype(np.float64)

    def err(p, beta, clip):
        xa, da, _ = oracle.rtn_quantize(X, oracle.PER_ROW, p, beta, clip=clip)
        wb, db, _ = oracle.rtn_quantize(W, oracle.PER_COL, p, beta, clip=clip)
        Cf = oracle.dequant(oracle.gemm_exact(xa, wb), da, oracle.PER_ROW, db, oracle.PER_COL)
        return np.linalg.norm(Cf - ref) / np.linalg.norm(ref)

    e_method = err(0.95, 15, False)
    e_clip = err(0.995, 15, True)
    e_wide = err(1.0, 255, False)
    assert e_method < 0.1 * e_clip, (e_method, e_clip)
    assert e_method < 0.2 and e_wide < 0.2


def test_rtn_granularities_agree_with_per_group_calls():
    rng = np.random.default_rng(14)
    X = rng.standard_normal((9, 13)).astype(np.float32)
    xr, dr, qr = oracle.rtn_quantize(X, oracle.PER_ROW, 0.9, 15)
    xc, dc, qc = oracle.rtn_quantize(X, oracle.PER_COL, 0.9, 15)
    for r in range(9):
        a, d, q = oracle.rtn_quantize(X[r:r + 1], oracle.PER_TENSOR, 0.9, 15)
        assert np.array_equal(a[0], xr[r]) and d[0] == dr[r] and q[0] == qr[r]
    for c in range(13):
        a, d, q = oracle.rtn_quantize(X[:, c:c + 1].copy(), oracle.PER_TENSOR, 0.9, 15)
        assert np.array_equal(a[:, 0], xc[:, c]) and d[0] == dc[c]


def test_rtn_zero_groups_and_errors():
    x = np.zeros((2, 40), np.float32)
    x[1, 3] = 2.0  # 39 zeros: the 95% rank is 0, so the maximum is used
    xi, d, q = oracle.rtn_quantize(x, oracle.PER_ROW, 0.95, 15)
    assert d[0] == 1.0 and q[0] == 0.0 and not xi[0].any()
    assert q[1] == 2.0 and xi[1, 3] == 15
    bad = np.ones((1, 4), np.float32)
    bad[0, 2] = np.nan
    with pytest.raises(oracle.OracleError) as e:
        oracle.rtn_quantize(bad, oracle.PER_TENSOR, 0.95, 15)
    assert e.value.status == oracle.ERR_NONFINITE
    big = np.full((1, 100), 1e-3, np.float32)
    big[0, 0] = 1e8  # 1e8 / 1e-3 * 15 >= 2^31
    with pytest.raises(oracle.OracleError) as e:
        oracle.rtn_quantize(big, oracle.PER_TENSOR, 0.95, 15)
    assert e.value.status == oracle.ERR_RANGE


# ------------------------------------------------------------------------------------------------
# digits ("Approach": an out-of-bound integer becomes several in-bound b-bit integers)
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("b", range(2, 9))
def test_digits_exhaustive(b):
    R = 1 << (b - 1)
    nl = math.ceil(21 / (b - 1)) + 1
    v = np.arange(-(1 << 20) + 1, 1 << 20, dtype=np.int64)
    d, lev = oracle.digits_array(v, b, nl)
    w = np.array([R ** l for l in range(nl)], dtype=np.int64)
    assert np.array_equal(d @ w, v)                          # reconstruction
    assert np.abs(d).max() <= R - 1                          # in range
    assert np.all(d * np.sign(v)[:, None] >= 0)              # every digit carries v's sign
    # level: 1 for |v| <= R-1, else the smallest L with |v| < R^L
    a = np.abs(v)
    want = np.ones_like(a)
    for L in range(2, nl + 1):
        want[a >= R ** (L - 1)] = L
    assert np.array_equal(lev, want)
    # digits above the level are zero
    cols = np.arange(nl)[None, :]
    assert not d[cols >= lev[:, None]].any()


# ------------------------------------------------------------------------------------------------
# unpacked product == direct product ("Approach": the original GEMM is reproduced exactly)
# ------------------------------------------------------------------------------------------------
def _brute(A, B):
    M, K = A.shape
    N = B.shape[1]
    return np.array([[sum(int(A[i, t]) * int(B[t, j]) for t in range(K)) for j in range(N)]
                     for i in range(M)], dtype=np.int64)


def test_unpacked_equals_direct_random_tiny():
    rng = np.random.default_rng(21)
    for case in range(1000):
        M, K, N = (int(x) for x in rng.integers(1, 10, size=3))
        b = int(rng.integers(2, 9))
        A, B = workloads.random_case(rng, M, K, N, big=5000, frac=float(rng.choice([0.0, 0.05, 0.3])))
        direct = _brute(A, B) if case < 100 else oracle.gemm_i64(A, B)
        if case < 100:
            assert np.array_equal(direct, oracle.gemm_i64(A, B))
        R = 1 << (b - 1)
        for st in range(7):
            pl = oracle.plan(A, B, b, st)
            Au, Bu = oracle.unpack(pl, A, B)
            assert np.abs(Au.astype(np.int64)).max(initial=0) <= R - 1
            assert np.abs(Bu.astype(np.int64)).max(initial=0) <= R - 1
            assert np.array_equal(oracle.unpacked_gemm(pl, Au, Bu), direct), (case, st, b)
            # the bound covers |C|
            assert np.abs(direct).max(initial=0) <= pl.bound


def test_direct_product_against_numpy_int64():
    rng = np.random.default_rng(22)
    for M, K, N in [(1, 1, 1), (3, 5, 7), (64, 128, 64), (512, 512, 512), (37, 511, 129)]:
        A, B = workloads.random_case(rng, M, K, N, big=30000)
        want = np.matmul(A, B)  # exact here: |C| < 2^63
        assert np.array_equal(oracle.gemm_i64(A, B), want)
        assert np.array_equal(oracle.gemm_exact(A, B), want)


def test_tiny_config_int64_against_brute_force():
    g = workloads.tiny()[0]
    A, dA, _ = oracle.rtn_quantize(oracle.as_f32(g.A.data, "f32"), oracle.PER_TENSOR, 0.95, 15)
    B, dB, _ = oracle.rtn_quantize(oracle.as_f32(g.B.data, "f32"), oracle.PER_TENSOR, 0.95, 15)
    direct = _brute(A, B)
    assert np.array_equal(oracle.gemm_i64(A, B), direct)
    pl = oracle.plan(A, B, 5, oracle.MIX)
    Au, Bu = oracle.unpack(pl, A, B)
    assert np.array_equal(oracle.unpacked_gemm(pl, Au, Bu), direct)
    assert pl.ratio > 1.0  # the planted heavy hitters need unpacking


# ------------------------------------------------------------------------------------------------
# unpack ratio (named as a metric; no formula on the page) -- closed forms
# ------------------------------------------------------------------------------------------------
def test_ratio_closed_forms():
    K, M, N, b = 40, 6, 5, 5
    A = np.full((M, K), 3, np.int64)
    A[:, 7] = 100          # one column, every row, level 2 at b=5 (16 <= 100 < 256)
    B = np.full((K, N), -2, np.int64)
    pl = oracle.plan(A, B, b, oracle.COL_ROW)
    assert pl.K_eff == K + 1 and pl.ratio == pytest.approx((K + 1) / K, rel=0, abs=1e-15)
    pl = oracle.plan(A, B, b, oracle.ROW_ROW)
    assert pl.M_eff == 2 * M and pl.ratio == 2.0
    # Mix picks the column for A (factor (K+1)/K < 2) and does not unpack B
    pl = oracle.plan(A, B, b, oracle.MIX)
    assert (pl.dir_a, pl.dir_b) == (oracle.DIR_INNER, oracle.DIR_NONE)
    # nothing out of range: identity plan, ratio exactly 1, product is a plain int8 GEMM
    rng = np.random.default_rng(23)
    A8 = rng.integers(-127, 128, size=(33, 70)).astype(np.int64)
    B8 = rng.integers(-127, 128, size=(70, 17)).astype(np.int64)
    pl = oracle.plan(A8, B8, 8, oracle.MIX)
    assert (pl.dir_a, pl.dir_b, pl.ratio) == (oracle.DIR_NONE, oracle.DIR_NONE, 1.0)
    assert (pl.M_eff, pl.N_eff, pl.K_eff) == (33, 17, 70)
    Au, Bu = oracle.unpack(pl, A8, B8)
    assert np.array_equal(Au, A8.astype(np.int8))
    assert np.array_equal(Bu, B8.T.astype(np.int8))


def test_ratio_equals_counted_macs():
    """The ratio (computed from the line levels) equals the multiply-adds the naive unpacked loop
    counts while it rebuilds the product, over the original M N K."""
    rng = np.random.default_rng(24)
    for _ in range(200):
        M, K, N = (int(x) for x in rng.integers(1, 12, size=3))
        b = int(rng.integers(2, 9))
        A, B = workloads.random_case(rng, M, K, N, big=3000, frac=0.2)
        for st in range(7):
            pl = oracle.plan(A, B, b, st)
            Au, Bu = oracle.unpack(pl, A, B)
            C, macs = oracle.unpacked_gemm(pl, Au, Bu, return_macs=True)
            assert np.array_equal(C, A @ B)
            assert macs == pl.M_eff * pl.N_eff * pl.K_eff
            assert pl.ratio == pytest.approx(macs / (M * N * K), rel=1e-12)


# ------------------------------------------------------------------------------------------------
# Mix ("Approach": direction chosen per matrix from outlier counts)
# ------------------------------------------------------------------------------------------------
def _levels_numpy(X, b):
    R = 1 << (b - 1)
    a = np.abs(X)
    L = np.ones_like(a)
    t = a // R
    while (t > 0).any():
        L += (t > 0)
        t //= R
    return L


def test_mix_choice_bruteforce():
    rng = np.random.default_rng(25)
    for _ in range(300):
        M, K, N = (int(x) for x in rng.integers(1, 10, size=3))
        b = int(rng.integers(2, 9))
        A, B = workloads.random_case(rng, M, K, N, big=int(rng.choice([50, 5000])), frac=0.15)
        pl = oracle.plan(A, B, b, oracle.MIX)
        LA, LB = _levels_numpy(A, b), _levels_numpy(B, b)
        lar, lac, lbr, lbc = LA.max(1), LA.max(0), LB.max(1), LB.max(0)
        assert np.array_equal(pl.levels["a_row"], lar) and np.array_equal(pl.levels["a_col"], lac)
        assert np.array_equal(pl.levels["b_row"], lbr) and np.array_equal(pl.levels["b_col"], lbc)

        def choose(row_lv, col_lv, row_is_outer):
            if (row_lv > 1).sum() == 0 and (col_lv > 1).sum() == 0:
                return oracle.DIR_NONE
            fr, fc = Fraction(int(row_lv.sum()), row_lv.size), Fraction(int(col_lv.sum()), col_lv.size)
            nr, nc = int((row_lv > 1).sum()), int((col_lv > 1).sum())
            row_dir = oracle.DIR_OUTER if row_is_outer else oracle.DIR_INNER
            col_dir = oracle.DIR_INNER if row_is_outer else oracle.DIR_OUTER
            if fr != fc:
                return row_dir if fr < fc else col_dir
            if nr != nc:
                return row_dir if nr < nc else col_dir
            return row_dir

        assert pl.dir_a == choose(lar, lac, True)
        assert pl.dir_b == choose(lbr, lbc, False)


def _pair_cost(lar, lac, lbr, lbc, da, db):
    """Exact unpacked size M_eff * N_eff * K_eff of one direction pair, from the line levels."""
    M, N = lar.size, lbc.size
    me = int(lar.sum()) if da == oracle.DIR_OUTER else M
    ne = int(lbc.sum()) if db == oracle.DIR_OUTER else N
    la = lac if da == oracle.DIR_INNER else np.ones_like(lac)
    lb = lbr if db == oracle.DIR_INNER else np.ones_like(lbr)
    return me * ne * int((la.astype(np.int64) * lb.astype(np.int64)).sum())


def test_joint_mix_is_the_cheapest_pair_bruteforce():
    """Joint Mix (a reading of the per-matrix choice that weighs both matrices together): the pair of
    least exact unpacked size, strict improvements over the per-matrix Mix choice taken in the order
    row/row, row/col, col/row, col/col.  Costs re-derived from numpy levels."""
    rng = np.random.default_rng(27)
    pairs = [(oracle.DIR_OUTER, oracle.DIR_INNER), (oracle.DIR_OUTER, oracle.DIR_OUTER),
             (oracle.DIR_INNER, oracle.DIR_INNER), (oracle.DIR_INNER, oracle.DIR_OUTER)]
    differs = 0
    for _ in range(400):
        M, K, N = (int(x) for x in rng.integers(1, 10, size=3))
        b = int(rng.integers(2, 9))
        A, B = workloads.random_case(rng, M, K, N, big=int(rng.choice([50, 5000])), frac=0.15)
        LA, LB = _levels_numpy(A, b), _levels_numpy(B, b)
        lar, lac, lbr, lbc = LA.max(1), LA.max(0), LB.max(1), LB.max(0)
        mix = oracle.plan(A, B, b, oracle.MIX)
        joint = oracle.plan(A, B, b, oracle.MIX_JOINT)
        da, db = mix.dir_a, mix.dir_b
        best = _pair_cost(lar, lac, lbr, lbc, da, db)
        for pa, pb in pairs:
            ca = oracle.DIR_NONE if mix.dir_a == oracle.DIR_NONE else pa
            cb = oracle.DIR_NONE if mix.dir_b == oracle.DIR_NONE else pb
            c = _pair_cost(lar, lac, lbr, lbc, ca, cb)
            if c < best:
                best, da, db = c, ca, cb
        assert (joint.dir_a, joint.dir_b) == (da, db)
        assert joint.ratio <= mix.ratio
        differs += (joint.dir_a, joint.dir_b) != (mix.dir_a, mix.dir_b)
        # the exact product whatever the directions
        Au, Bu = oracle.unpack(joint, A, B)
        assert np.array_equal(oracle.unpacked_gemm(joint, Au, Bu), A @ B)
    assert differs > 0  # the two rules do part ways on some inputs


def test_joint_mix_worked_case():
    """Closed form, b = 5 (R = 16): 300 needs 3 digits.  A 3x4 with 300 at (0,0), B 4x1 with 300 at
    (0,0), all else 1.  Levels: A rows 3,1,1 and columns 3,1,1,1; B rows 3,1,1,1 and column 3.
    Per-matrix Mix: A's column side 6*3 = 18 < row side 5*4 = 20, B's row side 6*1 < column side 3*4,
    so col/row with size 3*1*(3*3+1+1+1) = 36.  Row/row costs 5*1*6 = 30, row/col 5*3*4 = 60 and
    col/col 3*3*6 = 54, so Joint Mix takes row/row: ratio 30/12 = 2.5 against Mix's 36/12 = 3."""
    A = np.ones((3, 4), dtype=np.int64)
    B = np.ones((4, 1), dtype=np.int64)
    A[0, 0] = 300
    B[0, 0] = 300
    mix = oracle.plan(A, B, 5, oracle.MIX)
    joint = oracle.plan(A, B, 5, oracle.MIX_JOINT)
    assert (mix.dir_a, mix.dir_b) == (oracle.DIR_INNER, oracle.DIR_INNER)
    assert mix.ratio == pytest.approx(3.0)
    assert (joint.dir_a, joint.dir_b) == (oracle.DIR_OUTER, oracle.DIR_INNER)
    assert joint.ratio == pytest.approx(2.5)
    Au, Bu = oracle.unpack(joint, A, B)
    assert np.array_equal(oracle.unpacked_gemm(joint, Au, Bu), A @ B)


def _hybrid_expected(X, b, outer_axis):
    """Brute force of the hybrid choice for one matrix, from numpy levels: every threshold tau from 1 to
    (largest out-of-range count) + 1, the lines with count >= tau OUTER with their own level, the inner
    levels the maxima over the other lines; least size, smallest tau on a tie.  Returns the (outer,
    inner) level vectors each line carries and the size."""
    L = _levels_numpy(X, b)
    if outer_axis == 1:
        L = L.T  # outer lines as rows
    cnt = (L > 1).sum(axis=1)
    lo_true = L.max(axis=1, initial=1)
    best = None
    for tau in range(1, int(cnt.max(initial=0)) + 2):
        S = cnt >= tau
        lo = np.where(S, lo_true, 1)
        li = L[~S].max(axis=0, initial=1) if L.shape[1] else np.zeros(0, np.int64)
        size = int(lo.sum()) * int(li.sum())
        if best is None or size < best[0]:
            best = (size, lo, li)
    return best[1], best[2], best[0]


def test_hybrid_choice_bruteforce():
    """Hybrid ("unpack both", a reading: the outer lines dense with out-of-range entries unpacked OUTER,
    the rest INNER): the levels each line carries equal a brute force over every threshold, the
    per-matrix size is never above the smaller of the pure row and pure column sizes (which are its
    thresholds 1 and max + 1), and the unpacked product is exact."""
    rng = np.random.default_rng(29)
    wins = 0
    for case in range(300):
        M, K, N = (int(x) for x in rng.integers(1, 14, size=3))
        b = int(rng.integers(2, 9))
        if case % 2:
            A, B = workloads.rows_and_cols_case(rng, M, K, N, big=int(rng.choice([100, 5000])),
                                                dense_rows=int(rng.integers(0, 3)), dense_cols=int(rng.integers(0, 3)))
        else:
            A, B = workloads.random_case(rng, M, K, N, big=int(rng.choice([50, 5000])), frac=0.15)
        pl = oracle.plan(A, B, b, oracle.HYBRID)
        lar, lac, size_a = _hybrid_expected(A, b, 0)
        lbc, lbr, size_b = _hybrid_expected(B, b, 1)
        assert np.array_equal(pl.levels["a_row"], lar) and np.array_equal(pl.levels["a_col"], lac)
        assert np.array_equal(pl.levels["b_row"], lbr) and np.array_equal(pl.levels["b_col"], lbc)
        assert pl.dir_a == (oracle.DIR_OUTER if (lar > 1).any() else 0) | (oracle.DIR_INNER if (lac > 1).any() else 0)
        assert pl.dir_b == (oracle.DIR_OUTER if (lbc > 1).any() else 0) | (oracle.DIR_INNER if (lbr > 1).any() else 0)
        LA, LB = _levels_numpy(A, b), _levels_numpy(B, b)
        assert size_a <= min(int(LA.max(1).sum()) * K, M * int(LA.max(0).sum()))
        assert size_b <= min(int(LB.max(0).sum()) * K, N * int(LB.max(1).sum()))
        wins += size_a < min(int(LA.max(1).sum()) * K, M * int(LA.max(0).sum()))
        Au, Bu = oracle.unpack(pl, A, B)
        assert np.abs(Au.astype(np.int64)).max(initial=0) <= (1 << (b - 1)) - 1
        assert np.array_equal(oracle.unpacked_gemm(pl, Au, Bu), A @ B), case
    assert wins > 0  # the hybrid is strictly smaller than both pure directions on some inputs


def test_hybrid_worked_case():
    """Closed form, b = 5 (R = 16, 100 has 2 digits).  A 64 x 64 of ones with row 0 all 100 and
    columns 5 and 9 equal to 100 in rows 10..29.  Row unpacking doubles the 21 rows holding outliers:
    85 x 64.  Column unpacking doubles every column (row 0 reaches all of them): 64 x 128.  The hybrid
    unpacks row 0 (64 outliers) OUTER and columns 5 and 9 INNER over the other rows (2 outliers each,
    below any threshold from 3 to 64): 65 x 66, the smallest threshold of that size being 3.  B is 64 x 8
    of ones (nothing to unpack).  Ratios: Mix 85/64, hybrid 65 * 66 / 64^2."""
    A = np.ones((64, 64), np.int64)
    A[0, :] = 100
    A[10:30, 5] = 100
    A[10:30, 9] = 100
    B = np.ones((64, 8), np.int64)
    mix = oracle.plan(A, B, 5, oracle.MIX)
    hyb = oracle.plan(A, B, 5, oracle.HYBRID)
    assert (mix.dir_a, mix.M_eff, mix.K_eff) == (oracle.DIR_OUTER, 85, 64)
    assert (hyb.dir_a, hyb.dir_b, hyb.M_eff, hyb.K_eff, hyb.N_eff) == (oracle.DIR_BOTH, oracle.DIR_NONE, 65, 66, 8)
    assert hyb.ratio == pytest.approx(65 * 66 / 64 ** 2, rel=1e-15)
    want_rows = np.ones(64, np.int32)
    want_rows[0] = 2
    want_cols = np.ones(64, np.int32)
    want_cols[[5, 9]] = 2
    assert np.array_equal(hyb.levels["a_row"], want_rows) and np.array_equal(hyb.levels["a_col"], want_cols)
    Au, Bu = oracle.unpack(hyb, A, B)
    # row 0's two lines (0, 0) and (0, 1) hold its digits (4 and 6: 100 = 6 * 16 + 4) at the triples
    # with lA = 0 only
    al, pr = hyb.lines["a_lines"], hyb.lines["pairs"]
    assert al[:3].tolist() == [[0, 0], [0, 1], [1, 0]]
    lo = pr[:, 1] == 0
    hi = ~lo
    assert int(hi.sum()) == 2 and sorted(pr[hi, 0].tolist()) == [5, 9]
    assert np.all(Au[0, lo] == 4) and np.all(Au[1, lo] == 6)
    assert not Au[:2][:, hi].any()
    # row 10 (line 11) carries the high digits of columns 5 and 9 at their lA = 1 triples
    assert al[11].tolist() == [10, 0]
    assert sorted(Au[11, hi].tolist()) == [6, 6]
    assert np.array_equal(oracle.unpacked_gemm(hyb, Au, Bu), A @ B)


def test_mix_beats_fixed_on_channel_outliers():
    """The measured-effects table reports Mix below every fixed strategy on linear layers, where
    heavy hitters sit in channels; a channel-structured case reproduces that ordering."""
    rng = np.random.default_rng(26)
    M, K, N, b = 64, 96, 48, 5
    A = rng.integers(-15, 16, size=(M, K)).astype(np.int64)
    B = rng.integers(-15, 16, size=(K, N)).astype(np.int64)
    A[:, [3, 50]] *= 40          # activation outlier channels: columns of A
    B[[10, 70], :] *= 30         # weight outlier input channels: rows of B
    ratios = {st: oracle.plan(A, B, b, st).ratio for st in range(5)}
    mix = oracle.plan(A, B, b, oracle.MIX)
    assert (mix.dir_a, mix.dir_b) == (oracle.DIR_INNER, oracle.DIR_INNER)  # col/row
    assert ratios[oracle.MIX] == ratios[oracle.COL_ROW]
    others = (oracle.ROW_ROW, oracle.ROW_COL, oracle.COL_COL)
    assert all(ratios[oracle.MIX] < ratios[st] for st in others), ratios
    assert ratios[oracle.MIX] < 1.1


# ------------------------------------------------------------------------------------------------
# dequantisation (implied by RTN GEMMs replacing FP GEMMs)
# ------------------------------------------------------------------------------------------------
def test_dequant_exact_rational_bound():
    rng = np.random.default_rng(27)
    C = rng.integers(-(1 << 40), 1 << 40, size=(7, 5)).astype(np.int64)
    C[0, 0] = 0
    dA = rng.uniform(1e-4, 1.0, 7).astype(np.float32)
    dB = rng.uniform(1e-4, 1.0, 5).astype(np.float32)
    Cf = oracle.dequant(C, dA, oracle.PER_ROW, dB, oracle.PER_COL)
    assert Cf[0, 0] == 0.0
    for i in range(7):
        for j in range(5):
            exact = Fraction(int(C[i, j])) * Fraction(float(dA[i])) * Fraction(float(dB[j]))
            if exact != 0:
                assert abs(Fraction(float(Cf[i, j])) - exact) / abs(exact) <= Fraction(1, 2 ** 51)
    ones = np.ones(1, np.float32)
    assert np.array_equal(oracle.dequant(C, ones, oracle.PER_TENSOR, ones, oracle.PER_TENSOR),
                          C.astype(np.float64))


# ------------------------------------------------------------------------------------------------
# the unpacked lines and inner triples ("Approach": a row or column with out-of-bound entries becomes
# several in-bound ones) -- re-derived from numpy levels, independent of the oracle's C code
# ------------------------------------------------------------------------------------------------
def test_unpacked_lines_and_triples_from_levels():
    """Line (i, l) of A for every l below the level row i carries when A is unpacked OUTER (l = 0 only
    otherwise); likewise (j, m) for B; triple (t, lA, lB) for lA below A's column level when A is INNER
    and lB below B's row level when B is INNER.  The exponent counts are those of the triples."""
    rng = np.random.default_rng(28)
    for case in range(150):
        M, K, N = (int(x) for x in rng.integers(1, 30, size=3))
        b = int(rng.integers(2, 9))
        A, B = workloads.random_case(rng, M, K, N, big=4000, frac=0.2)
        if case % 3 == 0:
            A, B = workloads.rows_and_cols_case(rng, M, K, N, big=4000, dense_rows=2, dense_cols=2)
        LA, LB = _levels_numpy(A, b), _levels_numpy(B, b)
        for st in range(6):  # the hybrid's carried levels are pinned by its own brute force above
            pl = oracle.plan(A, B, b, st)
            la_row = LA.max(1) if pl.dir_a & oracle.DIR_OUTER else np.ones(M, np.int64)
            la_col = LA.max(0) if pl.dir_a & oracle.DIR_INNER else np.ones(K, np.int64)
            lb_row = LB.max(1) if pl.dir_b & oracle.DIR_INNER else np.ones(K, np.int64)
            lb_col = LB.max(0) if pl.dir_b & oracle.DIR_OUTER else np.ones(N, np.int64)
            a_lines = [[i, l] for i in range(M) for l in range(la_row[i])]
            b_lines = [[j, m] for j in range(N) for m in range(lb_col[j])]
            pairs = [[t, x, y] for t in range(K) for x in range(la_col[t]) for y in range(lb_row[t])]
            assert pl.lines["a_lines"].tolist() == a_lines
            assert pl.lines["b_lines"].tolist() == b_lines
            assert pl.lines["pairs"].tolist() == pairs
            assert (pl.M_eff, pl.N_eff, pl.K_eff) == (len(a_lines), len(b_lines), len(pairs))
            es = {}
            for _, x, y in pairs:
                es[x + y] = es.get(x + y, 0) + 1
            assert pl.groups == sorted(es.items())


def test_cached_plan_is_exact_for_covered_inputs():
    """A plan made from one A serves any other A' whose entries stay within the first one's column
    maxima, |A'[i,t]| <= max_i |A[i,t]| (what the fused quantise-and-unpack path checks against a plan
    kept with an unpacked weight): the levels, the inner layout and the bound all still hold, so the
    unpacked product with the kept B' is exact.  Random inputs, A not unpacked OUTER (A's rows are then
    single lines whose layout does not depend on the new values)."""
    rng = np.random.default_rng(31)
    checked = 0
    for case in range(400):
        M, K, N = (int(x) for x in rng.integers(1, 12, size=3))
        b = int(rng.integers(2, 9))
        A, B = workloads.random_case(rng, M, K, N, big=int(rng.choice([60, 3000])), frac=0.15)
        pl = oracle.plan(A, B, b, oracle.COL_ROW if case % 2 else oracle.MIX)
        if pl.dir_a & oracle.DIR_OUTER:
            continue
        cmax = np.abs(A).max(axis=0)
        A2 = rng.integers(-cmax, cmax + 1, size=(M, K)).astype(np.int64)  # within the column maxima
        Au, Bu = oracle.unpack(pl, A2, B)
        assert np.array_equal(oracle.unpacked_gemm(pl, Au, Bu), A2 @ B), case
        checked += 1
    assert checked > 150
