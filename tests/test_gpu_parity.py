"""GPU parity of every stage of the path against the CPU oracle, through the C ABI.

Integer results (quantised values, levels, plan sizes, unpacked bytes, the product C) must be
bit-exact; dequantised fp32 outputs within 1e-6 relative of the oracle's float64 value.  Sizes span
several 128 x 256 GEMM tiles and ragged edges.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_common import (assert_f32_close, check_layout, check_unpacked, logical, plan_matches, to_device,
                               unsupported)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def imq():
    import bit_integer_gemm_b200 as m
    assert torch.cuda.is_available(), "a GPU is required"
    m.lib()
    m.imq_device_status(clear=True)
    return m


# ------------------------------------------------------------------------------------------------
# quantisation
# ------------------------------------------------------------------------------------------------
def _matrix(rng, shape, heavy=True):
    x = rng.standard_normal(shape).astype(np.float32) * np.float32(rng.uniform(0.01, 10))
    if heavy and x.size:
        idx = rng.choice(x.size, max(1, x.size // 200), replace=False)
        x.reshape(-1)[idx] *= np.float32(40)
    return x


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("gran", [oracle.PER_TENSOR, oracle.PER_ROW, oracle.PER_COL])
@pytest.mark.parametrize("shape", [(1, 1), (3, 5), (37, 129), (128, 4096), (257, 1000), (1000, 64)])
@pytest.mark.parametrize("p,beta", [(0.95, 15), (1.0, 31), (0.5, 255)])
def test_quantize_parity(imq, dtype, gran, shape, p, beta):
    rng = np.random.default_rng(zlib.crc32(repr((dtype, gran, shape, p)).encode()))
    x = _matrix(rng, shape)
    st = workloads.Stored("x", workloads.f32_to_bf16_bits(x) if dtype == "bf16" else x, dtype)
    want_i, want_d, want_q = oracle.rtn_quantize(oracle.as_f32(st.data, dtype), gran, p, beta)
    X = to_device(st)
    for out in (torch.int16, torch.int32):
        if out == torch.int16 and np.abs(want_i).max() > 32767:
            continue
        r = imq.imq_rtn_quantize(X, gran, p, beta, out_dtype=out)
        torch.cuda.synchronize()
        assert imq.imq_device_status() == imq.IMQ_OK
        assert np.array_equal(r.xint.cpu().numpy().astype(np.int64), want_i)
        assert np.array_equal(r.delta.cpu().numpy().view(np.uint32), want_d.view(np.uint32))
        assert np.array_equal(r.qval.cpu().numpy().view(np.uint32), want_q.view(np.uint32))
        assert np.array_equal(r.rowmax.cpu().numpy(), np.abs(want_i).max(axis=1))
        assert np.array_equal(r.colmax.cpu().numpy(), np.abs(want_i).max(axis=0))


def _select_patterns(rng, n):
    """bf16 groups of n entries built against a select that brackets the rank from an evenly spaced
    sample: sorted groups, ties, a period equal to the sample spacing (the sample then sees only the
    large entries and the bracket misses), heavy tails, signed zeros and subnormals."""
    spaced = ((2 * np.arange(256) + 1) * n) // 512
    rows = []
    rows.append(rng.standard_normal(n))
    rows.append(np.sort(np.abs(rng.standard_normal(n))))
    rows.append(-np.sort(np.abs(rng.standard_normal(n)))[::-1])
    rows.append(np.full(n, 0.5))
    rows.append(rng.integers(0, 3, n) * 0.25 * rng.choice([-1.0, 1.0], n))
    r = rng.standard_normal(n) * 0.01
    r[spaced] = 10.0
    rows.append(r)
    r = rng.standard_normal(n)
    r[: n // 2] = 0.0
    rows.append(rng.permutation(r))
    rows.append(np.clip(rng.standard_cauchy(n), -1e3, 1e3))
    r = rng.choice([1e-40, -1e-40, 0.0, -0.0, 3e-39], n)
    normal = rng.random(n) < 0.6
    r[normal] = rng.standard_normal(int(normal.sum())) * 1e-30
    rows.append(r)
    rows.append(np.zeros(n))
    r = rng.standard_normal(n) * 1e-3
    r[rng.integers(n)] = 2.0
    rows.append(r)
    r = rng.standard_normal(n)
    r[rng.choice(n, n // 20, replace=False)] *= 60.0  # 5 % heavy hitters: the rank sits at their edge
    rows.append(r)
    return np.stack(rows).astype(np.float32)


@pytest.mark.parametrize("n", [1024, 1031, 4096, 11008])
@pytest.mark.parametrize("p", [0.95, 0.5, 1.0, 0.999, 1e-4])
def test_quantize_select_adversarial_groups(imq, n, p):
    """The sampled bf16 select (groups of 1024 and more) against the oracle's full sort, per row and per
    column (the transposed matrix: the staged column kernel), including the groups that defeat it."""
    rng = np.random.default_rng(zlib.crc32(repr(("sel", n, p)).encode()))
    x = _select_patterns(rng, n)
    for gran, mat in ((oracle.PER_ROW, x), (oracle.PER_COL, np.ascontiguousarray(x.T))):
        bits = workloads.f32_to_bf16_bits(mat)
        want_i, want_d, want_q = oracle.rtn_quantize(oracle.bf16_bits_to_f32(bits), gran, p, 15)
        X = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
        r = imq.imq_rtn_quantize(X, gran, p, 15, out_dtype=torch.int32)
        torch.cuda.synchronize()
        assert imq.imq_device_status() == imq.IMQ_OK
        assert np.array_equal(r.qval.cpu().numpy().view(np.uint32), want_q.view(np.uint32)), gran
        assert np.array_equal(r.delta.cpu().numpy().view(np.uint32), want_d.view(np.uint32)), gran
        assert np.array_equal(r.xint.cpu().numpy().astype(np.int64), want_i), gran
        assert np.array_equal(r.rowmax.cpu().numpy(), np.abs(want_i).max(axis=1)), gran
        assert np.array_equal(r.colmax.cpu().numpy(), np.abs(want_i).max(axis=0)), gran


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("gran", [oracle.PER_TENSOR, oracle.PER_ROW, oracle.PER_COL])
@pytest.mark.parametrize("shape", [(3, 5), (37, 129), (257, 1000), (1000, 64), (20000, 8)])
@pytest.mark.parametrize("p,beta", [(0.995, 15), (0.9, 255)])
@pytest.mark.parametrize("trans_out", [False, True])
def test_quantize_clip_parity(imq, dtype, gran, shape, p, beta, trans_out):
    """The clipping comparison variant (imq_rtn_quantize_ex, IMQ_RTN_CLIP) on every quantiser path:
    per tensor, per row, per column staged and streamed (20000-row columns), plain and transposed out."""
    rng = np.random.default_rng(zlib.crc32(repr(("clip", dtype, gran, shape, p, trans_out)).encode()))
    x = _matrix(rng, shape)
    st = workloads.Stored("x", workloads.f32_to_bf16_bits(x) if dtype == "bf16" else x, dtype)
    want_i, want_d, want_q = oracle.rtn_quantize(oracle.as_f32(st.data, dtype), gran, p, beta, clip=True)
    assert np.abs(want_i).max() <= beta
    r = imq.imq_rtn_quantize(to_device(st), gran, p, beta, trans_out=trans_out, clip=True)
    torch.cuda.synchronize()
    assert imq.imq_device_status() == imq.IMQ_OK
    got = r.xint.cpu().numpy().astype(np.int64)
    assert np.array_equal(got.T if trans_out else got, want_i)
    assert np.array_equal(r.delta.cpu().numpy().view(np.uint32), want_d.view(np.uint32))
    assert np.array_equal(r.qval.cpu().numpy().view(np.uint32), want_q.view(np.uint32))
    assert np.array_equal(r.rowmax.cpu().numpy(), np.abs(want_i).max(axis=1))
    assert np.array_equal(r.colmax.cpu().numpy(), np.abs(want_i).max(axis=0))


def test_quantize_ex_rejects_unknown_flags(imq):
    X = torch.ones((4, 8), device="cuda")
    Xint = torch.empty((4, 8), dtype=torch.int16, device="cuda")
    d = torch.empty(4, device="cuda")
    st = imq.lib().imq_rtn_quantize_ex(imq._ptr(X), imq.IMQ_F32, 4, 8, 8, imq.IMQ_PER_ROW, 0.95, 15, imq._ptr(Xint),
                                       imq.IMQ_I16, 8, 0, imq._ptr(d), None, None, None, 2, imq._stream(None))
    assert st == imq.IMQ_ERR_ARG


@pytest.mark.parametrize("gran", [oracle.PER_TENSOR, oracle.PER_ROW, oracle.PER_COL])
@pytest.mark.parametrize("shape", [(5, 3), (300, 130), (4096, 96), (1000, 17)])
def test_quantize_transposed_output(imq, gran, shape):
    rng = np.random.default_rng(zlib.crc32(repr(("T", gran, shape)).encode()))
    x = _matrix(rng, shape)
    bits = workloads.f32_to_bf16_bits(x)
    want_i, want_d, _ = oracle.rtn_quantize(oracle.bf16_bits_to_f32(bits), gran, 0.95, 15)
    X = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    r = imq.imq_rtn_quantize(X, gran, 0.95, 15, trans_out=True)
    assert tuple(r.xint.shape) == (shape[1], shape[0])
    assert np.array_equal(r.xint.cpu().numpy().astype(np.int64), want_i.T)
    assert np.array_equal(r.delta.cpu().numpy(), want_d)
    assert np.array_equal(r.rowmax.cpu().numpy(), np.abs(want_i).max(axis=1))
    assert np.array_equal(r.colmax.cpu().numpy(), np.abs(want_i).max(axis=0))


def test_quantize_tall_columns(imq):
    """Columns too tall for the staged kernel (11008 rows: 8-column slabs) and taller (streaming)."""
    rng = np.random.default_rng(15)
    for rows in (11008, 20000):
        x = _matrix(rng, (rows, 40))
        bits = workloads.f32_to_bf16_bits(x)
        want_i, want_d, _ = oracle.rtn_quantize(oracle.bf16_bits_to_f32(bits), oracle.PER_COL, 0.95, 31)
        X = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
        r = imq.imq_rtn_quantize(X, oracle.PER_COL, 0.95, 31, out_dtype=torch.int32)
        assert np.array_equal(r.xint.cpu().numpy().astype(np.int64), want_i)
        assert np.array_equal(r.delta.cpu().numpy(), want_d)
        assert np.array_equal(r.rowmax.cpu().numpy(), np.abs(want_i).max(axis=1))


def test_quantize_strided_input(imq):
    rng = np.random.default_rng(5)
    x = _matrix(rng, (70, 300))
    bits = workloads.f32_to_bf16_bits(x)
    full = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    X = full[:, 17:17 + 211]  # leading dimension 300, 211 columns, unaligned start
    sub = oracle.bf16_bits_to_f32(np.ascontiguousarray(bits[:, 17:228]))
    for gran in (oracle.PER_TENSOR, oracle.PER_ROW, oracle.PER_COL):
        want_i, want_d, _ = oracle.rtn_quantize(sub, gran, 0.95, 15)
        out = torch.zeros((70, 256), dtype=torch.int16, device="cuda")
        r = imq.imq_rtn_quantize(X, gran, 0.95, 15, Xint=out[:, :211])
        assert np.array_equal(r.xint.cpu().numpy().astype(np.int64), want_i)
        assert np.array_equal(r.delta.cpu().numpy(), want_d)
        assert not out[:, 211:].any()


def test_quantize_errors(imq):
    x = torch.ones((4, 64), device="cuda")
    x[2, 7] = float("nan")
    imq.imq_rtn_quantize(x, imq.IMQ_PER_ROW, 0.95, 15)
    assert imq.imq_device_status(clear=True) == imq.IMQ_ERR_NONFINITE
    y = torch.full((1, 1000), 1e-3, device="cuda")
    y[0, 0] = 100.0  # 100 / 1e-3 * 15 = 1.5e6: fits int32, not int16
    imq.imq_rtn_quantize(y, imq.IMQ_PER_TENSOR, 0.95, 15, out_dtype=torch.int16)
    assert imq.imq_device_status(clear=True) == imq.IMQ_ERR_RANGE
    r = imq.imq_rtn_quantize(y, imq.IMQ_PER_TENSOR, 0.95, 15, out_dtype=torch.int32)
    assert imq.imq_device_status(clear=True) == imq.IMQ_OK and int(r.xint[0, 0]) == 1500000
    for p, beta in ((0.0, 15), (1.5, 15), (0.95, 0)):
        with pytest.raises(imq.ImqError) as e:
            imq.imq_rtn_quantize(y, imq.IMQ_PER_TENSOR, p, beta)
        assert e.value.status == imq.IMQ_ERR_ARG


def test_quantize_empty(imq):
    x = torch.empty((0, 5), device="cuda")
    r = imq.imq_rtn_quantize(x, imq.IMQ_PER_COL, 0.95, 15)
    assert np.array_equal(r.delta.cpu().numpy(), np.ones(5, np.float32))


# ------------------------------------------------------------------------------------------------
# plan, unpack, GEMM on random integer matrices
# ------------------------------------------------------------------------------------------------
def _run_path(imq, A, B, b, strategy, transA, transB, dtype=torch.int16, check_unpack=True):
    """A, B: logical int64 numpy matrices.  Runs plan -> unpack -> GEMM on the GPU and checks each
    stage against the oracle."""
    M, K = A.shape
    N = B.shape[1]
    pl = oracle.plan(A, B, b, strategy)
    A_st = np.ascontiguousarray(A.T if transA else A)
    B_st = np.ascontiguousarray(B.T if transB else B)
    npdt = np.int16 if dtype == torch.int16 else np.int32
    Ad = torch.from_numpy(A_st.astype(npdt)).cuda()
    Bd = torch.from_numpy(B_st.astype(npdt)).cuda()
    if unsupported(pl):
        with pytest.raises(imq.ImqError) as e:
            imq.imq_plan(Ad, Bd, b, strategy, transA, transB)
        assert e.value.status == imq.IMQ_ERR_UNSUPPORTED
        return None
    plan = imq.imq_plan(Ad, Bd, b, strategy, transA, transB)
    plan_matches(plan.info, pl, plan.groups())
    lv = plan.levels()
    for k in ("a_row", "a_col", "b_row", "b_col"):
        assert np.array_equal(lv[k].astype(np.int32), pl.levels[k]), k
    Au, Bu = imq.imq_unpack(plan, Ad, Bd)
    if check_unpack:
        mp = check_unpacked(plan, pl, Au.cpu().numpy(), Bu.cpu().numpy(), A, B)
        check_layout(plan, mp)
    rng = np.random.default_rng(M * 7 + N)
    dA = rng.uniform(1e-3, 1.0, M).astype(np.float32)
    dB = rng.uniform(1e-3, 1.0, N).astype(np.float32)
    C, Cf = imq.imq_gemm_unpacked(plan, Au, Bu, torch.from_numpy(dA).cuda(), imq.IMQ_PER_ROW,
                                  torch.from_numpy(dB).cuda(), imq.IMQ_PER_COL)
    torch.cuda.synchronize()
    assert imq.imq_device_status() == imq.IMQ_OK
    want = oracle.gemm_exact(A, B)
    got = C.cpu().numpy().astype(np.int64)
    assert np.array_equal(got, want), f"C mismatch at {np.argwhere(got != want)[:5]}"
    assert_f32_close(Cf.cpu().numpy(), oracle.dequant(want, dA, oracle.PER_ROW, dB, oracle.PER_COL))
    return plan


@pytest.mark.parametrize("b", [2, 3, 5, 8])
@pytest.mark.parametrize("strategy", [0, 1, 2, 3, 4, 5, 6])
@pytest.mark.parametrize("trans", [(False, False), (True, False), (False, True), (True, True)])
def test_path_parity_int32_regime(imq, b, strategy, trans):
    rng = np.random.default_rng(1000 * b + 10 * strategy + 2 * trans[0] + trans[1])
    A, B = workloads.random_case(rng, 300, 500, 700, big=300, frac=0.05)
    _run_path(imq, A, B, b, strategy, *trans)


@pytest.mark.parametrize("b", [2, 3, 4, 5, 8])
@pytest.mark.parametrize("strategy", [0, 1, 2, 3, 4, 5, 6])
def test_path_parity_int64_regime(imq, b, strategy):
    rng = np.random.default_rng(77 + 10 * b + strategy)
    A, B = workloads.random_case(rng, 200, 384, 300, big=3000, frac=0.05)
    plan = _run_path(imq, A, B, b, strategy, False, True)
    if plan is not None:
        assert plan.info["acc_bits"] == 64


def test_joint_mix_parity_where_it_differs_from_mix(imq):
    """Joint Mix on inputs where it picks another direction pair than per-matrix Mix: the closed-form
    worked case of the oracle pins, and random cases found by the oracle."""
    A = np.ones((3, 4), dtype=np.int64)
    B = np.ones((4, 1), dtype=np.int64)
    A[0, 0] = 300
    B[0, 0] = 300
    plan = _run_path(imq, A, B, 5, imq.IMQ_MIX_JOINT, False, False)
    assert (plan.info["dir_a"], plan.info["dir_b"]) == (imq.IMQ_DIR_OUTER, imq.IMQ_DIR_INNER)
    rng = np.random.default_rng(4242)
    found = 0
    while found < 6:
        M, K, N = (int(x) for x in rng.integers(1, 40, size=3))
        b = int(rng.integers(2, 8))
        A, B = workloads.random_case(rng, M, K, N, big=int(rng.choice([50, 5000])), frac=0.15)
        mix, joint = oracle.plan(A, B, b, oracle.MIX), oracle.plan(A, B, b, oracle.MIX_JOINT)
        if (mix.dir_a, mix.dir_b) == (joint.dir_a, joint.dir_b):
            continue
        found += 1
        for transB in (False, True):
            _run_path(imq, A, B, b, imq.IMQ_MIX_JOINT, False, transB)


@pytest.mark.parametrize("b", [3, 5])
@pytest.mark.parametrize("trans", [(False, False), (True, False), (False, True), (True, True)])
def test_hybrid_parity_rows_and_columns(imq, b, trans):
    """Hybrid (unpack both) on operands whose heavy hitters sit in a few whole rows and a few whole
    columns, sizes spanning several tiles with ragged edges: the device's choice, levels, layout bytes
    and the exact product equal the oracle's, and both matrices are unpacked in both directions."""
    rng = np.random.default_rng(500 + 10 * b + 2 * trans[0] + trans[1])
    A, B = workloads.rows_and_cols_case(rng, 300, 520, 270, big=3000, dense_rows=3, dense_cols=4, scatter=0.002)
    plan = _run_path(imq, A, B, b, imq.IMQ_HYBRID, *trans)
    assert (plan.info["dir_a"], plan.info["dir_b"]) == (imq.IMQ_DIR_BOTH, imq.IMQ_DIR_BOTH)
    mix = oracle.plan(A, B, b, oracle.MIX)
    assert plan.info["ratio"] < mix.ratio


def test_hybrid_parity_worked_case_and_random(imq):
    """The oracle pins' worked case (one dense row and two outlier columns; the hybrid takes the row
    OUTER and the columns INNER), then random small cases of both input kinds, int16 and int32."""
    A = np.ones((64, 64), np.int64)
    A[0, :] = 100
    A[10:30, 5] = 100
    A[10:30, 9] = 100
    B = np.ones((64, 8), np.int64)
    plan = _run_path(imq, A, B, 5, imq.IMQ_HYBRID, False, False)
    assert (plan.info["dir_a"], plan.info["M_eff"], plan.info["K_eff"]) == (imq.IMQ_DIR_BOTH, 65, 66)
    rng = np.random.default_rng(4343)
    for case in range(24):
        M, K, N = (int(x) for x in rng.integers(1, 90, size=3))
        b = int(rng.integers(2, 9))
        if case % 2:
            A, B = workloads.rows_and_cols_case(rng, M, K, N, big=int(rng.choice([100, 5000])),
                                                dense_rows=int(rng.integers(0, 3)), dense_cols=int(rng.integers(0, 3)))
        else:
            A, B = workloads.random_case(rng, M, K, N, big=int(rng.choice([50, 5000])), frac=0.1)
        _run_path(imq, A, B, b, imq.IMQ_HYBRID, bool(case % 3 == 1), bool(case % 4 >= 2),
                  dtype=torch.int32 if case % 5 == 0 else torch.int16)


def test_path_parity_no_outliers_is_plain_int8(imq):
    rng = np.random.default_rng(3)
    A = rng.integers(-127, 128, size=(256 + 17, 1024 + 40)).astype(np.int64)
    B = rng.integers(-127, 128, size=(1024 + 40, 512 + 3)).astype(np.int64)
    plan = _run_path(imq, A, B, 8, 0, False, False)
    assert plan.info["ratio"] == 1.0 and plan.info["dir_a"] == 0 and plan.info["dir_b"] == 0


@pytest.mark.parametrize("shape", [(1, 1, 1), (1, 300, 1), (129, 1, 257), (128, 128, 256), (5, 3000, 9)])
def test_path_parity_edge_shapes(imq, shape):
    rng = np.random.default_rng(sum(shape))
    A, B = workloads.random_case(rng, *shape, big=3000, frac=0.1)
    for st in range(7):
        _run_path(imq, A, B, 5, st, False, False)


def test_path_group_split_along_k(imq):
    """K = 140000 at b = 8: the e = 0 group could overflow one int32 accumulator (140000 * 127^2 >= 2^31)
    and the bound does not rule it out, so the plan splits the group along K into two jobs."""
    rng = np.random.default_rng(14)
    A = rng.integers(-32767, 32768, size=(8, 140000)).astype(np.int64)
    B = rng.integers(-32767, 32768, size=(140000, 16)).astype(np.int64)
    plan = _run_path(imq, A, B, 8, 0, False, True)
    assert plan.info["acc_bits"] == 64


def test_path_int32_inputs(imq):
    rng = np.random.default_rng(9)
    A, B = workloads.random_case(rng, 130, 260, 270, big=100000, frac=0.01)
    _run_path(imq, A, B, 8, 0, True, False, dtype=torch.int32)


def test_gemm_rejects_int32_output_when_bound_exceeds(imq):
    rng = np.random.default_rng(10)
    A, B = workloads.random_case(rng, 64, 256, 64, big=30000, frac=0.05)
    pl = oracle.plan(A, B, 8, 0)
    assert not pl.bound_lt_2_31
    Ad = torch.from_numpy(A.astype(np.int16)).cuda()
    Bd = torch.from_numpy(B.astype(np.int16)).cuda()
    plan = imq.imq_plan(Ad, Bd, 8, 0)
    with pytest.raises(imq.ImqError) as e:
        imq.imq_unpacked_gemm(plan, Ad, Bd, c_dtype=torch.int32, want_f32=False)
    assert e.value.status == imq.IMQ_ERR_RANGE


def test_unpacked_gemm_workspace_checks(imq):
    rng = np.random.default_rng(11)
    A, B = workloads.random_case(rng, 40, 90, 50, big=200, frac=0.1)
    Ad = torch.from_numpy(A.astype(np.int16)).cuda()
    Bd = torch.from_numpy(B.astype(np.int16)).cuda()
    plan = imq.imq_plan(Ad, Bd, 4, 0)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(imq.ImqError) as e:
        imq.imq_unpacked_gemm(plan, Ad, Bd, workspace=small, want_f32=False)
    assert e.value.status == imq.IMQ_ERR_BUFFER
    C, _ = imq.imq_unpacked_gemm(plan, Ad, Bd, want_f32=False)
    assert np.array_equal(C.cpu().numpy().astype(np.int64), oracle.gemm_i64(A, B))


def test_plan_uses_given_line_maxima(imq):
    rng = np.random.default_rng(12)
    A, B = workloads.random_case(rng, 100, 200, 150, big=500, frac=0.05)
    Ad = torch.from_numpy(A.astype(np.int16)).cuda()
    Bd = torch.from_numpy(B.astype(np.int16)).cuda()
    mx = [torch.from_numpy(v.astype(np.int32)).cuda() for v in
          (np.abs(A).max(1), np.abs(A).max(0), np.abs(B).max(1), np.abs(B).max(0))]
    p1 = imq.imq_plan(Ad, Bd, 5, 0)
    p2 = imq.imq_plan(Ad, Bd, 5, 0, maxes=mx)
    assert p1.info == p2.info


def test_repeatable(imq):
    rng = np.random.default_rng(13)
    A, B = workloads.random_case(rng, 300, 700, 600, big=2000, frac=0.05)
    Ad = torch.from_numpy(A.astype(np.int16)).cuda()
    Bd = torch.from_numpy(B.astype(np.int16)).cuda()
    plan = imq.imq_plan(Ad, Bd, 5, 0)
    C1, _ = imq.imq_unpacked_gemm(plan, Ad, Bd, want_f32=False)
    C2, _ = imq.imq_unpacked_gemm(plan, Ad, Bd, want_f32=False)
    assert torch.equal(C1, C2)


@pytest.mark.parametrize("strategy", [0, 1, 4, 6])
@pytest.mark.parametrize("transB", [False, True])
def test_plan_unpack_matches_plan_then_unpack(imq, strategy, transB):
    """imq_plan_unpack: the same plan and the same unpacked bytes as imq_plan followed by imq_unpack, and
    the exact product through imq_gemm_unpacked on its workspace views."""
    rng = np.random.default_rng(31 + strategy)
    A, B = workloads.rows_and_cols_case(rng, 200, 300, 150, big=3000, dense_rows=2, dense_cols=2)
    Ad = torch.from_numpy(A.astype(np.int16)).cuda()
    Bd = torch.from_numpy(np.ascontiguousarray(B.T if transB else B).astype(np.int16)).cuda()
    ref = imq.imq_plan(Ad, Bd, 5, strategy, transB=transB)
    rAu, rBu = imq.imq_unpack(ref, Ad, Bd)
    ws = imq.workspace_for(ref)
    plan, Au, Bu = imq.imq_plan_unpack(Ad, Bd, 5, strategy, transB=transB, workspace=ws)
    assert plan.info == ref.info
    assert torch.equal(Au, rAu) and torch.equal(Bu, rBu)
    C, _ = imq.imq_gemm_unpacked(plan, Au, Bu, want_f32=False, c_dtype=torch.int64)
    torch.cuda.synchronize()
    assert imq.imq_device_status() == imq.IMQ_OK
    assert np.array_equal(C.cpu().numpy(), oracle.gemm_i64(A, B))


def test_plan_unpack_small_workspace(imq):
    """A workspace below the plan's size: a valid plan, nothing written, IMQ_ERR_BUFFER turned into
    (plan, None, None); without a workspace the same."""
    rng = np.random.default_rng(41)
    A, B = workloads.random_case(rng, 64, 96, 80, big=3000, frac=0.05)
    Ad = torch.from_numpy(A.astype(np.int16)).cuda()
    Bd = torch.from_numpy(B.astype(np.int16)).cuda()
    small = torch.full((4096,), 7, dtype=torch.uint8, device="cuda")
    plan, Au, Bu = imq.imq_plan_unpack(Ad, Bd, 4, 0, workspace=small)
    assert Au is None and Bu is None and plan.info["workspace_bytes"] > 4096 - 1024
    torch.cuda.synchronize()
    assert bool((small == 7).all())
    plan2, Au2, _ = imq.imq_plan_unpack(Ad, Bd, 4, 0)
    assert Au2 is None and plan2.info == plan.info
    Au, Bu = imq.imq_unpack(plan, Ad, Bd)
    C, _ = imq.imq_gemm_unpacked(plan, Au, Bu, want_f32=False, c_dtype=torch.int64)
    assert np.array_equal(C.cpu().numpy(), oracle.gemm_i64(A, B))
