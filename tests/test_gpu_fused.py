"""Fused per-row RTN + unpack of the activations into a kept plan's A' layout (imq_rtn_quantize_unpack),
with the weight quantised, planned and unpacked once: the A' bytes and row scales equal the separate
quantise-then-unpack path and the oracle's, the GEMM with the kept B'^T is the exact product, and inputs
outside the plan's column maxima are reported as IMQ_ERR_PLAN."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_common import assert_f32_close, check_unpacked, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def imq():
    import bit_integer_gemm_b200 as m
    assert torch.cuda.is_available(), "a GPU is required"
    m.lib()
    m.imq_device_status(clear=True)
    return m


def _levels(v, b):
    R = 1 << (b - 1)
    L = np.ones_like(v)
    t = np.abs(v) // R
    while (t > 0).any():
        L += (t > 0)
        t //= R
    return L


def _weight(imq, W, p, beta):
    """W stored K x N, quantised per output channel straight into N x K (B given transposed)."""
    return imq.imq_rtn_quantize(W, imq.IMQ_PER_COL, p, beta, trans_out=True)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(1, 16, 1), (37, 129, 50), (64, 1000, 96), (300, 520, 270), (128, 4096, 64)])
@pytest.mark.parametrize("b", [3, 5])
def test_fused_matches_separate_path_and_oracle(imq, dtype, shape, b):
    M, K, N = shape
    rng = np.random.default_rng(M * 31 + K * 7 + N + b)
    X = rng.standard_normal((M, K), dtype=np.float32)
    X[:, rng.choice(K, min(3, K), replace=False)] *= np.float32(40)
    W = (rng.standard_normal((K, N), dtype=np.float32) * np.float32(0.02))
    Xs = workloads.Stored("X", workloads.f32_to_bf16_bits(X) if dtype == "bf16" else X, dtype)
    Ws = workloads.Stored("W", workloads.f32_to_bf16_bits(W), "bf16")
    Xd, Wd = to_device(Xs), to_device(Ws)
    p, beta = 0.95, 15
    qx = imq.imq_rtn_quantize(Xd, imq.IMQ_PER_ROW, p, beta)
    qw = _weight(imq, Wd, p, beta)
    plan = imq.imq_plan(qx.xint, qw.xint, b, imq.IMQ_COL_ROW, transB=True,
                        maxes=(qx.rowmax, qx.colmax, qw.rowmax, qw.colmax))
    Au, Bu = imq.imq_unpack(plan, qx.xint, qw.xint)
    Af, dAf = imq.imq_rtn_quantize_unpack(plan, Xd, p, beta)
    torch.cuda.synchronize()
    assert imq.imq_device_status(clear=True) == imq.IMQ_OK
    assert torch.equal(Af, Au), "fused A' differs from quantise + unpack"
    assert torch.equal(dAf, qx.delta)
    # the oracle: RTN of X, unpacked in the oracle plan's layout
    xi, dx, _ = oracle.rtn_quantize(oracle.as_f32(Xs.data, dtype), oracle.PER_ROW, p, beta)
    wi, dw, _ = oracle.rtn_quantize(oracle.as_f32(Ws.data, "bf16"), oracle.PER_COL, p, beta)
    pl = oracle.plan(xi, wi, b, oracle.COL_ROW)
    check_unpacked(plan, pl, Af.cpu().numpy(), Bu.cpu().numpy(), xi, wi)
    assert np.array_equal(dAf.cpu().numpy(), dx)
    # the GEMM with the kept B'^T
    C, Cf = imq.imq_gemm_unpacked(plan, Af, Bu, dAf, imq.IMQ_PER_ROW, qw.delta, imq.IMQ_PER_COL)
    torch.cuda.synchronize()
    want = oracle.gemm_exact(xi, wi)
    assert np.array_equal(C.cpu().numpy().astype(np.int64), want)
    assert_f32_close(Cf.cpu().numpy(), oracle.dequant(want, dx, oracle.PER_ROW, dw, oracle.PER_COL))
    plan.destroy()


def _class_ordered(plan):
    """True when some segment of the plan's inner layout is not in index order (the plan grouped its inner
    indices by level class: the staging order)."""
    mp = plan.maps()
    for e, off, n, padded in plan.groups():
        t = mp["tK"][off:off + n].astype(np.int64)
        la = mp["lAk"][off:off + n].astype(np.int64)
        key = la * (1 << 32) + t
        if not np.all(np.diff(key) > 0):
            return True
    return False


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fused_with_class_ordered_plan(imq, dtype):
    """A plan whose inner indices are grouped by level class (half the columns of X and half the rows of W
    scaled down, so that every segment beyond the first is about half dense): the fused path stages its
    int16 row in that order and must still equal the separate path, the oracle and the exact product."""
    M, K, N, b, p, beta = 300, 520, 270, 3, 0.95, 15
    rng = np.random.default_rng(2024)
    X = rng.standard_normal((M, K), dtype=np.float32)
    X[:, rng.permutation(K)[:K // 2]] *= np.float32(0.4)
    W = rng.standard_normal((K, N), dtype=np.float32) * np.float32(0.02)
    W[rng.permutation(K)[:K // 2], :] *= np.float32(0.4)
    Xs = workloads.Stored("X", workloads.f32_to_bf16_bits(X) if dtype == "bf16" else X, dtype)
    Ws = workloads.Stored("W", workloads.f32_to_bf16_bits(W), "bf16")
    Xd, Wd = to_device(Xs), to_device(Ws)
    qx = imq.imq_rtn_quantize(Xd, imq.IMQ_PER_ROW, p, beta)
    qw = _weight(imq, Wd, p, beta)
    plan = imq.imq_plan(qx.xint, qw.xint, b, imq.IMQ_COL_ROW, transB=True,
                        maxes=(qx.rowmax, qx.colmax, qw.rowmax, qw.colmax))
    assert _class_ordered(plan), "the case was built to take the class-grouped order"
    Au, Bu = imq.imq_unpack(plan, qx.xint, qw.xint)
    Af, dAf = imq.imq_rtn_quantize_unpack(plan, Xd, p, beta)
    torch.cuda.synchronize()
    assert imq.imq_device_status(clear=True) == imq.IMQ_OK
    assert torch.equal(Af, Au), "fused A' differs from quantise + unpack"
    xi, dx, _ = oracle.rtn_quantize(oracle.as_f32(Xs.data, dtype), oracle.PER_ROW, p, beta)
    wi, dw, _ = oracle.rtn_quantize(oracle.as_f32(Ws.data, "bf16"), oracle.PER_COL, p, beta)
    pl = oracle.plan(xi, wi, b, oracle.COL_ROW)
    check_unpacked(plan, pl, Af.cpu().numpy(), Bu.cpu().numpy(), xi, wi)
    C, Cf = imq.imq_gemm_unpacked(plan, Af, Bu, dAf, imq.IMQ_PER_ROW, qw.delta, imq.IMQ_PER_COL)
    torch.cuda.synchronize()
    want = oracle.gemm_exact(xi, wi)
    assert np.array_equal(C.cpu().numpy().astype(np.int64), want)
    assert_f32_close(Cf.cpu().numpy(), oracle.dequant(want, dx, oracle.PER_ROW, dw, oracle.PER_COL))
    plan.destroy()


def test_fused_q_proj_kept_weight_new_batches(imq):
    """q_proj shapes: the plan is made once with widened column maxima (each raised to the largest value
    with the same number of base-R digits, R^L - 1) and W' is unpacked once; three new activation batches
    with the same heavy channels then go through the fused path and the GEMM.  Each result equals the
    exact product of the oracle's quantised batch with W, or the status reports that the batch left the
    widened maxima (checked against the oracle's quantised values)."""
    g = workloads.q_proj()[0]
    Wd = to_device(g.B)
    qw = _weight(imq, Wd, g.p, g.beta)
    wi, dw, _ = oracle.rtn_quantize(oracle.as_f32(g.B.data, "bf16"), oracle.PER_COL, g.p, g.beta)
    X0 = to_device(g.A)
    qx0 = imq.imq_rtn_quantize(X0, imq.IMQ_PER_ROW, g.p, g.beta)
    R = 1 << (g.b - 1)
    L = _levels(qx0.colmax.cpu().numpy().astype(np.int64), g.b)
    widened_np = (R ** L - 1).astype(np.int64)
    widened = torch.from_numpy(np.minimum(widened_np, 32767).astype(np.int32)).cuda()
    plan = imq.imq_plan(qx0.xint, qw.xint, g.b, imq.IMQ_MIX, transB=True,
                        maxes=(qx0.rowmax, widened, qw.rowmax, qw.colmax))
    assert plan.info["dir_a"] == imq.IMQ_DIR_INNER
    _, Bu = imq.imq_unpack(plan, qx0.xint, qw.xint)
    rng = np.random.default_rng(77)
    ch = np.flatnonzero(oracle.as_f32(g.A.data, "bf16").std(axis=0) > 10)  # the heavy channels of the workload
    covered = 0
    for k in range(3):
        Xn = rng.standard_normal((g.M, g.K), dtype=np.float32)
        Xn[:, ch] *= np.float32(60)
        Xs = workloads.Stored("X", workloads.f32_to_bf16_bits(Xn), "bf16")
        Af, dAf = imq.imq_rtn_quantize_unpack(plan, to_device(Xs), g.p, g.beta)
        xi, dx, _ = oracle.rtn_quantize(oracle.as_f32(Xs.data, "bf16"), oracle.PER_ROW, g.p, g.beta)
        inside = bool(np.all(np.abs(xi) <= np.minimum(widened_np, 32767)[None, :]))
        C, Cf = imq.imq_gemm_unpacked(plan, Af, Bu, dAf, imq.IMQ_PER_ROW, qw.delta, imq.IMQ_PER_COL)
        torch.cuda.synchronize()
        st = imq.imq_device_status(clear=True)
        if not inside:
            assert st == imq.IMQ_ERR_PLAN
            continue
        assert st == imq.IMQ_OK
        covered += 1
        assert np.array_equal(dAf.cpu().numpy(), dx)
        rows = np.arange(k, g.M, 7)
        want = oracle.gemm_exact(xi[rows], wi)
        assert np.array_equal(C.cpu().numpy()[rows].astype(np.int64), want)
        assert_f32_close(Cf.cpu().numpy()[rows], oracle.dequant(want, dx[rows], oracle.PER_ROW, dw, oracle.PER_COL))
    assert covered >= 1
    plan.destroy()


def test_fused_reports_uncovered_input_and_refuses_outer_plans(imq):
    rng = np.random.default_rng(5)
    M, K, N, b = 64, 256, 32, 5
    X = rng.standard_normal((M, K), dtype=np.float32)
    W = rng.standard_normal((K, N), dtype=np.float32)
    Xd = torch.from_numpy(X).cuda()
    Wd = torch.from_numpy(W).cuda()
    qx = imq.imq_rtn_quantize(Xd, imq.IMQ_PER_ROW, 0.95, 15)
    qw = _weight(imq, Wd, 0.95, 15)
    plan = imq.imq_plan(qx.xint, qw.xint, b, imq.IMQ_COL_ROW, transB=True)
    X2 = X.copy()
    X2[:, 7] *= 100.0  # a new heavy channel: its entries leave the plan's column maximum
    imq.imq_rtn_quantize_unpack(plan, torch.from_numpy(X2).cuda(), 0.95, 15)
    torch.cuda.synchronize()
    assert imq.imq_device_status(clear=True) == imq.IMQ_ERR_PLAN
    # the same batch as the plan's is covered
    imq.imq_rtn_quantize_unpack(plan, Xd, 0.95, 15)
    torch.cuda.synchronize()
    assert imq.imq_device_status(clear=True) == imq.IMQ_OK
    plan.destroy()
    outer = imq.imq_plan(qx.xint, qw.xint, b, imq.IMQ_ROW_ROW, transB=True)
    with pytest.raises(imq.ImqError) as e:
        imq.imq_rtn_quantize_unpack(outer, Xd, 0.95, 15)
    assert e.value.status == imq.IMQ_ERR_ARG
    outer.destroy()
