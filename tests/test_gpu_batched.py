"""Batches of equal-shaped GEMMs through imq_plan_batched / imq_unpack_batched / imq_gemm_unpacked_batched:
every problem of a batch against the CPU oracle (plan fields, every unpacked byte through the library's
maps, the exact product and its dequantisation), and against the same problem planned alone.  The full
attention workload (32 heads of Q.K^T and of P.V) runs here in one batch per GEMM, all heads compared.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_common import assert_f32_close, check_unpacked, plan_matches

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def imq():
    import bit_integer_gemm_b200 as m
    assert torch.cuda.is_available(), "a GPU is required"
    m.lib()
    m.imq_device_status(clear=True)
    return m


def _run_batch(imq, As, Bs, b, strategy, transB, dtype=torch.int16, compare_single=True):
    """As, Bs: lists of logical int64 matrices of one shape.  Stacks them (A row-major M x K per problem;
    B stored K x N, or N x K when transB), runs the batched calls and checks every problem."""
    n = len(As)
    M, K = As[0].shape
    N = Bs[0].shape[1]
    npdt = np.int16 if dtype == torch.int16 else np.int32
    A_st = np.concatenate([a.astype(npdt) for a in As], axis=0)
    B_st = np.concatenate([(bb.T if transB else bb).astype(npdt) for bb in Bs], axis=0)
    Ad = torch.from_numpy(np.ascontiguousarray(A_st)).cuda()
    Bd = torch.from_numpy(np.ascontiguousarray(B_st)).cuda()
    pls = [oracle.plan(a, bb, b, strategy) for a, bb in zip(As, Bs)]
    batch = imq.imq_plan_batched(Ad, Bd, n, M, K, N, b, strategy, transB=transB)
    for h in range(n):
        plan_matches(batch[h].info, pls[h], batch[h].groups())
    ws = imq.batch_workspace(batch)
    imq.imq_unpack_batched(batch, Ad, Bd, ws)
    views = imq.batch_views(batch, ws)
    wide = any(p.acc_bits == 64 for p in pls)
    C = torch.empty((n, M, N), dtype=torch.int64 if wide else torch.int32, device="cuda")
    Cf = torch.empty((n, M, N), dtype=torch.float32, device="cuda")
    rng = np.random.default_rng(n * 13 + M + N)
    dA = rng.uniform(1e-3, 1.0, n * M).astype(np.float32)
    dB = rng.uniform(1e-3, 1.0, n * N).astype(np.float32)
    imq.imq_gemm_unpacked_batched(batch, ws, torch.from_numpy(dA).cuda(), M, imq.IMQ_PER_ROW,
                                  torch.from_numpy(dB).cuda(), N, imq.IMQ_PER_COL, C, Cf)
    torch.cuda.synchronize()
    assert imq.imq_device_status() == imq.IMQ_OK
    for h in range(n):
        Au, Bu = views[h]
        check_unpacked(batch[h], pls[h], Au.cpu().numpy(), Bu.cpu().numpy(), As[h], Bs[h])
        want = oracle.gemm_exact(As[h], Bs[h])
        assert np.array_equal(C[h].cpu().numpy().astype(np.int64), want), f"problem {h}"
        assert_f32_close(Cf[h].cpu().numpy(),
                         oracle.dequant(want, dA[h * M:(h + 1) * M], oracle.PER_ROW, dB[h * N:(h + 1) * N],
                                        oracle.PER_COL))
    if compare_single:
        # the same problems planned one by one: same plans, same bytes
        for h in range(n):
            one = imq.imq_plan(Ad[h * M:(h + 1) * M], Bd[h * B_st.shape[0] // n:(h + 1) * B_st.shape[0] // n], b,
                               strategy, transB=transB)
            assert one.info == batch[h].info
            Au1, Bu1 = imq.imq_unpack(one, Ad[h * M:(h + 1) * M], Bd[h * B_st.shape[0] // n:(h + 1) * B_st.shape[0] // n])
            assert torch.equal(Au1, views[h][0]) and torch.equal(Bu1, views[h][1])
            one.destroy()
    batch.destroy()


@pytest.mark.parametrize("strategy", [0, 1, 2, 3, 4, 5, 6])
@pytest.mark.parametrize("transB", [False, True])
def test_batch_random_problems(imq, strategy, transB):
    rng = np.random.default_rng(100 + 2 * strategy + transB)
    n, M, K, N = 5, 150, 260, 90
    cases = [workloads.random_case(rng, M, K, N, big=int(rng.choice([300, 3000])), frac=0.05) for _ in range(n)]
    _run_batch(imq, [c[0] for c in cases], [c[1] for c in cases], 5, strategy, transB)


@pytest.mark.parametrize("dtype", [torch.int16, torch.int32])
def test_batch_heads_with_different_directions_and_split_k(imq, dtype):
    """Problems whose Mix choices differ (some A unpacked OUTER, some INNER), with few output tiles and a
    long inner dimension, so that the GEMM splits K; int16 and int32 sources."""
    rng = np.random.default_rng(7 if dtype == torch.int16 else 8)
    M, K, N, b = 64, 3000, 40, 4
    As, Bs = [], []
    for h in range(6):
        A = rng.integers(-5, 6, size=(M, K)).astype(np.int64)
        B = rng.integers(-5, 6, size=(K, N)).astype(np.int64)
        if h % 2:
            A[rng.choice(M, 3, replace=False), :] *= 200   # a few heavy rows: OUTER
        else:
            A[:, rng.choice(K, 3, replace=False)] *= 200   # a few heavy columns: INNER
        As.append(A)
        Bs.append(B)
    dirs = {oracle.plan(a, bb, b, 0).dir_a for a, bb in zip(As, Bs)}
    assert dirs == {oracle.DIR_OUTER, oracle.DIR_INNER}
    _run_batch(imq, As, Bs, b, 0, True, dtype=dtype)


def test_batch_rejects_mixed_plans_and_small_workspace(imq):
    rng = np.random.default_rng(9)
    A, B = workloads.random_case(rng, 40, 64, 30, big=500, frac=0.1)
    Ad = torch.from_numpy(np.concatenate([A, A]).astype(np.int16)).cuda()
    Bd = torch.from_numpy(np.concatenate([B, B]).astype(np.int16)).cuda()
    batch = imq.imq_plan_batched(Ad, Bd, 2, 40, 64, 30, 5)
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(imq.ImqError) as e:
        imq.imq_unpack_batched(batch, Ad, Bd, small)
    assert e.value.status == imq.IMQ_ERR_BUFFER
    other = imq.imq_plan(Ad[:40, :32], Bd[:32], 5)  # another shape
    mixed = imq.PlanBatch([batch[0], other], Ad, Bd)
    ws = imq.batch_workspace(batch)
    with pytest.raises(imq.ImqError) as e:
        imq.imq_unpack_batched(mixed, Ad, Bd, ws)
    assert e.value.status == imq.IMQ_ERR_ARG
    other.destroy()
    batch.destroy()


# ------------------------------------------------------------------------------------------------
# the attention workload: 32 heads, batch 1, seq 2048, head dim 128
# ------------------------------------------------------------------------------------------------
def _attention_inputs(heads=32):
    gs = [workloads.attention_head(h) for h in range(heads)]
    Q = np.concatenate([g[0].A.data for g in gs])          # (heads * seq) x dim, head-major
    Kt = np.concatenate([g[0].B.data for g in gs])         # (heads * seq) x dim
    P = np.concatenate([g[1].A.data for g in gs])          # (heads * seq) x seq
    V = np.concatenate([g[1].B.data for g in gs], axis=1)  # seq x (heads * dim)
    return gs, Q, Kt, P, V


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("which", ["qk", "pv"])
def test_config_attention_all_heads_batched(imq, which):
    heads, seq, dim = 32, 2048, 128
    gs, Q, Kt, P, V = _attention_inputs(heads)
    g0 = gs[0][0 if which == "qk" else 1]
    p, beta, b = g0.p, g0.beta, g0.b
    if which == "qk":
        # A = Q per row (head-major stack: per row = per head and token); B = K^T, K stored per row
        qa_np = [oracle.rtn_quantize(oracle.as_f32(g[0].A.data, "bf16"), oracle.PER_ROW, p, beta) for g in gs]
        qb_np = [oracle.rtn_quantize(oracle.as_f32(g[0].B.data, "bf16"), oracle.PER_ROW, p, beta) for g in gs]
        wide = max(max(int(np.abs(x[0]).max()) for x in qa_np), max(int(np.abs(x[0]).max()) for x in qb_np)) > 32767
        dt = torch.int32 if wide else torch.int16
        qa = imq.imq_rtn_quantize(_dev(Q), imq.IMQ_PER_ROW, p, beta, out_dtype=dt)
        qb = imq.imq_rtn_quantize(_dev(Kt), imq.IMQ_PER_ROW, p, beta, out_dtype=dt)
        M, K, N = seq, dim, seq
        batch = imq.imq_plan_batched(qa.xint, qb.xint, heads, M, K, N, b, imq.IMQ_MIX, transB=True)
        As = [x[0] for x in qa_np]
        Bs = [x[0].T for x in qb_np]
        dAs = [x[1] for x in qa_np]
        dBs = [x[1] for x in qb_np]
        gB = imq.IMQ_PER_COL
        B_dev, sB = qb.xint, seq * dim
    else:
        # A = P per row; B = V per column, quantised straight into the (heads * dim) x seq layout
        qa_np = [oracle.rtn_quantize(oracle.as_f32(g[1].A.data, "bf16"), oracle.PER_ROW, p, beta) for g in gs]
        qb_np = [oracle.rtn_quantize(oracle.as_f32(g[1].B.data, "bf16"), oracle.PER_COL, p, beta) for g in gs]
        wide = max(max(int(np.abs(x[0]).max()) for x in qa_np), max(int(np.abs(x[0]).max()) for x in qb_np)) > 32767
        dt = torch.int32 if wide else torch.int16
        qa = imq.imq_rtn_quantize(_dev(P), imq.IMQ_PER_ROW, p, beta, out_dtype=dt)
        qb = imq.imq_rtn_quantize(_dev(V), imq.IMQ_PER_COL, p, beta, out_dtype=dt, trans_out=True)
        M, K, N = seq, seq, dim
        batch = imq.imq_plan_batched(qa.xint, qb.xint, heads, M, K, N, b, imq.IMQ_MIX, transB=True)
        As = [x[0] for x in qa_np]
        Bs = [x[0] for x in qb_np]
        dAs = [x[1] for x in qa_np]
        dBs = [x[1] for x in qb_np]
        gB = imq.IMQ_PER_COL
        B_dev, sB = qb.xint, dim * seq
    torch.cuda.synchronize()
    assert imq.imq_device_status() == imq.IMQ_OK
    for h in range(heads):
        assert np.array_equal(qa.xint[h * M:(h + 1) * M].cpu().numpy().astype(np.int64), As[h]), f"head {h} A ints"
        Bst = qb.xint[h * (N if which == "qk" else dim):(h + 1) * (N if which == "qk" else dim)].cpu().numpy()
        assert np.array_equal(Bst.astype(np.int64).T, Bs[h]), f"head {h} B ints"
    ws = imq.batch_workspace(batch)
    imq.imq_unpack_batched(batch, qa.xint, B_dev, ws, strideA=M * qa.xint.shape[1], strideB=sB)
    views = imq.batch_views(batch, ws)
    wide_c = any(batch[h].info["acc_bits"] == 64 for h in range(heads))
    C = torch.empty((heads, M, N), dtype=torch.int64 if wide_c else torch.int32, device="cuda")
    Cf = torch.empty((heads, M, N), dtype=torch.float32, device="cuda")
    imq.imq_gemm_unpacked_batched(batch, ws, qa.delta, M, imq.IMQ_PER_ROW, qb.delta, N, gB, C, Cf)
    torch.cuda.synchronize()
    assert imq.imq_device_status() == imq.IMQ_OK
    for h in range(heads):
        pl = oracle.plan(As[h], Bs[h], b, oracle.MIX)
        plan_matches(batch[h].info, pl, batch[h].groups())
        Au, Bu = views[h]
        check_unpacked(batch[h], pl, Au.cpu().numpy(), Bu.cpu().numpy(), As[h], Bs[h])
        want = oracle.gemm_exact(As[h], Bs[h])
        assert np.array_equal(C[h].cpu().numpy().astype(np.int64), want), f"head {h} C"
        assert_f32_close(Cf[h].cpu().numpy(), oracle.dequant(want, dAs[h], oracle.PER_ROW, dBs[h], oracle.PER_COL))
    batch.destroy()
