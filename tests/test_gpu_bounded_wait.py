"""A bounded wait that runs out: the library's wait helper (every wait of the GEMM goes through it) on an
mbarrier that nothing arrives at gives up after its limit, the kernel returns, the device status word
reads IMQ_ERR_TIMEOUT, and the context stays usable (a GEMM afterwards is exact and leaves the status
clear)."""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def imq():
    import bit_integer_gemm_b200 as m
    assert torch.cuda.is_available(), "a GPU is required"
    m.lib()
    m.imq_device_status(clear=True)
    return m


def test_bounded_wait_runs_out_and_reports(imq):
    t0 = time.perf_counter()
    imq.imq_check_bounded_wait(20_000_000)  # 20 ms
    torch.cuda.synchronize()
    took = time.perf_counter() - t0
    assert imq.imq_device_status(clear=True) == imq.IMQ_ERR_TIMEOUT
    assert 0.015 < took < 5.0
    # the context is still usable: an exact GEMM, status clear
    rng = np.random.default_rng(7)
    A, B = workloads.random_case(rng, 200, 300, 150, big=500, frac=0.05)
    Ad = torch.from_numpy(A.astype(np.int16)).cuda()
    Bd = torch.from_numpy(B.astype(np.int16)).cuda()
    plan = imq.imq_plan(Ad, Bd, 5, imq.IMQ_MIX)
    C, _ = imq.imq_unpacked_gemm(plan, Ad, Bd, want_f32=False)
    torch.cuda.synchronize()
    assert imq.imq_device_status() == imq.IMQ_OK
    assert np.array_equal(C.cpu().numpy().astype(np.int64), oracle.gemm_exact(A, B))
    plan.destroy()


def test_bounded_wait_limits_are_checked(imq):
    for bad in (0, 999, 2_000_000_000):
        with pytest.raises(imq.ImqError) as e:
            imq.imq_check_bounded_wait(bad)
        assert e.value.status == imq.IMQ_ERR_ARG
