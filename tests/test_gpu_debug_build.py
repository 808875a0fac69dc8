"""The IMQ_DEBUG build (libimq_debug.so, loaded with IMQ_LIB=debug): after every plan a kernel checks each
index the unpack and GEMM kernels read -- inner source indices and levels, exponent groups and padding,
run blocks, OUTER line positions, sources and groups -- against the plan's sizes, and reports a violation
as IMQ_ERR_BOUNDS in the status word.  The small parity cases run here under it in a child process (the
library a process loads is fixed at its first call): every status must stay IMQ_OK and every result must
equal the oracle's."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_CASES = r"""
import sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1])
import bit_integer_gemm_b200 as imq
import oracle
import workloads
from tests.gpu_common import check_unpacked, plan_matches
assert imq.LIB_PATH.endswith("libimq_debug.so"), imq.LIB_PATH
imq.lib()
rng = np.random.default_rng(2024)
n = 0
for case in range(60):
    M, K, N = (int(x) for x in rng.integers(1, 300, size=3))
    b = int(rng.integers(2, 9))
    st = case % 7
    transA, transB = bool(case % 3 == 1), bool(case % 4 >= 2)
    if case % 2:
        A, B = workloads.rows_and_cols_case(rng, M, K, N, big=int(rng.choice([100, 3000])), dense_rows=2, dense_cols=2)
    else:
        A, B = workloads.random_case(rng, M, K, N, big=int(rng.choice([60, 3000])), frac=0.1)
    pl = oracle.plan(A, B, b, st)
    if int(round(pl.bound)) >= 2 ** 63:
        continue
    dt = np.int32 if case % 5 == 0 else np.int16
    Ad = torch.from_numpy(np.ascontiguousarray(A.T if transA else A).astype(dt)).cuda()
    Bd = torch.from_numpy(np.ascontiguousarray(B.T if transB else B).astype(dt)).cuda()
    plan = imq.imq_plan(Ad, Bd, b, st, transA, transB)
    plan_matches(plan.info, pl, plan.groups())
    Au, Bu = imq.imq_unpack(plan, Ad, Bd)
    C, _ = imq.imq_gemm_unpacked(plan, Au, Bu, c_dtype=torch.int64, want_f32=False)
    torch.cuda.synchronize()
    s = imq.imq_device_status(clear=True)
    assert s == imq.IMQ_OK, (case, imq.imq_status_str(s))
    check_unpacked(plan, pl, Au.cpu().numpy(), Bu.cpu().numpy(), A, B)
    assert np.array_equal(C.cpu().numpy(), oracle.gemm_exact(A, B)), case
    plan.destroy()
    n += 1
# a batch planned together
As, Bs = zip(*[workloads.random_case(rng, 70, 200, 50, big=3000, frac=0.05) for _ in range(4)])
Ad = torch.from_numpy(np.ascontiguousarray(np.concatenate(As)).astype(np.int16)).cuda()
Bd = torch.from_numpy(np.ascontiguousarray(np.concatenate([x.T for x in Bs])).astype(np.int16)).cuda()
batch = imq.imq_plan_batched(Ad, Bd, 4, 70, 200, 50, 5, imq.IMQ_MIX, transB=True)
ws = imq.batch_workspace(batch)
imq.imq_unpack_batched(batch, Ad, Bd, ws)
C = torch.empty((4, 70, 50), dtype=torch.int64, device="cuda")
imq.imq_gemm_unpacked_batched(batch, ws, None, 0, 0, None, 0, 0, C, None)
torch.cuda.synchronize()
assert imq.imq_device_status(clear=True) == imq.IMQ_OK
for h in range(4):
    assert np.array_equal(C[h].cpu().numpy(), oracle.gemm_exact(As[h], Bs[h]))
print("CASES", n)
"""


def test_small_parity_cases_under_the_debug_build():
    lib = os.path.join(ROOT, "bit_integer_gemm_b200", "libimq_debug.so")
    if not os.path.exists(lib):
        from bit_integer_gemm_b200 import build as b
        b.build(debug=True)
    env = dict(os.environ, IMQ_LIB="debug")
    out = subprocess.run([sys.executable, "-c", _CASES, ROOT], capture_output=True, text=True, timeout=900, env=env,
                         cwd=ROOT)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-4000:]
    n = int([ln for ln in out.stdout.splitlines() if ln.startswith("CASES")][-1].split()[1])
    assert n >= 50
