"""The allocation-free per-row quantiser against the allocating one, through the C ABI.

imq_rtn_quantize_rows_noalloc runs the per-row kernel of imq_rtn_quantize with its partial column maxima
in a fixed device array, so every output must be identical to imq_rtn_quantize(g = IMQ_PER_ROW).  Each
test sets up what it uses, so the file passes alone in a fresh process as well as after the others.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def imq():
    import bit_integer_gemm_b200 as m
    assert torch.cuda.is_available(), "a GPU is required"
    m.lib()
    m.imq_device_status(clear=True)
    return m


def _input(seed, rows, cols, dtype):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)).astype(np.float32) * np.float32(rng.uniform(0.05, 5))
    if x.size:
        idx = rng.choice(x.size, max(1, x.size // 300), replace=False)
        x.reshape(-1)[idx] *= np.float32(60)
    t = torch.from_numpy(x).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _same(a, b):
    for name in ("xint", "delta", "qval", "rowmax", "colmax"):
        x, y = getattr(a, name), getattr(b, name)
        assert (x is None) == (y is None), name
        if x is not None:
            assert torch.equal(x, y), name


def _rejected(imq, rows, cols, dtype="bf16"):
    """True when the allocation-free call refuses this shape (IMQ_ERR_UNSUPPORTED: its scratch would
    exceed the fixed array).  A refused call launches nothing, so the output keeps its fill."""
    x = torch.zeros((rows, cols), dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device="cuda")
    xint = torch.full((rows, cols), 12345, dtype=torch.int16, device="cuda")
    try:
        imq.imq_rtn_quantize_rows_noalloc(x, 0.95, 15, Xint=xint)
    except imq.ImqError as e:
        assert e.status == imq.IMQ_ERR_UNSUPPORTED, e
        torch.cuda.synchronize()
        assert bool((xint == 12345).all()), "a refused call wrote its output"
        return True
    torch.cuda.synchronize()
    return False


def _widest_accepted(imq, rows, hi):
    """The widest bf16 row length (a multiple of 8, below hi) the call accepts for `rows` rows, found by
    bisection through the entry point itself (no launch constants restated here)."""
    lo = 8
    assert not _rejected(imq, rows, lo)
    while hi - lo > 8:
        mid = (lo + hi) // 16 * 8
        if _rejected(imq, rows, mid):
            hi = mid
        else:
            lo = mid
    return lo


PAIRS = [
    # two calls in a row with different shapes, so that a stale scratch slice would show
    (("bf16", 2048, 4096, torch.int16, 1), ("f32", 333, 1000, torch.int32, 2)),
    (("f32", 517, 1536, torch.int16, 3), ("bf16", 4096, 2048, torch.int16, 4)),
]


@pytest.mark.parametrize("pair", PAIRS, ids=["bf16_then_f32", "f32_then_bf16"])
def test_two_calls_in_a_row_match_the_allocating_entry_point(imq, pair):
    ins = [(_input(seed, r, c, dt), p, od) for (dt, r, c, od, seed), p in zip(pair, (0.95, 0.99))]
    beta = 15
    new = [imq.imq_rtn_quantize_rows_noalloc(x, p, beta, out_dtype=od) for x, p, od in ins]
    ref = [imq.imq_rtn_quantize(x, imq.IMQ_PER_ROW, p, beta, out_dtype=od) for x, p, od in ins]
    torch.cuda.synchronize()
    assert imq.imq_device_status(clear=True) == imq.IMQ_OK
    for a, b in zip(new, ref):
        _same(a, b)


def test_repeated_calls_on_one_stream(imq):
    x1 = _input(5, 1024, 4096, "bf16")
    x2 = _input(6, 1024, 4096, "bf16")
    ref1 = imq.imq_rtn_quantize(x1, imq.IMQ_PER_ROW, 0.95, 15)
    ref2 = imq.imq_rtn_quantize(x2, imq.IMQ_PER_ROW, 0.95, 15)
    for _ in range(2):
        _same(imq.imq_rtn_quantize_rows_noalloc(x1, 0.95, 15), ref1)
        _same(imq.imq_rtn_quantize_rows_noalloc(x2, 0.95, 15), ref2)
    torch.cuda.synchronize()
    assert imq.imq_device_status(clear=True) == imq.IMQ_OK


@pytest.mark.parametrize("rows,cols", [(0, 64), (64, 0), (0, 0)])
def test_empty(imq, rows, cols):
    x = torch.zeros((rows, cols), dtype=torch.float32, device="cuda")
    _same(imq.imq_rtn_quantize_rows_noalloc(x, 0.9, 7), imq.imq_rtn_quantize(x, imq.IMQ_PER_ROW, 0.9, 7))


def test_scratch_above_the_maximum_is_rejected_before_any_launch(imq):
    rows, cols = 1024, 16384
    if not _rejected(imq, rows, cols):
        pytest.skip("this device's launch shape fits the widest test row in the fixed array")
    x = _input(7, rows, cols, "bf16")
    xint = torch.full((rows, cols), 12345, dtype=torch.int16, device="cuda")
    with pytest.raises(imq.ImqError) as e:
        imq.imq_rtn_quantize_rows_noalloc(x, 0.95, 15, Xint=xint)
    assert e.value.status == imq.IMQ_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((xint == 12345).all()), "a rejected call wrote its output"
    # without column maxima no scratch is needed and the same shape runs
    got = imq.imq_rtn_quantize_rows_noalloc(x, 0.95, 15, colmax=None, want_max=False)
    ref = imq.imq_rtn_quantize(x, imq.IMQ_PER_ROW, 0.95, 15, want_max=False)
    _same(got, ref)


def test_shape_near_the_maximum(imq):
    """The widest accepted row length for 1000 rows runs and matches the allocating entry point; 8 more
    columns are refused."""
    rows = 1000
    if not _rejected(imq, rows, 16384):
        pytest.skip("this device's launch shape fits the widest test row in the fixed array")
    cols = _widest_accepted(imq, rows, 16384)
    assert _rejected(imq, rows, cols + 8)
    x = _input(8, rows, cols, "bf16")
    _same(imq.imq_rtn_quantize_rows_noalloc(x, 0.95, 15, out_dtype=torch.int32),
          imq.imq_rtn_quantize(x, imq.IMQ_PER_ROW, 0.95, 15, out_dtype=torch.int32))
    torch.cuda.synchronize()
    assert imq.imq_device_status(clear=True) == imq.IMQ_OK


# Run in a fresh process: no allocating call of the library may come first there, so the library's
# memory pool holds nothing that a pool allocation could reuse unseen.  The first call loads the
# kernels; then two passes over two shapes (the second needing more scratch than the first) must leave
# the device's free memory unchanged.
_FRESH = r"""
import sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1])
import bit_integer_gemm_b200 as imq
imq.lib()
bufs = []
for i, (r, c) in enumerate([(512, 1024), (2048, 8192)]):
    rng = np.random.default_rng(10 + i)
    x = torch.from_numpy(rng.standard_normal((r, c)).astype(np.float32)).cuda().to(torch.bfloat16)
    bufs.append(dict(X=x, Xint=torch.empty((r, c), dtype=torch.int16, device="cuda"),
                     delta=torch.empty(r, device="cuda"), qval=torch.empty(r, device="cuda"),
                     rowmax=torch.empty(r, dtype=torch.int32, device="cuda"),
                     colmax=torch.empty(c, dtype=torch.int32, device="cuda")))
imq.imq_rtn_quantize_rows_noalloc(p=0.95, beta=15, **bufs[0])
torch.cuda.synchronize()
free0 = torch.cuda.mem_get_info()[0]
for b in bufs + bufs:
    imq.imq_rtn_quantize_rows_noalloc(p=0.95, beta=15, **b)
torch.cuda.synchronize()
free1 = torch.cuda.mem_get_info()[0]
assert imq.imq_device_status(clear=True) == imq.IMQ_OK
print("FREE", free0, free1)
"""


def test_no_device_memory_is_allocated(imq):
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", _FRESH, root], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    line = [ln for ln in out.stdout.splitlines() if ln.startswith("FREE")][-1]
    free0, free1 = (int(v) for v in line.split()[1:])
    assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"
