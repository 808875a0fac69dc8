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


def _scratch_needed(rows, cols, itemsize, sms):
    """Bytes of partial column maxima the per-row kernel writes (its launch shape, restated)."""
    row_bytes = (cols * itemsize + 15) // 16 * 16
    cmax = (cols * 4 + 15) // 16 * 16
    budget = 200 * 1024
    if cmax + row_bytes > budget:
        return None
    nwarps = min((budget - cmax) // row_bytes, 8)
    smem = cmax + nwarps * row_bytes
    per_sm = min(max(budget // (smem + 8 * 384 * 4 + 1024), 1), 4)
    grid = min(rows, sms * per_sm)
    return grid * cols * 4


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
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rows, cols = 1024, 16384
    need = _scratch_needed(rows, cols, 2, sms)
    if need is None or need <= imq.IMQ_NOALLOC_SCRATCH_BYTES:
        pytest.skip(f"this device needs only {need} bytes for the rejected shape")
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
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rows, cols = 1000, 16384

    def fits(c):
        need = _scratch_needed(rows, c, 2, sms)
        return need is not None and need <= imq.IMQ_NOALLOC_SCRATCH_BYTES

    while not fits(cols):
        cols -= 8
    x = _input(8, rows, cols, "bf16")
    _same(imq.imq_rtn_quantize_rows_noalloc(x, 0.95, 15, out_dtype=torch.int32),
          imq.imq_rtn_quantize(x, imq.IMQ_PER_ROW, 0.95, 15, out_dtype=torch.int32))
    torch.cuda.synchronize()
    assert imq.imq_device_status(clear=True) == imq.IMQ_OK


def test_no_device_memory_is_allocated(imq):
    # outputs preallocated; a first pass loads every kernel the second pass launches
    shapes = [(512, 1024), (2048, 8192)]
    bufs = []
    for i, (r, c) in enumerate(shapes):
        x = _input(10 + i, r, c, "bf16")
        bufs.append(dict(X=x, Xint=torch.empty((r, c), dtype=torch.int16, device="cuda"),
                         delta=torch.empty(r, device="cuda"), qval=torch.empty(r, device="cuda"),
                         rowmax=torch.empty(r, dtype=torch.int32, device="cuda"),
                         colmax=torch.empty(c, dtype=torch.int32, device="cuda")))
    imq.imq_rtn_quantize_rows_noalloc(p=0.95, beta=15, **bufs[0])
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    # the second shape needs more scratch than the first: the allocating entry point would grow its buffer
    for b in bufs + bufs:
        imq.imq_rtn_quantize_rows_noalloc(p=0.95, beta=15, **b)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert imq.imq_device_status(clear=True) == imq.IMQ_OK
