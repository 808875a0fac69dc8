"""Python binding of libimq.so, the B200 (sm_100a) IM-Unpack exact low-bit integer GEMM.

Every function here has the name of the C entry point it calls (include/imq.h) and only marshals
arguments: it takes torch CUDA tensors, allocates outputs that the caller did not pass, and raises
:class:`ImqError` on a non-OK status.  All arithmetic runs in the library's CUDA kernels.  There is no
fallback: without the built library every call raises.

Method: "IM-Unpack: Training and Inference with Arbitrarily Low Precision Integers" (atlas.scime.ai
summary), "Approach" -- RTN quantisation, per-matrix row/column unpacking of heavy hitters into b-bit
integers, b-bit integer GEMMs and bit-shift accumulation that reproduce the integer product exactly.
"""
from __future__ import annotations

import ctypes
import os
from collections import namedtuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# IMQ_LIB=debug selects the IMQ_DEBUG build (index checks after every plan); anything else the release one
LIB_PATH = os.path.join(_HERE, "libimq_debug.so" if os.environ.get("IMQ_LIB") == "debug" else "libimq.so")

# status codes
IMQ_OK, IMQ_ERR_ARG, IMQ_ERR_NONFINITE, IMQ_ERR_RANGE = 0, 1, 2, 3
IMQ_ERR_BUFFER, IMQ_ERR_TIMEOUT, IMQ_ERR_CUDA, IMQ_ERR_UNSUPPORTED, IMQ_ERR_PLAN, IMQ_ERR_BOUNDS = 4, 5, 6, 7, 8, 9
# dtypes
IMQ_F32, IMQ_BF16, IMQ_I16, IMQ_I32, IMQ_I64 = 0, 1, 2, 3, 4
# quantisation groups
IMQ_PER_TENSOR, IMQ_PER_ROW, IMQ_PER_COL = 0, 1, 2
# strategies
IMQ_MIX, IMQ_ROW_ROW, IMQ_ROW_COL, IMQ_COL_ROW, IMQ_COL_COL, IMQ_MIX_JOINT, IMQ_HYBRID = 0, 1, 2, 3, 4, 5, 6
# directions
IMQ_DIR_NONE, IMQ_DIR_OUTER, IMQ_DIR_INNER, IMQ_DIR_BOTH = 0, 1, 2, 3
IMQ_MAX_GROUPS = 64
IMQ_NOALLOC_SCRATCH_BYTES = 8 << 20
IMQ_RTN_CLIP = 1

_TORCH_TO_IMQ = {torch.float32: IMQ_F32, torch.bfloat16: IMQ_BF16, torch.int16: IMQ_I16,
                 torch.int32: IMQ_I32, torch.int64: IMQ_I64}


class ImqError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {imq_status_str(status)} (status {status})")
        self.status = status


class imq_plan_info(ctypes.Structure):
    _fields_ = [
        ("b", ctypes.c_int32), ("strategy", ctypes.c_int32),
        ("dir_a", ctypes.c_int32), ("dir_b", ctypes.c_int32),
        ("M", ctypes.c_int64), ("K", ctypes.c_int64), ("N", ctypes.c_int64),
        ("M_unp", ctypes.c_int64), ("N_unp", ctypes.c_int64), ("K_unp", ctypes.c_int64),
        ("M_eff", ctypes.c_int64), ("N_eff", ctypes.c_int64), ("K_eff", ctypes.c_int64),
        ("ratio", ctypes.c_double), ("bound", ctypes.c_double),
        ("acc_bits", ctypes.c_int32), ("n_groups", ctypes.c_int32),
        ("lmax_a_row", ctypes.c_int32), ("lmax_a_col", ctypes.c_int32),
        ("lmax_b_row", ctypes.c_int32), ("lmax_b_col", ctypes.c_int32),
        ("sum_l_a_row", ctypes.c_int64), ("sum_l_a_col", ctypes.c_int64),
        ("sum_l_b_row", ctypes.c_int64), ("sum_l_b_col", ctypes.c_int64),
        ("oor_lines_a_row", ctypes.c_int64), ("oor_lines_a_col", ctypes.c_int64),
        ("oor_lines_b_row", ctypes.c_int64), ("oor_lines_b_col", ctypes.c_int64),
        ("workspace_bytes", ctypes.c_size_t),
    ]

    def as_dict(self) -> dict:
        return {k: getattr(self, k) for k, _ in self._fields_}


class imq_group(ctypes.Structure):
    _fields_ = [("e", ctypes.c_int32), ("pad_", ctypes.c_int32), ("k_offset", ctypes.c_int64),
                ("k_len", ctypes.c_int64), ("k_len_padded", ctypes.c_int64)]


# Names and argument types of every entry point of include/imq.h.
_VP, _I32, _I64, _F64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t
SIGNATURES = {
    "imq_rtn_quantize": [_VP, _I32, _I64, _I64, _I64, _I32, _F64, _I32, _VP, _I32, _I64, _I32, _VP, _VP, _VP, _VP,
                         _VP],
    "imq_rtn_quantize_ex": [_VP, _I32, _I64, _I64, _I64, _I32, _F64, _I32, _VP, _I32, _I64, _I32, _VP, _VP, _VP,
                            _VP, ctypes.c_uint32, _VP],
    "imq_rtn_quantize_rows_noalloc": [_VP, _I32, _I64, _I64, _I64, _F64, _I32, _VP, _I32, _I64, _VP, _VP, _VP,
                                      _VP, _VP],
    "imq_plan": [_VP, _VP, _I32, _I64, _I64, _I64, _I32, _I64, _I32, _I64, _I32, _I32, _VP, _VP, _VP, _VP,
                 ctypes.POINTER(_VP), _VP],
    "imq_plan_unpack": [_VP, _VP, _I32, _I64, _I64, _I64, _I32, _I64, _I32, _I64, _I32, _I32, _VP, _VP, _VP,
                        _VP, _VP, _SZ, ctypes.POINTER(_VP), _VP],
    "imq_plan_info_get": [_VP, ctypes.POINTER(imq_plan_info)],
    "imq_plan_levels": [_VP, _VP, _VP, _VP, _VP],
    "imq_plan_groups": [_VP, ctypes.POINTER(imq_group), _I32, ctypes.POINTER(_I32)],
    "imq_plan_maps": [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP],
    "imq_plan_destroy": [_VP],
    "imq_unpack": [_VP, _VP, _VP, _VP, _VP, _VP],
    "imq_rtn_quantize_unpack": [_VP, _VP, _I32, _I64, _F64, _I32, _VP, _VP, _VP],
    "imq_gemm_unpacked": [_VP, _VP, _VP, _VP, _I32, _VP, _I32, _VP, _I32, _I64, _VP, _I64, _VP],
    "imq_unpacked_gemm": [_VP, _VP, _VP, _VP, _I32, _VP, _I32, _VP, _I32, _I64, _VP, _I64, _VP, _SZ, _VP],
    "imq_level_cover": [_VP, _I64, _I32, _I32, _VP, _VP],
    "imq_plan_batched": [_I32, _VP, _I64, _VP, _I64, _I32, _I64, _I64, _I64, _I32, _I64, _I32, _I64, _I32, _I32,
                         _VP, _VP, _VP, _VP, _VP, _VP],
    "imq_batch_workspace": [_I32, _VP, _VP, _VP],
    "imq_unpack_batched": [_I32, _VP, _VP, _I64, _VP, _I64, _VP, _SZ, _VP],
    "imq_gemm_unpacked_batched": [_I32, _VP, _VP, _SZ, _VP, _I64, _I32, _VP, _I64, _I32, _VP, _I64, _I32, _I64, _VP,
                                  _I64, _I64, _VP],
    "imq_unpacked_gemm_batched": [_I32, _VP, _VP, _I64, _VP, _I64, _VP, _I64, _I32, _VP, _I64, _I32, _VP, _I64, _I32,
                                  _I64, _VP, _I64, _I64, _VP, _SZ, _VP],
    "imq_device_status": [_VP, _I32],
    "imq_check_bounded_wait": [ctypes.c_uint64, _VP],
    "imq_status_str": [_I32],
}

_lib = None


def lib():
    """Loads libimq.so (raises when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m bit_integer_gemm_b200.build`"
                               + (" --debug" if LIB_PATH.endswith("_debug.so") else ""))
        L = ctypes.CDLL(LIB_PATH)
        for name, args in SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int32
        L.imq_status_str.restype = ctypes.c_char_p
        _lib = L
    return _lib


def imq_status_str(status: int) -> str:
    return lib().imq_status_str(int(status)).decode()


def _check(status: int, what: str):
    if status != IMQ_OK:
        raise ImqError(status, what)


def _stream(stream) -> int:
    if stream is None:
        # torch's current stream on the current device, without building a Stream object
        return torch._C._cuda_getCurrentRawStream(torch.cuda.current_device())
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _ld(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit column stride")
    return t.stride(0) if t.size(0) > 1 else t.size(1)


# ------------------------------------------------------------------------------------------------
# 1. quantisation
# ------------------------------------------------------------------------------------------------
Quantized = namedtuple("Quantized", "xint delta qval rowmax colmax")


def imq_rtn_quantize(X: torch.Tensor, gran: int, p: float, beta: int, out_dtype=torch.int16,
                     Xint=None, delta=None, qval=None, rowmax=None, colmax=None, want_qval=True,
                     want_max=True, trans_out=False, clip=False, stream=None) -> Quantized:
    """RTN quantisation of a stored 2-D matrix (fp32 or bf16) per tensor / stored row / stored column.
    trans_out writes the quantised matrix transposed (cols x rows); clip selects the clipping
    comparison variant (imq_rtn_quantize_ex with IMQ_RTN_CLIP)."""
    rows, cols = X.shape
    dev = X.device
    if Xint is None:
        Xint = torch.empty((cols, rows) if trans_out else (rows, cols), dtype=out_dtype, device=dev)
    ng = 1 if gran == IMQ_PER_TENSOR else (rows if gran == IMQ_PER_ROW else cols)
    if delta is None:
        delta = torch.empty(ng, dtype=torch.float32, device=dev)
    if qval is None and want_qval:
        qval = torch.empty(ng, dtype=torch.float32, device=dev)
    if rowmax is None and want_max:
        rowmax = torch.empty(rows, dtype=torch.int32, device=dev)
    if colmax is None and want_max:
        colmax = torch.empty(cols, dtype=torch.int32, device=dev)
    args = (_ptr(X), _TORCH_TO_IMQ[X.dtype], rows, cols, _ld(X), gran, float(p), int(beta), _ptr(Xint),
            _TORCH_TO_IMQ[Xint.dtype], _ld(Xint), int(trans_out), _ptr(delta), _ptr(qval), _ptr(rowmax),
            _ptr(colmax))
    if clip:
        st = lib().imq_rtn_quantize_ex(*args, IMQ_RTN_CLIP, _stream(stream))
        _check(st, "imq_rtn_quantize_ex")
    else:
        st = lib().imq_rtn_quantize(*args, _stream(stream))
        _check(st, "imq_rtn_quantize")
    return Quantized(Xint, delta, qval, rowmax, colmax)


def imq_rtn_quantize_rows_noalloc(X: torch.Tensor, p: float, beta: int, out_dtype=torch.int16, Xint=None,
                                  delta=None, qval=None, rowmax=None, colmax=None, want_qval=True,
                                  want_max=True, stream=None) -> Quantized:
    """Per-row RTN quantisation like imq_rtn_quantize(X, IMQ_PER_ROW, ...), with the library's scratch
    in a fixed device array instead of allocated memory (outputs not given are allocated here by torch).
    Calls whose executions overlap on one device race on that array."""
    rows, cols = X.shape
    dev = X.device
    if Xint is None:
        Xint = torch.empty((rows, cols), dtype=out_dtype, device=dev)
    if delta is None:
        delta = torch.empty(rows, dtype=torch.float32, device=dev)
    if qval is None and want_qval:
        qval = torch.empty(rows, dtype=torch.float32, device=dev)
    if rowmax is None and want_max:
        rowmax = torch.empty(rows, dtype=torch.int32, device=dev)
    if colmax is None and want_max:
        colmax = torch.empty(cols, dtype=torch.int32, device=dev)
    st = lib().imq_rtn_quantize_rows_noalloc(_ptr(X), _TORCH_TO_IMQ[X.dtype], rows, cols, _ld(X), float(p),
                                             int(beta), _ptr(Xint), _TORCH_TO_IMQ[Xint.dtype], _ld(Xint),
                                             _ptr(delta), _ptr(qval), _ptr(rowmax), _ptr(colmax), _stream(stream))
    _check(st, "imq_rtn_quantize_rows_noalloc")
    return Quantized(Xint, delta, qval, rowmax, colmax)


# ------------------------------------------------------------------------------------------------
# 2. plan
# ------------------------------------------------------------------------------------------------
class Plan:
    """Owns an imq_plan_t handle; `info` is the imq_plan_info summary as a dict."""

    def __init__(self, handle, A, B, transA=False, transB=False):
        self.handle = handle
        self._keep = (A, B)  # the plan refers to A and B
        self._transA, self._transB = bool(transA), bool(transB)
        self.raw = imq_plan_info()  # the C struct; `info` is built from it on first use
        _check(lib().imq_plan_info_get(handle, ctypes.byref(self.raw)), "imq_plan_info_get")
        self._info = None

    @property
    def info(self) -> dict:
        if self._info is None:
            self._info = self.raw.as_dict()
        return self._info

    def levels(self):
        I = self.info
        import numpy as np
        out = [np.zeros(n, np.int8) for n in (I["M"], I["K"], I["K"], I["N"])]
        _check(lib().imq_plan_levels(self.handle, *[o.ctypes.data_as(ctypes.c_void_p) for o in out]),
               "imq_plan_levels")
        return dict(zip(("a_row", "a_col", "b_row", "b_col"), out))

    def maps(self):
        """The plan's index maps of the unpacked operands (imq_plan_maps), as numpy arrays: tK, lAk, lBk
        (K_unp), srcA, lvlA (M_unp), srcB, lvlB (N_unp)."""
        import numpy as np
        I = self.info
        out = {"tK": np.zeros(I["K_unp"], np.int32), "lAk": np.zeros(I["K_unp"], np.int8),
               "lBk": np.zeros(I["K_unp"], np.int8), "srcA": np.zeros(I["M_unp"], np.int32),
               "lvlA": np.zeros(I["M_unp"], np.int8), "srcB": np.zeros(I["N_unp"], np.int32),
               "lvlB": np.zeros(I["N_unp"], np.int8)}
        _check(lib().imq_plan_maps(self.handle, *[out[k].ctypes.data_as(ctypes.c_void_p) for k in
                                                  ("tK", "lAk", "lBk", "srcA", "lvlA", "srcB", "lvlB")]),
               "imq_plan_maps")
        return out

    def groups(self):
        arr = (imq_group * IMQ_MAX_GROUPS)()
        n = ctypes.c_int32(0)
        _check(lib().imq_plan_groups(self.handle, arr, IMQ_MAX_GROUPS, ctypes.byref(n)), "imq_plan_groups")
        return [(arr[i].e, arr[i].k_offset, arr[i].k_len, arr[i].k_len_padded) for i in range(n.value)]

    def destroy(self):
        if self.handle is not None:
            lib().imq_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def imq_plan(A: torch.Tensor, B: torch.Tensor, b: int, strategy: int = IMQ_MIX, transA: bool = False,
             transB: bool = False, maxes=None, stream=None) -> Plan:
    """A: stored M x K (K x M when transA); B: stored K x N (N x K when transB); int16 or int32.
    maxes: optional (a_rowmax, a_colmax, b_rowmax, b_colmax) int32 tensors over LOGICAL lines."""
    M = A.shape[1] if transA else A.shape[0]
    K = A.shape[0] if transA else A.shape[1]
    N = B.shape[0] if transB else B.shape[1]
    if A.dtype != B.dtype:
        raise ValueError("A and B must have the same integer dtype")
    mx = [None] * 4 if maxes is None else list(maxes)
    h = ctypes.c_void_p()
    st = lib().imq_plan(_ptr(A), _ptr(B), _TORCH_TO_IMQ[A.dtype], M, K, N, int(transA), _ld(A), int(transB),
                        _ld(B), int(b), int(strategy), *[_ptr(m) for m in mx], ctypes.byref(h), _stream(stream))
    _check(st, "imq_plan")
    return Plan(h, A, B)


_VIEWS = {}  # (workspace address, bytes, M_unp, N_unp, K_unp) -> (workspace, A' view, B'^T view)


def workspace_views(plan: Plan, workspace: torch.Tensor):
    """A' and B'^T views of a workspace in the layout of imq_plan_unpack and imq_unpacked_gemm (kept per
    workspace and plan shape, so that a loop over equal-shaped plans builds them once)."""
    r = plan.raw
    key = (workspace.data_ptr(), workspace.numel() * workspace.element_size(), r.M_unp, r.N_unp, r.K_unp)
    hit = _VIEWS.get(key)
    if hit is not None and hit[0] is workspace:
        return hit[1], hit[2]
    off = (-workspace.data_ptr()) % 1024
    w8 = workspace.view(torch.int8) if workspace.dtype != torch.int8 else workspace
    na = r.M_unp * r.K_unp
    b_off = off + (na + 1023) // 1024 * 1024
    views = (w8[off:off + na].view(r.M_unp, r.K_unp), w8[b_off:b_off + r.N_unp * r.K_unp].view(r.N_unp, r.K_unp))
    if len(_VIEWS) >= 4:  # the views keep their workspace alive: hold only a few
        _VIEWS.clear()
    _VIEWS[key] = (workspace,) + views
    return views


def imq_plan_unpack(A: torch.Tensor, B: torch.Tensor, b: int, strategy: int = IMQ_MIX, transA: bool = False,
                    transB: bool = False, maxes=None, workspace=None, stream=None):
    """imq_plan followed, in the same host call, by imq_unpack into `workspace` (a 1-D uint8/int8 device
    tensor).  Returns (plan, A_unp, B_unp_t) with the operands as views of the workspace, or (plan, None,
    None) when the workspace is smaller than the plan needs (nothing unpacked; workspace_for(plan) gives
    one that fits)."""
    M = A.shape[1] if transA else A.shape[0]
    K = A.shape[0] if transA else A.shape[1]
    N = B.shape[0] if transB else B.shape[1]
    if A.dtype != B.dtype:
        raise ValueError("A and B must have the same integer dtype")
    mx = [None] * 4 if maxes is None else list(maxes)
    wp, wn = (None, 0) if workspace is None else _aligned(workspace)
    h = ctypes.c_void_p()
    st = lib().imq_plan_unpack(_ptr(A), _ptr(B), _TORCH_TO_IMQ[A.dtype], M, K, N, int(transA), _ld(A), int(transB),
                               _ld(B), int(b), int(strategy), *[_ptr(m) for m in mx], wp, wn, ctypes.byref(h),
                               _stream(stream))
    if st == IMQ_ERR_BUFFER and h.value:
        return Plan(h, A, B), None, None
    _check(st, "imq_plan_unpack")
    plan = Plan(h, A, B)
    if workspace is None:
        return plan, None, None
    Au, Bu = workspace_views(plan, workspace)
    return plan, Au, Bu


# ------------------------------------------------------------------------------------------------
# 3. unpack and GEMM
# ------------------------------------------------------------------------------------------------
def imq_unpack(plan: Plan, A: torch.Tensor, B: torch.Tensor, A_unp=None, B_unp_t=None, stream=None):
    I = plan.info
    dev = A.device
    if A_unp is None:
        A_unp = torch.empty((I["M_unp"], I["K_unp"]), dtype=torch.int8, device=dev)
    if B_unp_t is None:
        B_unp_t = torch.empty((I["N_unp"], I["K_unp"]), dtype=torch.int8, device=dev)
    _check(lib().imq_unpack(plan.handle, _ptr(A), _ptr(B), _ptr(A_unp), _ptr(B_unp_t), _stream(stream)),
           "imq_unpack")
    return A_unp, B_unp_t


def imq_rtn_quantize_unpack(plan: Plan, X: torch.Tensor, p: float, beta: int, A_unp=None, deltaA=None,
                            stream=None):
    """Per-row RTN of X (M x K, float32 or bfloat16, row-major) fused with its unpacking into the plan's
    A' layout.  Returns (A_unp, deltaA).  IMQ_ERR_PLAN in the device status word when an entry exceeds
    the plan's column maxima (see include/imq.h)."""
    I = plan.info
    if X.dim() != 2 or X.stride(1) != 1 or tuple(X.shape) != (I["M"], I["K"]):
        raise ValueError("X must be a row-major M x K matrix of the plan's shape")
    if A_unp is None:
        A_unp = torch.empty((I["M_unp"], I["K_unp"]), dtype=torch.int8, device=X.device)
    if deltaA is None:
        deltaA = torch.empty(I["M"], dtype=torch.float32, device=X.device)
    _check(lib().imq_rtn_quantize_unpack(plan.handle, _ptr(X), _TORCH_TO_IMQ[X.dtype], _ld(X), float(p), int(beta),
                                         _ptr(A_unp), _ptr(deltaA), _stream(stream)), "imq_rtn_quantize_unpack")
    return A_unp, deltaA


def imq_level_cover(maxima: torch.Tensor, b: int, cap: int = 32767, out=None, stream=None) -> torch.Tensor:
    """min(R^L - 1, cap) for every line maximum (L its number of base-R digits), int32 on the device."""
    if out is None:
        out = torch.empty_like(maxima)
    _check(lib().imq_level_cover(_ptr(maxima), maxima.numel(), int(b), int(cap), _ptr(out), _stream(stream)),
           "imq_level_cover")
    return out


def imq_check_bounded_wait(timeout_ns: int, stream=None):
    """Diagnostic: a kernel whose bounded wait runs out after timeout_ns and records IMQ_ERR_TIMEOUT."""
    _check(lib().imq_check_bounded_wait(int(timeout_ns), _stream(stream)), "imq_check_bounded_wait")


def _outputs(I, dev, C, c_dtype, Cf, want_int, want_f32):
    if C is None and want_int:
        if c_dtype is None:
            c_dtype = torch.int32 if I["acc_bits"] == 32 else torch.int64
        C = torch.empty((I["M"], I["N"]), dtype=c_dtype, device=dev)
    if Cf is None and want_f32:
        Cf = torch.empty((I["M"], I["N"]), dtype=torch.float32, device=dev)
    return C, Cf


def imq_gemm_unpacked(plan: Plan, A_unp, B_unp_t, deltaA=None, gA=IMQ_PER_TENSOR, deltaB=None,
                      gB=IMQ_PER_TENSOR, C=None, c_dtype=None, Cf=None, want_int=True, want_f32=True,
                      stream=None):
    want_f32 = want_f32 and deltaA is not None
    if (C is None and want_int) or (Cf is None and want_f32):
        C, Cf = _outputs(plan.info, A_unp.device, C, c_dtype, Cf, want_int, want_f32)
    n = plan.raw.N
    st = lib().imq_gemm_unpacked(plan.handle, _ptr(A_unp), _ptr(B_unp_t), _ptr(deltaA), gA, _ptr(deltaB), gB,
                                 _ptr(C), _TORCH_TO_IMQ[C.dtype] if C is not None else IMQ_I32,
                                 _ld(C) if C is not None else n, _ptr(Cf),
                                 _ld(Cf) if Cf is not None else n, _stream(stream))
    _check(st, "imq_gemm_unpacked")
    return C, Cf


def workspace_for(plan: Plan, device=None) -> torch.Tensor:
    n = max(int(plan.info["workspace_bytes"]), 1) + 1024
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def _aligned(ws: torch.Tensor):
    off = (-ws.data_ptr()) % 1024
    nbytes = ws.numel() * ws.element_size()
    return ctypes.c_void_p(ws.data_ptr() + off), max(0, nbytes - off)


def imq_unpacked_gemm(plan: Plan, A, B, deltaA=None, gA=IMQ_PER_TENSOR, deltaB=None, gB=IMQ_PER_TENSOR,
                      C=None, c_dtype=None, Cf=None, workspace=None, want_int=True, want_f32=True,
                      stream=None):
    I = plan.info
    if workspace is None:
        workspace = workspace_for(plan, A.device)
    wp, wn = _aligned(workspace)
    C, Cf = _outputs(I, A.device, C, c_dtype, Cf, want_int, want_f32 and deltaA is not None)
    st = lib().imq_unpacked_gemm(plan.handle, _ptr(A), _ptr(B), _ptr(deltaA), gA, _ptr(deltaB), gB, _ptr(C),
                                 _TORCH_TO_IMQ[C.dtype] if C is not None else IMQ_I32,
                                 _ld(C) if C is not None else I["N"], _ptr(Cf),
                                 _ld(Cf) if Cf is not None else I["N"], wp, wn, _stream(stream))
    _check(st, "imq_unpacked_gemm")
    return C, Cf


def imq_device_status(clear: bool = False, stream=None) -> int:
    return int(lib().imq_device_status(_stream(stream), int(clear)))


# ------------------------------------------------------------------------------------------------
# 4. batches of equal-shaped GEMMs
# ------------------------------------------------------------------------------------------------
class PlanBatch:
    """The plans of one imq_plan_batched call (a list of Plan, problem h first at index h) and the
    handle array the batched calls take."""

    def __init__(self, plans, A, B):
        self.plans = plans
        self._keep = (A, B)
        self.handles = (ctypes.c_void_p * len(plans))(*[p.handle for p in plans])

    def __len__(self):
        return len(self.plans)

    def __getitem__(self, h):
        return self.plans[h]

    def workspace_layout(self):
        """(offsets [(A' offset, B'^T offset)] per problem, total bytes) of imq_batch_workspace."""
        n = len(self.plans)
        off = (ctypes.c_size_t * (2 * n))()
        tot = ctypes.c_size_t(0)
        _check(lib().imq_batch_workspace(n, self.handles, off, ctypes.byref(tot)), "imq_batch_workspace")
        return [(off[2 * h], off[2 * h + 1]) for h in range(n)], tot.value

    def destroy(self):
        for p in self.plans:
            p.destroy()


def imq_plan_batched(A: torch.Tensor, B: torch.Tensor, batch: int, M: int, K: int, N: int, b: int,
                     strategy: int = IMQ_MIX, transA: bool = False, transB: bool = False, strideA=None,
                     strideB=None, lda=None, ldb=None, maxes=None, stream=None) -> PlanBatch:
    """Plans `batch` problems of one shape: problem h's A starts strideA elements after problem h-1's
    (default: its stored rows times lda), likewise B; lda / ldb default to the tensors' row strides."""
    if A.dtype != B.dtype:
        raise ValueError("A and B must have the same integer dtype")
    lda = _ld(A) if lda is None else lda
    ldb = _ld(B) if ldb is None else ldb
    strideA = (K if transA else M) * lda if strideA is None else strideA
    strideB = (N if transB else K) * ldb if strideB is None else strideB
    mx = [None] * 4 if maxes is None else list(maxes)
    hs = (ctypes.c_void_p * batch)()
    st = lib().imq_plan_batched(batch, _ptr(A), strideA, _ptr(B), strideB, _TORCH_TO_IMQ[A.dtype], M, K, N,
                                int(transA), lda, int(transB), ldb, int(b), int(strategy), *[_ptr(m) for m in mx], hs,
                                _stream(stream))
    _check(st, "imq_plan_batched")
    return PlanBatch([Plan(hs[h], A, B, transA, transB) for h in range(batch)], A, B)


def batch_workspace(batch: PlanBatch, device=None) -> torch.Tensor:
    _, tot = batch.workspace_layout()
    return torch.empty(max(tot, 1) + 1024, dtype=torch.uint8, device=device or "cuda")


def batch_views(batch: PlanBatch, workspace: torch.Tensor):
    """[(A' view, B'^T view)] per problem in the batch workspace layout."""
    offs, _ = batch.workspace_layout()
    base = (-workspace.data_ptr()) % 1024
    w8 = workspace.view(torch.int8) if workspace.dtype != torch.int8 else workspace
    out = []
    for (oa, ob), p in zip(offs, batch.plans):
        r = p.raw
        out.append((w8[base + oa:base + oa + r.M_unp * r.K_unp].view(r.M_unp, r.K_unp),
                    w8[base + ob:base + ob + r.N_unp * r.K_unp].view(r.N_unp, r.K_unp)))
    return out


def imq_unpack_batched(batch: PlanBatch, A: torch.Tensor, B: torch.Tensor, workspace: torch.Tensor, strideA=None,
                       strideB=None, stream=None):
    r = batch.plans[0].raw
    strideA = (r.K if batch.plans[0]._transA else r.M) * _ld(A) if strideA is None else strideA
    strideB = (r.N if batch.plans[0]._transB else r.K) * _ld(B) if strideB is None else strideB
    wp, wn = _aligned(workspace)
    _check(lib().imq_unpack_batched(len(batch), batch.handles, _ptr(A), strideA, _ptr(B), strideB, wp, wn,
                                    _stream(stream)), "imq_unpack_batched")


def imq_gemm_unpacked_batched(batch: PlanBatch, workspace: torch.Tensor, deltaA, strideDA: int, gA: int, deltaB,
                              strideDB: int, gB: int, C: torch.Tensor, Cf: torch.Tensor, strideC=None, strideCf=None,
                              stream=None):
    """C, Cf: (batch, M, N)-shaped (or any tensors with the given batch strides and unit column stride)."""
    r = batch.plans[0].raw
    ldc = C.stride(-2) if C is not None else r.N
    ldcf = Cf.stride(-2) if Cf is not None else r.N
    strideC = (C.stride(0) if C is not None else 0) if strideC is None else strideC
    strideCf = (Cf.stride(0) if Cf is not None else 0) if strideCf is None else strideCf
    wp, wn = _aligned(workspace)
    st = lib().imq_gemm_unpacked_batched(len(batch), batch.handles, wp, wn, _ptr(deltaA), strideDA, gA, _ptr(deltaB),
                                         strideDB, gB, _ptr(C), strideC,
                                         _TORCH_TO_IMQ[C.dtype] if C is not None else IMQ_I32, ldc, _ptr(Cf), strideCf,
                                         ldcf, _stream(stream))
    _check(st, "imq_gemm_unpacked_batched")
