"""CPU oracle for the IM-Unpack exact low-bit integer GEMM.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its
``cpu_baseline`` leg and its ``--impl reference`` arm) may import this package.  The product library
under ``bit_integer_gemm_b200/`` never imports it, and it imports nothing from there.

The arithmetic lives in plain C (``oracle/*.c``, built with gcc, no fast-math, no FMA contraction);
this module only marshals numpy arrays.  The one numpy arithmetic step is :func:`gemm_exact`, a float64
BLAS product used only when every partial sum is an integer below 2**53 (so every floating-point
operation in it is exact, in any order); the int64 triple loop :func:`gemm_i64` is the definition.

Source of the method: "IM-Unpack: Training and Inference with Arbitrarily Low Precision Integers"
(atlas.scime.ai summary page): "Approach", "Problem", "Key results", the measured-effects table and
"Experimental setup".  Each C file cites the section it follows.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_SRCS = ["percentile.c", "rtn.c", "digits.c", "plan.c", "unpack.c", "gemm.c", "dequant.c"]

PER_TENSOR, PER_ROW, PER_COL = 0, 1, 2
MIX, ROW_ROW, ROW_COL, COL_ROW, COL_COL, MIX_JOINT, HYBRID = 0, 1, 2, 3, 4, 5, 6
DIR_NONE, DIR_OUTER, DIR_INNER, DIR_BOTH = 0, 1, 2, 3
OK, ERR_ARG, ERR_NONFINITE, ERR_RANGE = 0, 1, 2, 3
MAX_GROUPS = 64


class OracleError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"oracle {what} failed with status {status}")
        self.status = status


def build(force: bool = False) -> str:
    """Compiles oracle/*.c into oracle/liboracle.so when missing or older than a source."""
    srcs = [os.path.join(_HERE, s) for s in _SRCS] + [os.path.join(_HERE, "oracle.h")]
    if not force and os.path.exists(_SO):
        so_t = os.path.getmtime(_SO)
        if all(os.path.getmtime(s) <= so_t for s in srcs):
            return _SO
    tmp = _SO + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=gnu11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-o", tmp] + [os.path.join(_HERE, s) for s in _SRCS] + ["-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _SO)
    return _SO


_lib_handle = None


class _Plan(ctypes.Structure):
    _fields_ = [
        ("b", ctypes.c_int32), ("strategy", ctypes.c_int32),
        ("dir_a", ctypes.c_int32), ("dir_b", ctypes.c_int32),
        ("M", ctypes.c_int64), ("K", ctypes.c_int64), ("N", ctypes.c_int64),
        ("M_eff", ctypes.c_int64), ("N_eff", ctypes.c_int64), ("K_eff", ctypes.c_int64),
        ("ratio", ctypes.c_double), ("bound", ctypes.c_double),
        ("bound_lt_2_31", ctypes.c_int32), ("n_groups", ctypes.c_int32),
        ("lmax", ctypes.c_int32 * 4), ("suml", ctypes.c_int64 * 4), ("oor_lines", ctypes.c_int64 * 4),
        ("group_e", ctypes.c_int32 * MAX_GROUPS), ("group_len", ctypes.c_int64 * MAX_GROUPS),
    ]


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _lib():
    global _lib_handle
    if _lib_handle is None:
        lib = ctypes.CDLL(build())
        vp, i64, i32, f64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.oracle_percentile_abs.argtypes = [vp, i64, f64]
        lib.oracle_percentile_abs.restype = ctypes.c_float
        lib.oracle_rtn_quantize.argtypes = [vp, i64, i64, i32, f64, i32, vp, vp, vp]
        lib.oracle_rtn_quantize_ex.argtypes = [vp, i64, i64, i32, f64, i32, i32, vp, vp, vp]
        lib.oracle_level.argtypes = [i64, i32]
        lib.oracle_level.restype = i32
        lib.oracle_digit.argtypes = [i64, i32, i32]
        lib.oracle_digit.restype = i64
        lib.oracle_digits_array.argtypes = [vp, i64, i32, i32, vp, vp]
        lib.oracle_digits_array.restype = None
        lib.oracle_plan.argtypes = [vp, vp, i64, i64, i64, i32, i32, vp, vp, vp, vp,
                                    ctypes.POINTER(_Plan)]
        lib.oracle_unpack_lines.argtypes = [ctypes.POINTER(_Plan)] + [vp] * 7
        lib.oracle_unpack.argtypes = [ctypes.POINTER(_Plan)] + [vp] * 9
        lib.oracle_gemm_i64.argtypes = [vp, vp, i64, i64, i64, vp, i32]
        lib.oracle_gemm_i64.restype = None
        lib.oracle_unpacked_gemm.argtypes = [ctypes.POINTER(_Plan)] + [vp] * 7
        lib.oracle_dequant.argtypes = [vp, i64, i64, vp, i32, vp, i32, vp]
        lib.oracle_dequant.restype = None
        _lib_handle = lib
    return _lib_handle


# ----------------------------------------------------------------------------------------------
# inputs
# ----------------------------------------------------------------------------------------------
def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns (uint16) to float32: the bf16 bits are the top half."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def as_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    """x is float32 data (dtype 'f32') or bfloat16 bit patterns held in uint16 (dtype 'bf16')."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x)
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------------------------
# steps 1-2: percentile and RTN
# ----------------------------------------------------------------------------------------------
def percentile_abs(v: np.ndarray, p: float) -> np.float32:
    v = np.ascontiguousarray(v, dtype=np.float32).ravel()
    return np.float32(_lib().oracle_percentile_abs(_ptr(v), v.size, float(p)))


def rtn_quantize(x: np.ndarray, gran: int, p: float, beta: int, clip: bool = False):
    """x: 2-D float32.  Returns (xint int64, delta float32, qval float32); raises OracleError.  clip:
    the clipping comparison variant (scaled values clamped to [-beta, beta] before rounding)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, cols = x.shape
    ng = 1 if gran == PER_TENSOR else (rows if gran == PER_ROW else cols)
    xint = np.zeros((rows, cols), dtype=np.int64)
    delta = np.zeros(ng, dtype=np.float32)
    qval = np.zeros(ng, dtype=np.float32)
    st = _lib().oracle_rtn_quantize_ex(_ptr(x), rows, cols, gran, float(p), int(beta), int(bool(clip)),
                                       _ptr(xint), _ptr(delta), _ptr(qval))
    if st != OK:
        raise OracleError(st, "rtn_quantize")
    return xint, delta, qval


# ----------------------------------------------------------------------------------------------
# steps 3-5: levels, plan, layout, unpack
# ----------------------------------------------------------------------------------------------
def level(v: int, b: int) -> int:
    return int(_lib().oracle_level(int(v), int(b)))


def digit(v: int, l: int, b: int) -> int:
    return int(_lib().oracle_digit(int(v), int(l), int(b)))


def digits_array(v: np.ndarray, b: int, nl: int):
    """Returns (digits int64 [n, nl], levels int32 [n]) for an int64 vector v."""
    v = np.ascontiguousarray(v, dtype=np.int64).ravel()
    out = np.zeros((v.size, nl), np.int64)
    lev = np.zeros(v.size, np.int32)
    _lib().oracle_digits_array(_ptr(v), v.size, int(b), int(nl), _ptr(out), _ptr(lev))
    return out, lev


@dataclass
class Plan:
    """The oracle's plan: directions, level statistics, unpacked sizes and the unpacked lines and inner
    triples, with no memory layout (see oracle/plan.c)."""
    b: int
    strategy: int
    dir_a: int
    dir_b: int
    M: int
    K: int
    N: int
    M_eff: int
    N_eff: int
    K_eff: int
    ratio: float
    bound: float
    bound_lt_2_31: bool
    groups: list  # [(e, number of inner triples with lA + lB = e)], e ascending
    lmax: tuple
    suml: tuple
    oor_lines: tuple
    # a_row, a_col, b_row, b_col (int32): line levels; under HYBRID the levels each line carries in the
    # unpacked GEMM (1 for a row of A or column of B that is not unpacked OUTER, the inner levels taken
    # over the lines that are not)
    levels: dict = field(default_factory=dict)
    # a_lines (M_eff x 2: row i, level l), b_lines (N_eff x 2: column j, level m), pairs (K_eff x 3:
    # t, lA, lB), each in lexicographic order (int32)
    lines: dict = field(default_factory=dict)
    _raw: object = None

    @property
    def acc_bits(self) -> int:
        return 32 if self.bound_lt_2_31 else 64


def plan(A: np.ndarray, B: np.ndarray, b: int, strategy: int) -> Plan:
    """A: M x K int64 (logical), B: K x N int64 (logical)."""
    A = np.ascontiguousarray(A, dtype=np.int64)
    B = np.ascontiguousarray(B, dtype=np.int64)
    M, K = A.shape
    K2, N = B.shape
    assert K == K2
    lv = {"a_row": np.zeros(M, np.int32), "a_col": np.zeros(K, np.int32),
          "b_row": np.zeros(K, np.int32), "b_col": np.zeros(N, np.int32)}
    raw = _Plan()
    lib = _lib()
    st = lib.oracle_plan(_ptr(A), _ptr(B), M, K, N, int(b), int(strategy), _ptr(lv["a_row"]),
                         _ptr(lv["a_col"]), _ptr(lv["b_row"]), _ptr(lv["b_col"]), ctypes.byref(raw))
    if st != OK:
        raise OracleError(st, "plan")
    ln = {"a_lines": np.zeros((raw.M_eff, 2), np.int32), "b_lines": np.zeros((raw.N_eff, 2), np.int32),
          "pairs": np.zeros((raw.K_eff, 3), np.int32)}
    st = lib.oracle_unpack_lines(ctypes.byref(raw), _ptr(lv["a_row"]), _ptr(lv["a_col"]), _ptr(lv["b_row"]),
                                 _ptr(lv["b_col"]), _ptr(ln["a_lines"]), _ptr(ln["b_lines"]), _ptr(ln["pairs"]))
    if st != OK:
        raise OracleError(st, "unpack_lines")
    groups = [(raw.group_e[g], raw.group_len[g]) for g in range(raw.n_groups)]
    return Plan(b=raw.b, strategy=raw.strategy, dir_a=raw.dir_a, dir_b=raw.dir_b, M=raw.M, K=raw.K,
                N=raw.N, M_eff=raw.M_eff, N_eff=raw.N_eff, K_eff=raw.K_eff, ratio=raw.ratio, bound=raw.bound,
                bound_lt_2_31=bool(raw.bound_lt_2_31), groups=groups, lmax=tuple(raw.lmax),
                suml=tuple(raw.suml), oor_lines=tuple(raw.oor_lines), levels=lv, lines=ln, _raw=raw)


def unpack(pl: Plan, A: np.ndarray, B: np.ndarray):
    """Returns (A' int8 M_eff x K_eff, B'^T int8 N_eff x K_eff): entry (u, p) of A' is the digit of A for
    unpacked line pl.lines['a_lines'][u] and inner triple pl.lines['pairs'][p]; likewise B'^T."""
    A = np.ascontiguousarray(A, dtype=np.int64)
    B = np.ascontiguousarray(B, dtype=np.int64)
    Aq = np.zeros((pl.M_eff, pl.K_eff), np.int8)
    Bq = np.zeros((pl.N_eff, pl.K_eff), np.int8)
    ln = pl.lines
    st = _lib().oracle_unpack(ctypes.byref(pl._raw), _ptr(pl.levels["a_row"]), _ptr(pl.levels["b_col"]),
                              _ptr(ln["a_lines"]), _ptr(ln["b_lines"]), _ptr(ln["pairs"]), _ptr(A), _ptr(B),
                              _ptr(Aq), _ptr(Bq))
    if st != OK:
        raise OracleError(st, "unpack")
    return Aq, Bq


def unpacked_gemm(pl: Plan, Aq: np.ndarray, Bq: np.ndarray, return_macs: bool = False):
    """The integer product rebuilt from the unpacked operands (each inner triple weighted by R^(lA+lB),
    each pair of lines by R^(l+m)); with return_macs also the multiply-adds the loop executed."""
    Aq = np.ascontiguousarray(Aq, dtype=np.int8)
    Bq = np.ascontiguousarray(Bq, dtype=np.int8)
    C = np.zeros((pl.M, pl.N), np.int64)
    macs = ctypes.c_int64(0)
    ln = pl.lines
    st = _lib().oracle_unpacked_gemm(ctypes.byref(pl._raw), _ptr(ln["a_lines"]), _ptr(ln["b_lines"]),
                                     _ptr(ln["pairs"]), _ptr(Aq), _ptr(Bq), _ptr(C), ctypes.byref(macs))
    if st != OK:
        raise OracleError(st, "unpacked_gemm")
    return (C, int(macs.value)) if return_macs else C


# ----------------------------------------------------------------------------------------------
# steps 6-8: the integer product and its dequantisation
# ----------------------------------------------------------------------------------------------
def gemm_i64(A: np.ndarray, B: np.ndarray, nthreads: int = 0) -> np.ndarray:
    """Definition: C = A * B by an int64 triple loop (OpenMP over rows)."""
    A = np.ascontiguousarray(A, dtype=np.int64)
    B = np.ascontiguousarray(B, dtype=np.int64)
    M, K = A.shape
    N = B.shape[1]
    C = np.zeros((M, N), np.int64)
    _lib().oracle_gemm_i64(_ptr(A), _ptr(B), M, K, N, _ptr(C), int(nthreads))
    return C


def product_bound(A: np.ndarray, B: np.ndarray) -> int:
    """sum_t max_i |A[i,t]| * max_j |B[t,j]| as a Python integer."""
    ca = np.abs(A).max(axis=0).astype(object) if A.shape[0] else np.zeros(A.shape[1], object)
    rb = np.abs(B).max(axis=1).astype(object) if B.shape[1] else np.zeros(B.shape[0], object)
    return int(sum(int(a) * int(b) for a, b in zip(ca, rb)))


def gemm_exact(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """C = A * B exactly.  When the bound is below 2**53 every product and every partial sum of the
    float64 BLAS product is an integer of magnitude below 2**53, so each floating-point operation is
    exact whatever order or fusion BLAS uses; otherwise the int64 triple loop runs."""
    A = np.asarray(A)
    B = np.asarray(B)
    if product_bound(A, B) < 2 ** 53:
        C = np.matmul(A.astype(np.float64), B.astype(np.float64))
        return C.astype(np.int64)
    return gemm_i64(A, B)


def dequant(C: np.ndarray, dA: np.ndarray, gA: int, dB: np.ndarray, gB: int) -> np.ndarray:
    """Cf = C * (DeltaA[i] * DeltaB[j]) in float64 from the fp32 steps."""
    C = np.ascontiguousarray(C, dtype=np.int64)
    M, N = C.shape
    dA = np.ascontiguousarray(dA, dtype=np.float32)
    dB = np.ascontiguousarray(dB, dtype=np.float32)
    Cf = np.zeros((M, N), np.float64)
    _lib().oracle_dequant(_ptr(C), M, N, _ptr(dA), int(gA), _ptr(dB), int(gB), _ptr(Cf))
    return Cf


def nearest_rank(n: int, p: float) -> int:
    """k = clamp(ceil(p*n), 1, n) in double, the rank the percentile step selects."""
    return min(max(math.ceil(p * n), 1), n)
