"""Helpers shared by the GPU parity tests: moving seeded workloads to the device and running the
library path and the oracle on the same bytes."""
import numpy as np
import torch

import oracle
import workloads


def to_device(st: workloads.Stored) -> torch.Tensor:
    if st.dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(st.data).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(st.data, dtype=np.float32)).cuda()


def oracle_quantize(st: workloads.Stored, gran: int, p: float, beta: int):
    return oracle.rtn_quantize(oracle.as_f32(st.data, st.dtype), gran, p, beta)


def logical(x: np.ndarray, trans: bool) -> np.ndarray:
    return np.ascontiguousarray(x.T) if trans else x


def logical_maxes(imq, qa, qb, transA, transB):
    """(a_rowmax, a_colmax, b_rowmax, b_colmax) over LOGICAL lines from the quantiser side outputs."""
    a_row, a_col = (qa.colmax, qa.rowmax) if transA else (qa.rowmax, qa.colmax)
    b_row, b_col = (qb.colmax, qb.rowmax) if transB else (qb.rowmax, qb.colmax)
    return a_row, a_col, b_row, b_col


def assert_f32_close(got: np.ndarray, want: np.ndarray, rel: float = 1e-6):
    """|got - want| <= rel * |want| elementwise; zeros must match exactly."""
    got = got.astype(np.float64)
    want = want.astype(np.float64)
    zero = want == 0
    assert np.all(got[zero] == 0), "dequantised zero mismatch"
    err = np.abs(got - want)
    bad = err > rel * np.abs(want)
    if bad.any():
        k = np.argmax(err / np.maximum(np.abs(want), 1e-300))
        raise AssertionError(f"{int(bad.sum())} fp32 outputs off by more than {rel} relative; worst at "
                             f"{np.unravel_index(k, want.shape)}: got {got.ravel()[k]} want {want.ravel()[k]}")


def plan_matches(info: dict, pl: oracle.Plan):
    fields = {"dir_a": pl.dir_a, "dir_b": pl.dir_b, "M_unp": pl.M_unp, "N_unp": pl.N_unp, "K_unp": pl.K_unp,
              "M_eff": pl.M_eff, "N_eff": pl.N_eff, "K_eff": pl.K_eff, "n_groups": len(pl.groups),
              "acc_bits": pl.acc_bits,
              "lmax_a_row": pl.lmax[0], "lmax_a_col": pl.lmax[1], "lmax_b_row": pl.lmax[2], "lmax_b_col": pl.lmax[3],
              "sum_l_a_row": pl.suml[0], "sum_l_a_col": pl.suml[1], "sum_l_b_row": pl.suml[2],
              "sum_l_b_col": pl.suml[3],
              "oor_lines_a_row": pl.oor_lines[0], "oor_lines_a_col": pl.oor_lines[1],
              "oor_lines_b_row": pl.oor_lines[2], "oor_lines_b_col": pl.oor_lines[3]}
    for k, v in fields.items():
        assert info[k] == v, f"plan field {k}: library {info[k]} oracle {v}"
    assert info["ratio"] == pl.ratio or abs(info["ratio"] - pl.ratio) <= 1e-12 * pl.ratio
    assert info["bound"] == pl.bound


def unsupported(pl: oracle.Plan) -> bool:
    """True when the library must refuse the plan: the bound reaches 2^63 (C may leave int64)."""
    return int(round(pl.bound)) >= 2 ** 63
