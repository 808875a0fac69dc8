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


def plan_matches(info: dict, pl: oracle.Plan, groups=None):
    """The library's plan summary against the oracle's: directions, unpacked sizes (unpadded), level
    statistics, accumulator width, ratio and bound; with `groups` (the library's imq_plan_groups list)
    also the exponent of every inner group and its number of real triples."""
    fields = {"dir_a": pl.dir_a, "dir_b": pl.dir_b,
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
    if groups is not None:
        assert [(e, n) for e, _, n, _ in groups] == list(pl.groups)


def _keys_lines(src, lvl):
    return src.astype(np.int64) * 64 + lvl.astype(np.int64)


def _match(lib_keys, want_keys, what):
    """Indices into lib_keys, in the order of want_keys, of a bijection between the used library entries
    (keys >= 0) and the oracle's (keys strictly increasing); the unused library entries are returned too."""
    used = np.flatnonzero(lib_keys >= 0)
    order = np.argsort(lib_keys[used], kind="stable")
    got = lib_keys[used][order]
    assert got.size == want_keys.size, f"{what}: library has {got.size} used entries, oracle {want_keys.size}"
    assert np.array_equal(got, want_keys), f"{what}: the library's entries are not the oracle's"
    return used[order], np.flatnonzero(lib_keys < 0)


def check_unpacked(plan, pl: oracle.Plan, Au: np.ndarray, Bu: np.ndarray, A: np.ndarray, B: np.ndarray):
    """The library's unpacked operands against the oracle's, entry by entry, through the library's own
    index maps (imq_plan_maps): the used rows of A' are exactly the oracle's unpacked lines (i, l) of A,
    each once, the used inner positions exactly its triples (t, lA, lB), likewise for B'^T; every byte at
    a used row and position equals the oracle's digit there; unused rows and padding are zero."""
    mp = plan.maps()
    ln = pl.lines
    tK = mp["tK"].astype(np.int64)
    pkey = np.where(tK >= 0, tK * 4096 + mp["lAk"].astype(np.int64) * 64 + mp["lBk"].astype(np.int64), -1)
    pw = ln["pairs"].astype(np.int64)
    pos, pad = _match(pkey, pw[:, 0] * 4096 + pw[:, 1] * 64 + pw[:, 2], "inner triples")
    srcA = mp["srcA"].astype(np.int64)
    akey = np.where(srcA >= 0, _keys_lines(srcA, mp["lvlA"]), -1)
    al = ln["a_lines"].astype(np.int64)
    rows_a, unused_a = _match(akey, al[:, 0] * 64 + al[:, 1], "lines of A")
    srcB = mp["srcB"].astype(np.int64)
    bkey = np.where(srcB >= 0, _keys_lines(srcB, mp["lvlB"]), -1)
    bl = ln["b_lines"].astype(np.int64)
    rows_b, unused_b = _match(bkey, bl[:, 0] * 64 + bl[:, 1], "lines of B")
    oAq, oBq = oracle.unpack(pl, A, B)
    assert np.array_equal(Au[np.ix_(rows_a, pos)], oAq), "A' bytes"
    del oAq
    assert np.array_equal(Bu[np.ix_(rows_b, pos)], oBq), "B'^T bytes"
    del oBq
    assert not Au[unused_a].any() and not Bu[unused_b].any(), "unused unpacked lines are not zero"
    assert not Au[:, pad].any() and not Bu[:, pad].any(), "inner padding is not zero"
    return mp


def check_layout(plan, mp=None):
    """The library's documented layout (imq_unpack), from its own maps: inner positions grouped by
    exponent e ascending, each group's triples ordered by lA and then either by t, or by the class
    (la_t, lb_t) of t descending and then t (one of the two for the whole plan), and padded with -1 to a
    multiple of IMQ_INNER_PAD; OUTER lines in groups of 32
    holding floor(32 / L) sources of one level L, the L lines of a source consecutive with levels
    0..L-1, sources sorted by (level, index); unused lines last in a group.  This checks the library
    against its own specification, not against the oracle."""
    I = plan.info
    mp = plan.maps() if mp is None else mp
    lv = plan.levels()
    # class of each inner index: its A column level when A is unpacked INNER, its B row level when B is
    cla = lv["a_col"].astype(np.int64) if I["dir_a"] & 2 else np.ones(I["K"], np.int64)
    clb = lv["b_row"].astype(np.int64) if I["dir_b"] & 2 else np.ones(I["K"], np.int64)
    in_order = {True: True, False: True}  # whether every group so far follows the index / class order
    for e, off, n, padded in plan.groups():
        assert off % 128 == 0 and padded % 128 == 0 and 0 <= padded - n < 128
        t, la, lb = mp["tK"][off:off + n], mp["lAk"][off:off + n], mp["lBk"][off:off + n]
        assert (t >= 0).all() and np.all(la.astype(int) + lb == e)
        tt = t.astype(np.int64)
        by_index = la.astype(np.int64) * (1 << 32) + tt
        by_class = la.astype(np.int64) * (1 << 60) + (63 - cla[tt]) * (1 << 54) + (63 - clb[tt]) * (1 << 48) + tt
        in_order[False] &= bool(np.all(np.diff(by_index) > 0))
        in_order[True] &= bool(np.all(np.diff(by_class) > 0))
        assert np.all(mp["tK"][off + n:off + padded] == -1)
    assert in_order[True] or in_order[False], "inner positions follow neither documented order"
    assert sum(g[3] for g in plan.groups()) == I["K_unp"]
    for src, lvl, lines, dirv in ((mp["srcA"], mp["lvlA"], lv["a_row"], I["dir_a"]),
                                  (mp["srcB"], mp["lvlB"], lv["b_col"], I["dir_b"])):
        if not dirv & 1:
            assert np.array_equal(src, np.arange(src.size)) and not lvl.any()
            continue
        G = 32
        assert src.size % G == 0
        seen = []
        for g0 in range(0, src.size, G):
            s, l = src[g0:g0 + G], lvl[g0:g0 + G]
            used = s >= 0
            n = int(used.sum())
            assert used[:n].all() and not used[n:].any()
            L = int(lines[s[0]])
            assert n % L == 0 and n // L <= G // L
            for k in range(n // L):
                assert np.all(s[k * L:(k + 1) * L] == s[k * L])
                assert np.array_equal(l[k * L:(k + 1) * L], np.arange(L))
                seen.append((L, int(s[k * L])))
        assert seen == sorted(seen) and len(seen) == lines.size


def unsupported(pl: oracle.Plan) -> bool:
    """True when the library must refuse the plan: the bound reaches 2^63 (C may leave int64)."""
    return int(round(pl.bound)) >= 2 ** 63
