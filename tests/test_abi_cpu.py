"""CPU checks of the boundary: the library builds for sm_100a, loads, and exports every entry point
declared in include/imq.h with the argument count the binding uses.  No compute calls."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "imq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    decls = {}
    for m in re.finditer(r"(?:imq_status|const char\s*\*)\s*(imq_\w+)\s*\(([^)]*)\)\s*;", text):
        args = [a for a in m.group(2).split(",") if a.strip() and a.strip() != "void"]
        decls[m.group(1)] = len(args)
    return decls


def test_header_declares_the_entry_points():
    d = _declared()
    for name in ("imq_rtn_quantize", "imq_plan", "imq_unpacked_gemm", "imq_unpack", "imq_gemm_unpacked",
                 "imq_plan_info_get", "imq_plan_levels", "imq_plan_groups", "imq_plan_destroy",
                 "imq_device_status", "imq_status_str", "imq_plan_unpack", "imq_rtn_quantize_rows_noalloc"):
        assert name in d, name


def test_library_builds_and_exports_every_declared_symbol():
    from bit_integer_gemm_b200 import build as b
    path = b.build()
    lib = ctypes.CDLL(path)
    import bit_integer_gemm_b200 as imq
    for name, nargs in _declared().items():
        assert hasattr(lib, name), f"{name} not exported"
        assert name in imq.SIGNATURES, f"{name} has no binding"
        assert len(imq.SIGNATURES[name]) == nargs, f"{name}: binding has {len(imq.SIGNATURES[name])} args, header {nargs}"


def test_debug_library_builds_and_exports_every_declared_symbol():
    from bit_integer_gemm_b200 import build as b
    lib = ctypes.CDLL(b.build(debug=True))
    for name in _declared():
        assert hasattr(lib, name), f"{name} not exported by the debug build"


def test_struct_layouts_match_header():
    import bit_integer_gemm_b200 as imq
    # imq_plan_info: 4 int32, 9 int64, 2 double, 6 int32, 8 int64, size_t
    assert ctypes.sizeof(imq.imq_plan_info) == 4 * 4 + 9 * 8 + 2 * 8 + 6 * 4 + 8 * 8 + 8
    assert ctypes.sizeof(imq.imq_group) == 32


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import bit_integer_gemm_b200 as imq
    monkeypatch.setattr(imq, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(imq, "_lib", None)
    with pytest.raises(RuntimeError):
        imq.lib()


def test_workspace_views_follow_the_documented_layout():
    """A' at the workspace's first 1024-byte boundary, B'^T at the next 1024-byte boundary after A' (the
    layout imq_plan_unpack and imq_unpacked_gemm use); views are reused for the same workspace and shape
    and rebuilt for another shape.  Host logic only: CPU tensors and a plan's info struct filled here."""
    import torch

    import bit_integer_gemm_b200 as imq

    class FakePlan:
        def __init__(self, m, n, k):
            self.raw = imq.imq_plan_info()
            self.raw.M_unp, self.raw.N_unp, self.raw.K_unp = m, n, k

    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    base = ws.data_ptr()
    for m, n, k in ((3, 5, 48), (64, 40, 256), (7, 1, 16)):
        p = FakePlan(m, n, k)
        a, b = imq.workspace_views(p, ws)
        off = (-base) % 1024
        assert a.data_ptr() == base + off and tuple(a.shape) == (m, k) and a.dtype == torch.int8
        assert b.data_ptr() == base + off + (m * k + 1023) // 1024 * 1024 and tuple(b.shape) == (n, k)
        assert (b.data_ptr() - base) % 1024 == off % 1024
        a2, b2 = imq.workspace_views(p, ws)
        assert a2 is a and b2 is b
        a[:] = 1
        assert int(ws[off:off + m * k].sum()) == m * k  # a view, not a copy
        ws.zero_()
