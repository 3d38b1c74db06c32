"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol the header declares, and rejects bad arguments before launching
anything."""
import ctypes
import os
import re
import subprocess

import pytest

from kolmogorov_arnold_network_b200 import _native as N
from kolmogorov_arnold_network_b200 import build as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "kan_b200.h")
FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced: every call below fails validation first


@pytest.fixture(scope="module")
def lib():
    B.build()
    return N.load()


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"KAN_API\s+[\w\s\*]+?\b(kan_\w+)\s*\(", src)))


def test_header_and_binding_agree():
    assert declared_symbols() == sorted(N.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", N.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (kan_\w+)", out))
    assert exported == set(declared_symbols())


def test_abi_version(lib):
    assert N.kan_abi_version() == 2


def test_shape_struct_layout():
    assert ctypes.sizeof(N.kan_shape) == 56
    assert N.kan_shape.G.offset == 24 and N.kan_shape.path.offset == 44 and N.kan_shape.degree.offset == 48


def st(code):
    return code


def fwd(shape, x=FAKE, coef=FAKE, wb=None, y=FAKE, ws=None, wsb=0):
    lib = N.load()
    return lib.kan_forward(ctypes.byref(shape) if shape is not None else None, x, coef, wb, y, ws, wsb, None)


def bwd(shape, x=FAKE, coef=FAKE, wb=None, dY=FAKE, dx=FAKE, dc=FAKE, dwb=None, ws=None, wsb=0):
    lib = N.load()
    return lib.kan_backward(ctypes.byref(shape) if shape is not None else None, x, coef, wb, dY, dx, dc, dwb, ws,
                            wsb, None)


def shp(**kw):
    d = dict(batch=64, n_in=16, n_out=32, G=8, lo=-1.0, hi=1.0, dtype=N.KAN_F32, has_base=False,
             path=N.KAN_PATH_AUTO)
    d.update(kw)
    return N.make_shape(**d)


@pytest.mark.parametrize("kw,code", [
    (dict(G=0), 1), (dict(G=-2), 1), (dict(G=251), 2), (dict(hi=-1.0), 1), (dict(lo=float("nan")), 1),
    (dict(hi=float("inf")), 1), (dict(n_in=0), 1), (dict(n_out=0), 1), (dict(batch=-1), 1), (dict(dtype=3), 1),
    (dict(path=7), 1), (dict(degree=0), 1), (dict(degree=6), 1),
])
def test_bad_shapes(lib, kw, code):
    assert fwd(shp(**kw)) == code
    assert bwd(shp(**kw)) == code
    n = ctypes.c_size_t(0)
    assert lib.kan_workspace_size(ctypes.byref(shp(**kw)), 0, ctypes.byref(n)) == code
    assert lib.kan_last_error().decode() != ""


def test_null_and_misaligned_pointers(lib):
    assert lib.kan_forward(None, FAKE, FAKE, None, FAKE, None, 0, None) == 1
    assert fwd(shp(), x=None) == 1
    assert fwd(shp(), y=None) == 1
    assert fwd(shp(), coef=None) == 1
    assert fwd(shp(), x=FAKE + 4) == 2
    assert fwd(shp(), y=FAKE + 8) == 2
    assert bwd(shp(), dY=None) == 1
    assert bwd(shp(), dc=FAKE + 2) == 2
    assert "aligned" in lib.kan_last_error().decode()


def test_base_branch_consistency(lib):
    assert fwd(shp(has_base=True), wb=None) == 1
    assert fwd(shp(has_base=False), wb=FAKE) == 1
    assert bwd(shp(has_base=False), dwb=FAKE) == 1


def test_forced_tensor_path_unsupported_stride(lib):
    # bf16, in=3, G=8: a coef row is 3*11*2 = 66 bytes, not a multiple of 16 (TMA row stride)
    s = shp(n_in=3, dtype=N.KAN_BF16, path=N.KAN_PATH_TENSOR)
    assert fwd(s) == 2
    assert "16 bytes" in lib.kan_last_error().decode()


def test_workspace_too_small(lib):
    # fp32 on the tensor path needs the fp16 hi/lo copies of coef (and the operand maxima)
    s = shp(batch=4096, n_in=64, n_out=256, path=N.KAN_PATH_TENSOR)
    need = ctypes.c_size_t(0)
    assert lib.kan_workspace_size(ctypes.byref(s), 0, ctypes.byref(need)) == 0
    assert need.value > 0
    assert fwd(s, ws=None, wsb=0) == 3
    assert fwd(s, ws=FAKE, wsb=need.value - 1) == 3


def test_simt_path_needs_no_workspace(lib):
    n = ctypes.c_size_t(123)
    assert lib.kan_workspace_size(ctypes.byref(shp(path=N.KAN_PATH_SIMT)), 1, ctypes.byref(n)) == 0
    assert n.value == 0


def test_selftest_limits(lib):
    assert lib.kan_selftest_wait_timeout(0, None) == 1
    assert lib.kan_selftest_wait_timeout(3_000_000_000, None) == 1


def test_status_strings(lib):
    for code in range(7):
        assert lib.kan_status_string(code).decode() not in ("", "unknown status")
    assert lib.kan_status_string(99).decode() == "unknown status"


def test_binding_raises_with_detail(lib):
    with pytest.raises(N.KanError) as ei:
        N.kan_forward(shp(G=0), FAKE, FAKE, None, FAKE, None, 0, None)
    assert ei.value.status == 1 and "G must be" in str(ei.value)
