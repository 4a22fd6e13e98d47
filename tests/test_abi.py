"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every function the
public header declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import mixture_experts_ffn_13_b200 as moe
from mixture_experts_ffn_13_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.load_library()


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)
    return names


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("moe_plan", "moe_route", "moe_forward", "moe_get_status", "moe_destroy", "moe_strerror"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in _declared_functions():
        assert hasattr(lib, n), n
        assert isinstance(getattr(lib, n), ctypes._CFuncPtr)


def test_strerror(lib):
    assert moe.moe_strerror(0) == "MOE_OK"
    for code, name in moe.ERRORS.items():
        assert moe.moe_strerror(code) == name
    assert moe.moe_strerror(12345) == "MOE_ERR_UNKNOWN"


def _plan_rc(lib, **kw):
    d = dict(T_max=16, H=512, E=8, I=256, k=2, I_shared=0, wfmt=1)
    d.update(kw)
    dims = moe.moe_dims(*(d[n] for n in ("T_max", "H", "E", "I", "k", "I_shared", "wfmt")))
    h = ctypes.c_void_p()
    ws = ctypes.c_size_t()
    return lib.moe_plan(ctypes.byref(dims), ctypes.byref(h), ctypes.byref(ws))


@pytest.mark.parametrize("kw,code", [
    (dict(k=0), -1), (dict(k=9), -1), (dict(T_max=0), -1), (dict(H=0), -1), (dict(wfmt=7), -1),
    (dict(I_shared=-128), -1), (dict(E=2048, k=2), -2), (dict(k=33, E=64), -2), (dict(H=520), -2),
    (dict(I=200), -2), (dict(I_shared=100), -2), (dict(wfmt=2, H=4100), -2), (dict(wfmt=3, H=4100), -2),
    (dict(wfmt=3, I=160), -2), (dict(wfmt=0), -1), (dict(wfmt=5), -1), (dict(wfmt=4, H=200), -2),
])
def test_plan_rejects_bad_dims(lib, kw, code):
    assert _plan_rc(lib, **kw) == code


def test_null_arguments_rejected(lib):
    assert lib.moe_plan(None, None, None) == -1
    assert lib.moe_route(None, 0, None, None, None, None, None, None, None, 0, None) == -1
    assert lib.moe_forward(None, 0, None, None, None, None, None, 0, None) == -1
    assert lib.moe_get_status(None, None) == -1
    lib.moe_destroy(None)


def test_binding_raises_without_library(tmp_path):
    import importlib
    with pytest.raises(RuntimeError):
        moe._lib = None
        try:
            moe.load_library(str(tmp_path / "missing.so"))
        finally:
            moe._lib = None


def test_binding_rejects_unknown_weight_format():
    with pytest.raises(ValueError):
        moe.Plan(16, 512, 8, 256, 2, 0, "fp4")
