"""The C-ABI library loads and exports every entry point declared in
include/effort.h, and host-side argument checks reject bad calls before any
device work.  No GPU is needed: only calls that fail validation are made."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "effort.h")


@pytest.fixture(scope="module")
def L():
    from dynamic_approximate_gemv_b200 import build
    build.build()
    import dynamic_approximate_gemv_b200 as E
    return E.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:effort_status_t|const char\*)\s+(effort_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("effort_prepare", "effort_prepare_q8", "effort_gemv", "effort_gemv_ex", "effort_gemv_host", "effort_gemv_batched",
                 "effort_destroy",
                 "effort_dense_gemv", "effort_workspace_create", "effort_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    assert L.effort_status_string(0) == b"ok"
    assert L.effort_status_string(1) == b"invalid argument"
    assert L.effort_status_string(99) == b"unknown status"


def test_argument_errors_need_no_device(L):
    vp = ctypes.c_void_p
    h = vp()
    fake = vp(0x100000)  # never dereferenced: every call below fails validation first
    assert L.effort_prepare(None, 4, 4, ctypes.c_float(1.0), None, ctypes.byref(h)) == 1
    assert L.effort_prepare(fake, 0, 4, ctypes.c_float(1.0), None, ctypes.byref(h)) == 1
    assert L.effort_prepare(fake, 4, 4, ctypes.c_float(0.0), None, ctypes.byref(h)) == 1
    assert L.effort_prepare(fake, 4, 4, ctypes.c_float(1.5), None, ctypes.byref(h)) == 1
    assert L.effort_prepare(fake, 4, 4, ctypes.c_float(float("nan")), None, ctypes.byref(h)) == 1
    assert L.effort_prepare(vp(0x100001), 4, 4, ctypes.c_float(1.0), None, ctypes.byref(h)) == 1
    assert L.effort_prepare(fake, 4, 40000, ctypes.c_float(1.0), None, ctypes.byref(h)) == 6
    assert L.effort_prepare(fake, 50000, 4, ctypes.c_float(1.0), None, ctypes.byref(h)) == 6
    assert L.effort_prepare(fake, 4, 10, ctypes.c_float(0.04), None, ctypes.byref(h)) == 1  # keeps nothing
    q8 = L.effort_prepare_q8
    q8.argtypes = [vp, vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_float, vp, ctypes.POINTER(vp)]
    assert q8(None, fake, 4, 4, ctypes.c_float(1.0), None, ctypes.byref(h)) == 1      # no q
    assert q8(vp(0x100001), None, 4, 4, ctypes.c_float(1.0), None, ctypes.byref(h)) == 1  # no scales
    assert q8(vp(0x100001), vp(0x100001), 4, 4, ctypes.c_float(1.0), None, ctypes.byref(h)) == 1  # odd scales
    assert q8(vp(0x100001), fake, 4, 4, ctypes.c_float(0.0), None, ctypes.byref(h)) == 1
    assert q8(vp(0x100001), fake, 4, 40000, ctypes.c_float(1.0), None, ctypes.byref(h)) == 6
    assert q8(fake, fake, 4, 4, ctypes.c_float(1.0), None, None) == 1
    assert L.effort_gemv(None, fake, ctypes.c_float(0.5), fake, None) == 1
    assert L.effort_gemv_ex(None, fake, 0, ctypes.c_float(0.5), fake, None, None, None, None) == 1
    assert L.effort_gemv_host(None, fake, 0, ctypes.c_float(0.5), fake, None) == 1
    assert L.effort_check(None) == 1
    assert L.effort_destroy(None) == 1
    w = vp()
    assert L.effort_workspace_create(0, 4, 1, ctypes.byref(w)) == 1
    assert L.effort_workspace_create(4, 4, 0, ctypes.byref(w)) == 1
    assert L.effort_workspace_create(4, 40000, 1, ctypes.byref(w)) == 6
    assert L.effort_workspace_destroy(None) == 1
    assert L.effort_gemv_batched(None, None, None, None, 1, None, 0, None, None, None, None, None) == 1
    assert L.effort_dense_gemv(None, fake, 4, 4, fake, 0, fake, None) == 1
    assert L.effort_get_info(None, None, None, None, None) == 1
    assert L.effort_get_layout(None, None) == 1
    assert L.effort_workspace_check(None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import dynamic_approximate_gemv_b200 as E
    monkeypatch.setattr(E, "_lib", None)
    monkeypatch.setattr(E, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        E.lib()


def test_allocation_cap_gives_nomem_before_any_device_call(L, monkeypatch):
    """With the library's allocation cap below what a matrix needs,
    effort_prepare returns EFFORT_ERR_NOMEM (3) before it touches CUDA: the
    pointer below is never dereferenced and no GPU is present."""
    vp = ctypes.c_void_p
    h = vp()
    fake = vp(0x100000)
    monkeypatch.setenv("EFFORT_ALLOC_CAP_BYTES", "4096")
    assert L.effort_prepare(fake, 4096, 14336, ctypes.c_float(1.0), None, ctypes.byref(h)) == 3
    assert h.value is None
    assert L.effort_prepare(fake, 64, 64, ctypes.c_float(0.5), None, ctypes.byref(h)) == 3
    # argument errors still come first
    assert L.effort_prepare(fake, 0, 64, ctypes.c_float(1.0), None, ctypes.byref(h)) == 1
    held = ctypes.c_uint64(1)
    assert L.effort_device_bytes_held(ctypes.byref(held)) == 0
    assert held.value == 0


def test_debug_library_exports_the_same_symbols():
    """The bounds-checking build (kernels compiled with EFFORT_DEBUG) is a
    drop-in: it exports every entry point the header declares."""
    from dynamic_approximate_gemv_b200 import build
    import dynamic_approximate_gemv_b200 as E
    build.build()
    D = ctypes.CDLL(E.LIB_DEBUG_PATH)
    for name in declared_functions():
        assert hasattr(D, name), name
