"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before touching the GPU (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    # load the build script by path so a stale library is rebuilt before use
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "kda_build", os.path.join(ROOT, "kimi_delta_attention_26_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    build.build()
    return ctypes.CDLL(build.LIB)


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "kda.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert "kda_fwd" in names and len(names) >= 4
    for n in names:
        assert hasattr(lib, n), f"libkda.so does not export {n}"


def test_abi_version_and_status_strings(lib):
    lib.kda_abi_version.restype = ctypes.c_int32
    assert lib.kda_abi_version() == 2
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_status_string.argtypes = [ctypes.c_int]
    for code in range(6):
        assert len(lib.kda_status_string(code)) > 0
    assert lib.kda_status_string(99) == b"unknown status"


def _call(lib, q=0x1000, k=0x2000, v=0x3000, g=0x4000, beta=0x5000, scale=1.0, cu=0x6000, nseq=1,
          T=4, H=1, init=None, out=0x7000, fin=None):
    P = ctypes.c_void_p
    lib.kda_fwd.argtypes = [P, P, P, P, P, ctypes.c_float, P, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                            P, P, P, P]
    lib.kda_fwd.restype = ctypes.c_int
    return lib.kda_fwd(q, k, v, g, beta, scale, cu, nseq, T, H, init, out, fin, None)


def test_slice_columns_setting_validated(lib):
    lib.kda_set_slice_columns.argtypes = [ctypes.c_int32]
    lib.kda_set_slice_columns.restype = ctypes.c_int
    for bad in (-1, 1, 8, 24, 64, 128):
        assert lib.kda_set_slice_columns(bad) == 2  # KDA_ERR_SHAPE
    for good in (16, 32, 0):
        assert lib.kda_set_slice_columns(good) == 0


# These calls fail validation before any CUDA call, so the fake addresses are
# never dereferenced or handed to the driver.
def test_rejects_null_pointers(lib):
    for name in ("q", "k", "v", "g", "beta", "out"):
        assert _call(lib, **{name: None}) == 1, name
        # with T = 0 the token tensors are never touched, so NULL is fine; the
        # call then goes on to a misaligned init pointer and stops there
        assert _call(lib, T=0, init=0x8008, **{name: None}) == 3, name


def test_rejects_bad_shapes(lib):
    assert _call(lib, T=-1) == 2
    assert _call(lib, H=0) == 2
    assert _call(lib, nseq=0) == 2
    assert _call(lib, cu=None, nseq=2) == 2
    assert _call(lib, H=70000) == 2
    assert _call(lib, T=1 << 40, H=32) == 2


def test_rejects_misaligned_pointers(lib):
    for name in ("q", "k", "v", "g", "beta", "out", "init", "fin", "cu"):
        assert _call(lib, **{name: 0x8008}) == 3, name


def test_wait_timeouts_rejects_null(lib):
    lib.kda_wait_timeouts.argtypes = [ctypes.c_void_p, ctypes.c_int32]
    lib.kda_wait_timeouts.restype = ctypes.c_int
    assert lib.kda_wait_timeouts(None, 0) == 1
