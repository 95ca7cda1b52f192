"""CPU-side checks of the CUDA library: it builds for sm_100a, loads, and exports every
entry point that include/mimi_rvq.h declares. No compute call is made (no GPU here)."""
import ctypes
import os
import re

import pytest

import split_residual_vector_b200 as pkg
from split_residual_vector_b200 import build as lib_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(mimi_rvq_\w+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    lib_build.build()
    return ctypes.CDLL(lib_build.LIB)


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for required in ("mimi_rvq_create", "mimi_rvq_encode", "mimi_rvq_decode",
                     "mimi_rvq_encode_step", "mimi_rvq_destroy", "mimi_rvq_get_error",
                     "mimi_rvq_strerror"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_entry_points():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(pkg.EXPORTS) <= set(declared_entry_points())


def test_strerror_is_host_only(lib):
    lib.mimi_rvq_strerror.restype = ctypes.c_char_p
    assert lib.mimi_rvq_strerror(0) == b"ok"
    assert b"invalid" in lib.mimi_rvq_strerror(-1)
    assert b"outside" in lib.mimi_rvq_strerror(-4)
    assert lib.mimi_rvq_strerror(12345) == b"unknown status"


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(pkg, "_lib", None)
    monkeypatch.setattr(pkg, "LIBRARY_PATH", "/nonexistent/libmimi_rvq.so")
    with pytest.raises(ImportError):
        pkg.library()


def test_build_targets_sm100a_only():
    flags = " ".join(lib_build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert "sm_90" not in flags and "sm_80" not in flags
