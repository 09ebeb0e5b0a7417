"""The C-ABI library builds, loads without a GPU, and exports every symbol include/sla.h
declares (no compute calls: those need a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "sla.h")).read()
    return sorted(set(re.findall(r"SLA_API[^;(]*?\b(sla_\w+)\s*\(", text, flags=re.S)))


@pytest.fixture(scope="module")
def libsla():
    from differentiable_sparse_linear_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_entry_points():
    names = declared_symbols()
    for must in ("sla_csr_create", "sla_pcg_solve", "sla_pcg_adjoint", "sla_pcg_solve_batched",
                 "sla_pcg_adjoint_batched", "sla_spmv", "sla_precond_spai", "sla_precond_jacobi"):
        assert must in names


def test_every_declared_symbol_is_exported(libsla):
    missing = [n for n in declared_symbols() if not hasattr(libsla, n)]
    assert not missing, f"declared but not exported: {missing}"


def test_binding_covers_every_symbol():
    from differentiable_sparse_linear_b200 import _lib
    assert set(declared_symbols()) == set(_lib.SIGNATURES)


def test_host_only_calls(libsla):
    libsla.sla_version.restype = ctypes.c_char_p
    assert b"sm_100a" in libsla.sla_version()
    libsla.sla_status_string.restype = ctypes.c_char_p
    libsla.sla_status_string.argtypes = [ctypes.c_int32]
    assert libsla.sla_status_string(-2) == b"SLA_ERR_INVALID_CSR"
    # argument checks run before any device work
    libsla.sla_csr_create.restype = ctypes.c_int32
    assert libsla.sla_csr_create(None, 4, 4, 0, None, None, None, 0, 0, None) == -1
    h = ctypes.c_void_p()
    assert libsla.sla_csr_create(ctypes.byref(h), 4, 5, 0, None, None, None, 0, 0, None) == -1


def test_bsr_argument_checks(libsla):
    """sla_bsr_create refuses bad block sizes, shapes and pointers before any device work."""
    f = libsla.sla_bsr_create
    f.restype = ctypes.c_int32
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_uint32, ctypes.c_void_p]
    h = ctypes.c_void_p()
    assert f(None, 4, 3, 0, None, None, None, 0, 0, None) == -1               # out is NULL
    for bdim in (0, 1, 5):
        assert f(ctypes.byref(h), 4, bdim, 0, 16, None, None, 0, 0, None) == -1
    assert f(ctypes.byref(h), -1, 3, 0, 16, None, None, 0, 0, None) == -1     # negative size
    assert f(ctypes.byref(h), 2 ** 30, 3, 0, 16, None, None, 0, 0, None) == -1  # int32 overflow
    assert f(ctypes.byref(h), 4, 3, 0, 16, None, None, 7, 0, None) == -1      # bad dtype
    assert f(ctypes.byref(h), 4, 3, 5, 16, None, None, 0, 0, None) == -1      # nnzb > 0, no col
    assert f(ctypes.byref(h), 4, 3, 0, 24, None, None, 0, 0, None) == -1      # row_ptr not 16-aligned
    assert h.value is None


def test_no_cpu_fallback_in_binding():
    """The binding has no arithmetic path of its own: it never imports the oracle."""
    pkg = os.path.join(ROOT, "differentiable_sparse_linear_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn)).read()
            assert "oracle" not in src.replace("the oracle", ""), fn
