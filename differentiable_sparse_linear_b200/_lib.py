"""ctypes declarations of libsla's C ABI (include/sla.h).  Loading only; no arithmetic."""
from __future__ import annotations

import ctypes as C
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "lib", "libsla.so")

SLA_SUCCESS = 0
SLA_NOT_CONVERGED = 1
SLA_BREAKDOWN = 2
SLA_ERR_INVALID_ARG = -1
SLA_ERR_INVALID_CSR = -2
SLA_ERR_CUDA = -3
SLA_ERR_OOM = -4
SLA_ERR_UNSUPPORTED = -5
SLA_F32 = 0
SLA_F64 = 1
SLA_SPD = 1
SLA_VALIDATE = 2
SLA_STATIC_VALUES = 4
SLA_ENGINE_AUTO = 0
SLA_ENGINE_GRAPH = 1
SLA_ENGINE_PERSISTENT = 2
SLA_ENGINE_LIST = 3


class sla_pcg_opts(C.Structure):
    _fields_ = [("rtol", C.c_double), ("maxit", C.c_int64), ("vector_f64", C.c_int32),
                ("engine", C.c_int32)]


class sla_pcg_info(C.Structure):
    _fields_ = [("iters", C.c_int64), ("relres", C.c_double), ("status", C.c_int32),
                ("engine", C.c_int32)]


_vp = C.c_void_p
_st = C.c_int32

# name -> (restype, argtypes)
SIGNATURES = {
    "sla_version": (C.c_char_p, []),
    "sla_status_string": (C.c_char_p, [_st]),
    "sla_last_error": (C.c_char_p, []),
    "sla_csr_create": (_st, [C.POINTER(_vp), C.c_int64, C.c_int64, C.c_int64, _vp, _vp, _vp,
                             C.c_int, C.c_uint32, _vp]),
    "sla_csr_create_list": (_st, [C.POINTER(_vp), C.c_int32, C.POINTER(C.c_int64), C.c_int64, _vp,
                                  _vp, _vp, C.c_int, C.c_uint32, _vp]),
    "sla_bsr_create": (_st, [C.POINTER(_vp), C.c_int64, C.c_int32, C.c_int64, _vp, _vp, _vp,
                             C.c_int, C.c_uint32, _vp]),
    "sla_csr_destroy": (_st, [_vp]),
    "sla_csr_values_changed": (_st, [_vp, _vp]),
    "sla_csr_shape": (_st, [_vp, C.POINTER(C.c_int64), C.POINTER(C.c_int64), C.POINTER(C.c_int32)]),
    "sla_spmv": (_st, [_vp, _vp, _vp, _vp]),
    "sla_spmv_multi": (_st, [_vp, C.c_int32, _vp, _vp, _vp]),
    "sla_precond_jacobi": (_st, [C.POINTER(_vp), _vp, _vp]),
    "sla_precond_spai": (_st, [C.POINTER(_vp), _vp, _vp, C.c_double, _vp]),
    "sla_precond_refresh": (_st, [_vp, _vp]),
    "sla_precond_destroy": (_st, [_vp]),
    "sla_pcg_solve": (_st, [_vp, _vp, _vp, _vp, C.POINTER(sla_pcg_opts), C.POINTER(sla_pcg_info), _vp]),
    "sla_pcg_adjoint": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, C.POINTER(sla_pcg_opts),
                              C.POINTER(sla_pcg_info), _vp]),
    "sla_pcg_solve_batched": (_st, [_vp, _vp, C.c_int32, _vp, _vp, C.POINTER(sla_pcg_opts),
                                    C.POINTER(sla_pcg_info), _vp]),
    "sla_pcg_adjoint_batched": (_st, [_vp, _vp, C.c_int32, _vp, _vp, _vp, _vp,
                                      C.POINTER(sla_pcg_opts), C.POINTER(sla_pcg_info), _vp]),
    "sla_pattern_grad": (_st, [_vp, C.c_int32, _vp, _vp, _vp, _vp]),
    "sla_eigen_grad": (_st, [_vp, C.c_int32, _vp, _vp, _vp]),
    "sla_csr_add_diagonal": (_st, [_vp, _vp, _vp, _vp]),
    "sla_nonlinear_adjoint": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, C.POINTER(sla_pcg_opts),
                                    C.POINTER(sla_pcg_info), _vp]),
    "sla_vec_dot": (_st, [C.c_int32, C.c_int64, _vp, _vp, _vp, _vp]),
    "sla_pcg_update": (_st, [C.c_int32, C.c_int64, C.c_double, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "sla_pcg_direction": (_st, [C.c_int32, C.c_int64, C.c_double, _vp, _vp, _vp]),
    "sla_vec_gather": (_st, [C.c_int32, C.c_int64, _vp, _vp, _vp, _vp]),
    "sla_vec_scatter_add": (_st, [C.c_int32, C.c_int64, _vp, _vp, _vp, _vp]),
    "sla_list_kernel_ms": (_st, [_vp, C.POINTER(C.c_double)]),
    "sla_pcg_solve_batched_noalloc": (_st, [_vp, _vp, _vp, _vp, C.POINTER(sla_pcg_opts),
                                            C.POINTER(sla_pcg_info), _vp]),
    "sla_pcg_kernel_times": (_st, [_vp, _vp, C.c_int32, C.c_int32, C.c_int32, C.POINTER(C.c_double), _vp]),
    "sla_pcg_phase_times": (_st, [_vp, _vp, C.c_int32, C.c_int32, C.POINTER(C.c_double),
                                  C.POINTER(C.c_int64), _vp]),
    "sla_workspace_bytes": (C.c_size_t, [_vp, _vp, C.c_int32, C.c_int32]),
}

_lib = None


def load(path: str = LIB_PATH) -> C.CDLL:
    """Load libsla.so once; raise if it has not been built (there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            f"libsla.so not found at {path}: build it with "
            "`python -m differentiable_sparse_linear_b200.build` (nvcc, sm_100a)")
    lib = C.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
