"""Differentiable sparse SPD solve on B200: Python binding of libsla (include/sla.h).

Every computation runs in libsla's CUDA kernels; this module only marshals torch tensors
(device pointers, the current CUDA stream) into the C ABI and back.  There is no CPU or
PyTorch fallback: without the built library, or without a CUDA device, calls raise.

Functions keep the C names (``sla_spmv``, ``sla_pcg_solve``, ``sla_pcg_adjoint`` ...).
``solve(A, b, M)`` is the differentiable entry point: its backward pass is the adjoint of
"torch-sla: Differentiable Sparse Linear Algebra with Adjoint Solvers and Sparse Tensor
Parallelism for PyTorch", Methodology §2 (Linear Systems): one solve with A^T = A,
dL/db = lambda, dL/dA_ij = -lambda_i x_j on A's pattern; only x is saved for backward.
"""
from __future__ import annotations

import collections.abc as _abc
import ctypes as C
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np
import torch

from . import _lib
from ._lib import (SLA_BREAKDOWN, SLA_ERR_CUDA, SLA_ERR_INVALID_ARG, SLA_ERR_INVALID_CSR,
                   SLA_ERR_OOM, SLA_ERR_UNSUPPORTED, SLA_F32, SLA_F64, SLA_NOT_CONVERGED,
                   SLA_SPD, SLA_STATIC_VALUES, SLA_SUCCESS, SLA_VALIDATE)

__all__ = [
    "SlaError", "Matrix", "Preconditioner", "PcgInfo", "PcgInfoList", "lib",
    "sla_version", "sla_csr_create", "sla_csr_values_changed", "sla_bsr_create", "sla_csr_create_list", "sla_spmv", "sla_spmv_multi",
    "sla_precond_jacobi", "sla_precond_spai", "sla_pcg_solve", "sla_pcg_adjoint",
    "sla_pcg_solve_batched", "sla_pcg_adjoint_batched", "sla_pattern_grad",
    "sla_pcg_solve_batched_noalloc", "sla_list_kernel_ms", "sla_eigen_grad", "sla_csr_add_diagonal", "sla_nonlinear_adjoint",
    "sla_vec_dot", "sla_pcg_update", "sla_pcg_direction", "sla_vec_gather", "sla_vec_scatter_add",
    "sla_workspace_bytes", "sla_pcg_kernel_times", "sla_pcg_phase_times", "solve",
    "ENGINES",
]


def lib() -> C.CDLL:
    return _lib.load()


class SlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        L = lib()
        name = L.sla_status_string(status).decode()
        detail = L.sla_last_error().decode()
        super().__init__(f"{where}: {name}: {detail}")
        self.status = status


def _check(status: int, where: str) -> int:
    if status < 0:
        raise SlaError(status, where)
    return status


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libsla takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libsla takes contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return SLA_F32
    if dt == torch.float64:
        return SLA_F64
    raise ValueError(f"values must be float32 or float64, got {dt}")


# solve engines (SLA_ENGINE_*): "auto" takes the persistent engine where it applies
ENGINES = {"auto": 0, "graph": 1, "persistent": 2}
_ENGINE_NAMES = {0: "auto", 1: "graph", 2: "persistent", 3: "list"}


@dataclass
class PcgInfo:
    iters: int
    relres: float
    status: int
    engine: str = "auto"

    @property
    def converged(self) -> bool:
        return self.status == SLA_SUCCESS


class PcgInfoList(_abc.Sequence):
    """Per-system (or per-right-hand-side) results of a batched solve: a sequence of PcgInfo,
    each made when it is read, over the arrays `iters`, `relres`, `status` and `engine_codes`
    copied once from the library's result structs (a list of thousands of systems reads them
    in bulk, not one Python object per system)."""

    __slots__ = ("iters", "relres", "status", "engine_codes")

    def __init__(self, arr):
        a = np.ctypeslib.as_array(arr)
        self.iters = a["iters"].astype(np.int64)
        self.relres = a["relres"].astype(np.float64)
        self.status = a["status"].astype(np.int32)
        self.engine_codes = a["engine"].astype(np.int32)

    def __len__(self) -> int:
        return int(self.iters.shape[0])

    def __getitem__(self, i):
        if isinstance(i, slice):
            return [self[j] for j in range(*i.indices(len(self)))]
        return PcgInfo(int(self.iters[i]), float(self.relres[i]), int(self.status[i]),
                       _ENGINE_NAMES.get(int(self.engine_codes[i]), "?"))

    def __add__(self, other):
        return list(self) + list(other)

    def __radd__(self, other):
        return list(other) + list(self)

    @property
    def engines(self) -> set:
        return {_ENGINE_NAMES.get(int(e), "?") for e in np.unique(self.engine_codes)}


def _infos(arr) -> PcgInfoList:
    return PcgInfoList(arr)


def _info1(a) -> PcgInfo:
    return PcgInfo(int(a.iters), float(a.relres), int(a.status), _ENGINE_NAMES.get(int(a.engine), "?"))


def _opts(rtol: float, maxit: int, vector_f64: bool = False, engine: str = "auto") -> _lib.sla_pcg_opts:
    if engine not in ENGINES:
        raise ValueError(f"engine must be one of {sorted(ENGINES)}, got {engine!r}")
    o = _lib.sla_pcg_opts()
    o.rtol = float(rtol)
    o.maxit = int(maxit)
    o.vector_f64 = 1 if vector_f64 else 0
    o.engine = ENGINES[engine]
    return o


def sla_version() -> str:
    return lib().sla_version().decode()


class Matrix:
    """Handle on a CSR matrix held in CUDA tensors (int32 row_ptr/col, fp32/fp64 values).

    The tensors are borrowed by the library; this object keeps them alive.
    """

    def __init__(self, handle: int, row_ptr, col, val, sys_row_off=None, block: int = 1):
        self._h = C.c_void_p(handle)
        self.row_ptr, self.col, self.val = row_ptr, col, val
        self.sys_row_off = sys_row_off
        self.block = block                       # BSR block size (1: CSR)
        self.n = (row_ptr.numel() - 1) * block   # scalar rows
        self.nnz = col.numel() * block * block   # stored scalar values
        self.dtype = val.dtype
        self.batch = 1 if sys_row_off is None else len(sys_row_off) - 1

    @property
    def handle(self) -> C.c_void_p:
        if self._h is None or not self._h.value:
            raise ValueError("matrix handle is closed")
        return self._h

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().sla_csr_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def matvec(self, x: torch.Tensor) -> torch.Tensor:
        return sla_spmv(self, x)


class Preconditioner:
    def __init__(self, handle: int, kind: str, A: Matrix, G: Optional[Matrix] = None, eps: float = 0.0):
        self._h = C.c_void_p(handle)
        self.kind, self.A, self.G, self.eps = kind, A, G, eps

    @property
    def handle(self) -> C.c_void_p:
        if self._h is None or not self._h.value:
            raise ValueError("preconditioner handle is closed")
        return self._h

    def refresh(self, stream=None):
        _check(lib().sla_precond_refresh(self.handle, _stream(stream)), "sla_precond_refresh")

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().sla_precond_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _mh(M: Optional[Preconditioner]):
    return None if M is None else M.handle


def _check_vec(A: Matrix, v: torch.Tensor, vector_f64: bool):
    want = torch.float64 if (vector_f64 and A.dtype == torch.float32) else A.dtype
    if v.dtype != want:
        raise ValueError(f"vectors must be {want} here (matrix {A.dtype}, vector_f64={vector_f64})")


def sla_csr_create(row_ptr: torch.Tensor, col: torch.Tensor, val: torch.Tensor, *,
                   validate: bool = True, spd: bool = True, static_values: bool = False,
                   stream=None) -> Matrix:
    """sla_csr_create: one square CSR matrix (n = row_ptr.numel() - 1).  static_values: the
    caller changes the values only with sla_csr_values_changed (SLA_STATIC_VALUES)."""
    n = row_ptr.numel() - 1
    if row_ptr.dtype != torch.int32 or col.dtype != torch.int32:
        raise ValueError("row_ptr and col must be int32")
    h = C.c_void_p()
    flags = ((SLA_VALIDATE if validate else 0) | (SLA_SPD if spd else 0)
             | (SLA_STATIC_VALUES if static_values else 0))
    _check(lib().sla_csr_create(C.byref(h), n, n, col.numel(), _ptr(row_ptr), _ptr(col), _ptr(val),
                                _dtype_code(val.dtype), flags, _stream(stream)), "sla_csr_create")
    return Matrix(h.value, row_ptr, col, val)


def sla_csr_values_changed(A: Matrix, stream=None) -> None:
    """The values of a SLA_STATIC_VALUES handle were changed in place."""
    _check(lib().sla_csr_values_changed(A.handle, _stream(stream)), "sla_csr_values_changed")


def sla_bsr_create(row_ptr: torch.Tensor, col: torch.Tensor, val: torch.Tensor, *,
                   validate: bool = True, spd: bool = True, stream=None) -> Matrix:
    """sla_bsr_create: one square block sparse row matrix; val is [nnzb, b, b] (row-major
    blocks), row_ptr / col index the blocks.  Gradients on its pattern come back flat,
    aligned with val's elements."""
    if row_ptr.dtype != torch.int32 or col.dtype != torch.int32:
        raise ValueError("row_ptr and col must be int32")
    if val.dim() != 3 or val.shape[1] != val.shape[2] or val.shape[0] != col.numel():
        raise ValueError("val must be [nnzb, b, b]")
    if not val.is_contiguous():
        raise ValueError("val must be contiguous")
    b = int(val.shape[1])
    h = C.c_void_p()
    flags = (SLA_VALIDATE if validate else 0) | (SLA_SPD if spd else 0)
    _check(lib().sla_bsr_create(C.byref(h), row_ptr.numel() - 1, b, col.numel(), _ptr(row_ptr), _ptr(col),
                                _ptr(val), _dtype_code(val.dtype), flags, _stream(stream)), "sla_bsr_create")
    return Matrix(h.value, row_ptr, col, val, block=b)


def sla_csr_create_list(sys_row_off: Sequence[int], row_ptr: torch.Tensor, col: torch.Tensor,
                        val: torch.Tensor, *, validate: bool = True, spd: bool = True,
                        stream=None) -> Matrix:
    """sla_csr_create_list: independent systems as one block-diagonal CSR (global columns)."""
    off = (C.c_int64 * len(sys_row_off))(*[int(v) for v in sys_row_off])
    h = C.c_void_p()
    flags = (SLA_VALIDATE if validate else 0) | (SLA_SPD if spd else 0)
    _check(lib().sla_csr_create_list(C.byref(h), len(sys_row_off) - 1, off, col.numel(), _ptr(row_ptr),
                                     _ptr(col), _ptr(val), _dtype_code(val.dtype), flags,
                                     _stream(stream)), "sla_csr_create_list")
    return Matrix(h.value, row_ptr, col, val, sys_row_off=list(sys_row_off))


def sla_spmv(A: Matrix, x: torch.Tensor, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    y = torch.empty(A.n, dtype=A.dtype, device=x.device) if y is None else y
    _check(lib().sla_spmv(A.handle, _ptr(x), _ptr(y), _stream(stream)), "sla_spmv")
    return y


def sla_spmv_multi(A: Matrix, X: torch.Tensor, Y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    nrhs = X.shape[1]
    Y = torch.empty_like(X) if Y is None else Y
    _check(lib().sla_spmv_multi(A.handle, nrhs, _ptr(X), _ptr(Y), _stream(stream)), "sla_spmv_multi")
    return Y


def sla_precond_jacobi(A: Matrix, stream=None) -> Preconditioner:
    h = C.c_void_p()
    _check(lib().sla_precond_jacobi(C.byref(h), A.handle, _stream(stream)), "sla_precond_jacobi")
    return Preconditioner(h.value, "jacobi", A)


def sla_precond_spai(A: Matrix, G: Matrix, eps: float = 3e-3, stream=None) -> Preconditioner:
    h = C.c_void_p()
    _check(lib().sla_precond_spai(C.byref(h), A.handle, G.handle, float(eps), _stream(stream)),
           "sla_precond_spai")
    return Preconditioner(h.value, "spai", A, G, eps)


def sla_pcg_solve(A: Matrix, M: Optional[Preconditioner], b: torch.Tensor,
                  x: Optional[torch.Tensor] = None, *, rtol: float = 0.0, maxit: int = 0,
                  vector_f64: bool = False, engine: str = "auto", stream=None) -> tuple[torch.Tensor, PcgInfo]:
    """x = A^-1 b.  vector_f64 with an fp32 matrix: b and x are fp64 (mixed precision)."""
    _check_vec(A, b, vector_f64)
    x = torch.empty_like(b) if x is None else x
    info = _lib.sla_pcg_info()
    opts = _opts(rtol, maxit, vector_f64, engine)
    _check(lib().sla_pcg_solve(A.handle, _mh(M), _ptr(b), _ptr(x), C.byref(opts), C.byref(info),
                               _stream(stream)), "sla_pcg_solve")
    return x, _info1(info)


def sla_pcg_adjoint(A: Matrix, M: Optional[Preconditioner], x: torch.Tensor, dLdx: torch.Tensor, *,
                    want_dA: bool = True, rtol: float = 0.0, maxit: int = 0, vector_f64: bool = False,
                    engine: str = "auto", dLdb: Optional[torch.Tensor] = None,
                    dLdA: Optional[torch.Tensor] = None, stream=None):
    """Returns (dL/db, dL/dA on A's pattern or None, info); dLdb / dLdA: optional outputs."""
    _check_vec(A, dLdx, vector_f64)
    dLdb = torch.empty_like(dLdx) if dLdb is None else dLdb
    if want_dA and dLdA is None:
        dLdA = torch.empty(A.nnz, dtype=A.dtype, device=dLdx.device)
    elif not want_dA:
        dLdA = None
    info = _lib.sla_pcg_info()
    opts = _opts(rtol, maxit, vector_f64, engine)
    _check(lib().sla_pcg_adjoint(A.handle, _mh(M), _ptr(x), _ptr(dLdx), _ptr(dLdb), _ptr(dLdA),
                                 C.byref(opts), C.byref(info), _stream(stream)), "sla_pcg_adjoint")
    return dLdb, dLdA, _info1(info)


def sla_pcg_solve_batched(A: Matrix, M: Optional[Preconditioner], B: torch.Tensor,
                          X: Optional[torch.Tensor] = None, *, rtol: float = 0.0, maxit: int = 0,
                          vector_f64: bool = False, engine: str = "auto", stream=None) -> tuple[torch.Tensor, PcgInfoList]:
    """Shared matrix: B is [n, nrhs].  List handle: B is the concatenated [n_total] vector."""
    _check_vec(A, B, vector_f64)
    nrhs = 1 if (B.dim() == 1 or A.batch > 1) else B.shape[1]
    count = A.batch if A.batch > 1 else nrhs
    X = torch.empty_like(B) if X is None else X
    infos = (_lib.sla_pcg_info * count)()
    opts = _opts(rtol, maxit, vector_f64, engine)
    _check(lib().sla_pcg_solve_batched(A.handle, _mh(M), nrhs, _ptr(B), _ptr(X), C.byref(opts),
                                       infos, _stream(stream)), "sla_pcg_solve_batched")
    return X, _infos(infos)


def sla_list_kernel_ms(A: Matrix) -> float:
    """Device ms of the list kernel of the last (regular) list solve on list handle A."""
    ms = C.c_double(0.0)
    _check(lib().sla_list_kernel_ms(A.handle, C.byref(ms)), "sla_list_kernel_ms")
    return ms.value


def sla_pcg_solve_batched_noalloc(A: Matrix, M: Optional[Preconditioner], B: torch.Tensor,
                                  X: Optional[torch.Tensor] = None, *, rtol: float = 0.0, maxit: int = 0,
                                  stream=None) -> tuple[torch.Tensor, PcgInfoList]:
    """List-handle solve that allocates no device memory inside the call (X must be given
    by callers that cannot allocate either; here it is created when omitted)."""
    X = torch.empty_like(B) if X is None else X
    infos = (_lib.sla_pcg_info * A.batch)()
    opts = _opts(rtol, maxit)
    _check(lib().sla_pcg_solve_batched_noalloc(A.handle, _mh(M), _ptr(B), _ptr(X), C.byref(opts), infos,
                                               _stream(stream)), "sla_pcg_solve_batched_noalloc")
    return X, _infos(infos)


def sla_pcg_adjoint_batched(A: Matrix, M: Optional[Preconditioner], X: torch.Tensor, dLdX: torch.Tensor,
                            *, want_dA: bool = True, rtol: float = 0.0, maxit: int = 0,
                            vector_f64: bool = False, engine: str = "auto", dLdB: Optional[torch.Tensor] = None,
                            dLdA: Optional[torch.Tensor] = None, stream=None):
    """Returns (dL/dB, dL/dA on A's pattern or None, infos); dLdB / dLdA: optional outputs."""
    _check_vec(A, dLdX, vector_f64)
    nrhs = 1 if (dLdX.dim() == 1 or A.batch > 1) else dLdX.shape[1]
    count = A.batch if A.batch > 1 else nrhs
    dLdB = torch.empty_like(dLdX) if dLdB is None else dLdB
    if want_dA and dLdA is None:
        dLdA = torch.empty(A.nnz, dtype=A.dtype, device=dLdX.device)
    elif not want_dA:
        dLdA = None
    infos = (_lib.sla_pcg_info * count)()
    opts = _opts(rtol, maxit, vector_f64, engine)
    _check(lib().sla_pcg_adjoint_batched(A.handle, _mh(M), nrhs, _ptr(X), _ptr(dLdX), _ptr(dLdB),
                                         _ptr(dLdA), C.byref(opts), infos, _stream(stream)),
           "sla_pcg_adjoint_batched")
    return dLdB, dLdA, _infos(infos)


def sla_pattern_grad(A: Matrix, lam: torch.Tensor, x: torch.Tensor, g: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    nrhs = 1 if lam.dim() == 1 else lam.shape[1]
    g = torch.empty(A.nnz, dtype=A.dtype, device=lam.device) if g is None else g
    _check(lib().sla_pattern_grad(A.handle, nrhs, _ptr(lam), _ptr(x), _ptr(g), _stream(stream)),
           "sla_pattern_grad")
    return g


def sla_eigen_grad(A: Matrix, V: torch.Tensor, g: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """d mu / d A_k = v_row(k) v_col(k) on A's pattern for unit eigenvector(s) V ([n] or
    [n, nvec]; summed over the columns)."""
    nvec = 1 if V.dim() == 1 else V.shape[1]
    _check_vec(A, V, False)
    g = torch.empty(A.nnz, dtype=A.dtype, device=V.device) if g is None else g
    _check(lib().sla_eigen_grad(A.handle, nvec, _ptr(V), _ptr(g), _stream(stream)), "sla_eigen_grad")
    return g


def sla_csr_add_diagonal(A: Matrix, c: torch.Tensor, out: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """Values of A + diag(c) on A's pattern (e.g. a Jacobian J = A + diag(N'(u)))."""
    _check_vec(A, c, False)
    out = torch.empty_like(A.val.reshape(-1)) if out is None else out
    _check(lib().sla_csr_add_diagonal(A.handle, _ptr(c), _ptr(out), _stream(stream)), "sla_csr_add_diagonal")
    return out


def sla_nonlinear_adjoint(J: Matrix, M: Optional[Preconditioner], A: Optional[Matrix], u: torch.Tensor,
                          dLdu: torch.Tensor, *, want_dA: bool = True, rtol: float = 0.0, maxit: int = 0,
                          vector_f64: bool = False, engine: str = "auto", lam: Optional[torch.Tensor] = None,
                          dLdA: Optional[torch.Tensor] = None, stream=None):
    """Backward pass of F(u) = A u + N(u) - b = 0 at its solution u: solves J^T lambda = dL/du
    (J = A + diag(N'(u)), SPD) and returns (lambda = dL/db, dL/dA on A's pattern or None, info)."""
    _check_vec(J, dLdu, vector_f64)
    lam = torch.empty_like(dLdu) if lam is None else lam
    if want_dA and A is not None and dLdA is None:
        dLdA = torch.empty(A.nnz, dtype=A.dtype, device=dLdu.device)
    elif not want_dA or A is None:
        dLdA = None
    info = _lib.sla_pcg_info()
    opts = _opts(rtol, maxit, vector_f64, engine)
    _check(lib().sla_nonlinear_adjoint(J.handle, _mh(M), None if A is None else A.handle, _ptr(u), _ptr(dLdu),
                                       _ptr(lam), _ptr(dLdA), C.byref(opts), C.byref(info), _stream(stream)),
           "sla_nonlinear_adjoint")
    return lam, dLdA, _info1(info)


def sla_vec_dot(x: torch.Tensor, y: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out[0] = x . y in fp64 (device tensor; no host synchronisation)."""
    out = torch.empty(1, dtype=torch.float64, device=x.device) if out is None else out
    _check(lib().sla_vec_dot(_dtype_code(x.dtype), x.numel(), _ptr(x), _ptr(y), _ptr(out), _stream(stream)),
           "sla_vec_dot")
    return out


def sla_pcg_update(alpha: float, p: torch.Tensor, q: torch.Tensor, x: torch.Tensor, r: torch.Tensor,
                   dinv: Optional[torch.Tensor], z: torch.Tensor, out2: Optional[torch.Tensor] = None,
                   n: Optional[int] = None, stream=None) -> torch.Tensor:
    """x += alpha p, r -= alpha q, z = dinv * r; returns the device tensor [r.r, r.z] (fp64).
    n: number of leading elements to update (default: all of r)."""
    out2 = torch.empty(2, dtype=torch.float64, device=r.device) if out2 is None else out2
    n = r.numel() if n is None else int(n)
    _check(lib().sla_pcg_update(_dtype_code(r.dtype), n, float(alpha), _ptr(p), _ptr(q), _ptr(x), _ptr(r),
                                _ptr(dinv), _ptr(z), _ptr(out2), _stream(stream)), "sla_pcg_update")
    return out2


def sla_pcg_direction(beta: float, z: torch.Tensor, p: torch.Tensor, n: Optional[int] = None, stream=None):
    """p = z + beta p on the leading n elements (default: all)."""
    n = p.numel() if n is None else int(n)
    _check(lib().sla_pcg_direction(_dtype_code(p.dtype), n, float(beta), _ptr(z), _ptr(p), _stream(stream)),
           "sla_pcg_direction")
    return p


def sla_vec_gather(idx: torch.Tensor, src: torch.Tensor, dst: torch.Tensor, stream=None) -> torch.Tensor:
    """dst[k] = src[idx[k]] (idx int32)."""
    if idx.dtype != torch.int32:
        raise ValueError("idx must be int32")
    _check(lib().sla_vec_gather(_dtype_code(src.dtype), idx.numel(), _ptr(idx), _ptr(src), _ptr(dst),
                                _stream(stream)), "sla_vec_gather")
    return dst


def sla_vec_scatter_add(idx: torch.Tensor, src: torch.Tensor, dst: torch.Tensor, stream=None) -> torch.Tensor:
    """dst[idx[k]] += src[k] (idx int32, distinct)."""
    if idx.dtype != torch.int32:
        raise ValueError("idx must be int32")
    _check(lib().sla_vec_scatter_add(_dtype_code(dst.dtype), idx.numel(), _ptr(idx), _ptr(src), _ptr(dst),
                                     _stream(stream)), "sla_vec_scatter_add")
    return dst


def sla_pcg_kernel_times(A: Matrix, M: Optional[Preconditioner] = None, nrhs: int = 1, reps: int = 20,
                         vector_f64: bool = False, stream=None) -> list[float]:
    """Mean ms per launch of the iteration's kernels: [q = A p, x/r update, z = G y + eps r]."""
    out = (C.c_double * 3)()
    _check(lib().sla_pcg_kernel_times(A.handle, _mh(M), nrhs, 1 if vector_f64 else 0, reps, out,
                                      _stream(stream)), "sla_pcg_kernel_times")
    return list(out)


def sla_pcg_phase_times(A: Matrix, M: Optional[Preconditioner] = None, nrhs: int = 1,
                        vector_f64: bool = False, stream=None) -> tuple[list[float], list[int]]:
    """In-kernel mean ms per phase of the last persistent-engine solve, and phase counts:
    [q = A p, x/r update + y = G^T r, z = G y + eps r, x/r update + z = D^-1 r]."""
    ms = (C.c_double * 4)()
    cnt = (C.c_int64 * 4)()
    _check(lib().sla_pcg_phase_times(A.handle, _mh(M), nrhs, 1 if vector_f64 else 0, ms, cnt,
                                     _stream(stream)), "sla_pcg_phase_times")
    return list(ms), [int(c) for c in cnt]


def sla_workspace_bytes(A: Matrix, M: Optional[Preconditioner] = None, nrhs: int = 1,
                        vector_f64: bool = False) -> int:
    return int(lib().sla_workspace_bytes(A.handle, _mh(M), nrhs, 1 if vector_f64 else 0))


class _Solve(torch.autograd.Function):
    @staticmethod
    def forward(ctx, val, b, A, M, rtol, maxit, vector_f64):
        x, info = sla_pcg_solve(A, M, b, rtol=rtol, maxit=maxit, vector_f64=vector_f64)
        if info.status == SLA_BREAKDOWN:
            raise SlaError(SLA_BREAKDOWN, "solve")
        ctx.A, ctx.M, ctx.rtol, ctx.maxit, ctx.vf64 = A, M, rtol, maxit, vector_f64
        ctx.info = info
        ctx.save_for_backward(x)
        return x

    @staticmethod
    def backward(ctx, gx):
        (x,) = ctx.saved_tensors
        need_A = ctx.needs_input_grad[0]
        dLdb, dLdA, info = sla_pcg_adjoint(ctx.A, ctx.M, x, gx.contiguous(), want_dA=need_A,
                                           rtol=ctx.rtol, maxit=ctx.maxit, vector_f64=ctx.vf64)
        if dLdA is not None:
            dLdA = dLdA.view(ctx.A.val.shape)       # BSR values are [nnzb, b, b]
        return dLdA, dLdb, None, None, None, None, None


def solve(A: Matrix, b: torch.Tensor, M: Optional[Preconditioner] = None, *, rtol: float = 0.0,
          maxit: int = 0, vector_f64: bool = False) -> torch.Tensor:
    """x = A^-1 b, differentiable in A's values (A.val) and in b.

    Gradients flow to ``A.val`` if it requires grad; the backward pass is one adjoint PCG
    solve and one pattern-gradient pass, independent of the forward iteration count.
    """
    return _Solve.apply(A.val, b, A, M, rtol, maxit, vector_f64)
