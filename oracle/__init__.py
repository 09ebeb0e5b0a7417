"""fp64 CPU oracle for PCG, its preconditioners, the adjoint and the pattern gradient.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it; the CUDA library and its Python binding never import it.

The arithmetic lives in ``oracle.c`` (plain sequential fp64 C, built by ``build.py``);
this module marshals numpy arrays and loops over right-hand sides and systems for the
batched forms.  Inputs in fp32 are promoted to fp64 exactly before any arithmetic.

Sources: "torch-sla: Differentiable Sparse Linear Algebra with Adjoint Solvers and Sparse
Tensor Parallelism for PyTorch" (Methodology §1 Jacobi-preconditioned native iterative
backend; Methodology §2 Linear Systems adjoint; Methodology §1 SparseTensor /
SparseTensorList batches) and "Learning Sparse Approximate Inverse Preconditioners for
Conjugate Gradient Solvers on GPUs" (Approach: M^-1 = G G^T + eps I).
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import build as _build

CONVERGED, NOT_CONVERGED, BREAKDOWN = 0, 1, 2

_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")


class _Precond(C.Structure):
    _fields_ = [
        ("kind", C.c_int32), ("pad", C.c_int32), ("diag", C.c_void_p),
        ("g_rp", C.c_void_p), ("g_ci", C.c_void_p), ("g_v", C.c_void_p),
        ("gt_rp", C.c_void_p), ("gt_ci", C.c_void_p), ("gt_v", C.c_void_p),
        ("eps", C.c_double),
    ]


@dataclass
class SolveResult:
    x: np.ndarray
    iters: int
    relres: float
    status: int
    hist: Optional[np.ndarray] = None


@dataclass
class AdjointResult:
    lam: np.ndarray       # dL/db
    grad: np.ndarray      # dL/dA on A's pattern, aligned with A.val
    iters: int
    relres: float
    status: int


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


class Oracle:
    """Handle on one build of the oracle library (the default one, or a test's variant)."""

    def __init__(self, libpath: Optional[str] = None):
        self.libpath = libpath or _build.build()
        lib = C.CDLL(self.libpath)
        lib.ora_spmv.argtypes = [C.c_int64, _i32p, _i32p, _f64p, _f64p, _f64p]
        lib.ora_spmv.restype = None
        lib.ora_dot.argtypes = [C.c_int64, _f64p, _f64p]
        lib.ora_dot.restype = C.c_double
        lib.ora_transpose.argtypes = [C.c_int64, C.c_int64, _i32p, _i32p, _f64p, _i32p, _i32p, _f64p]
        lib.ora_transpose.restype = C.c_int
        lib.ora_diagonal.argtypes = [C.c_int64, _i32p, _i32p, _f64p, _f64p]
        lib.ora_diagonal.restype = C.c_int
        lib.ora_precond_apply.argtypes = [C.c_int64, C.POINTER(_Precond), _f64p, _f64p, _f64p]
        lib.ora_precond_apply.restype = None
        lib.ora_pcg.argtypes = [C.c_int64, _i32p, _i32p, _f64p, C.POINTER(_Precond), _f64p, _f64p,
                                C.c_double, C.c_int64, C.c_int64, C.POINTER(C.c_int64),
                                C.POINTER(C.c_double), C.c_void_p]
        lib.ora_pcg.restype = C.c_int
        lib.ora_pcg_ex.argtypes = [C.c_int64, _i32p, _i32p, _f64p, C.POINTER(_Precond), _f64p, _f64p,
                                   C.c_double, C.c_int64, C.c_int64, C.c_int32, C.POINTER(C.c_int64),
                                   C.POINTER(C.c_double), C.c_void_p]
        lib.ora_pcg_ex.restype = C.c_int
        lib.ora_pattern_grad.argtypes = [C.c_int64, _i32p, _i32p, _f64p, _f64p, _f64p]
        lib.ora_pattern_grad.restype = None
        lib.ora_eigen_grad.argtypes = [C.c_int64, _i32p, _i32p, _f64p, _f64p]
        lib.ora_eigen_grad.restype = None
        lib.ora_add_diagonal.argtypes = [C.c_int64, _i32p, _i32p, _f64p, _f64p, _f64p]
        lib.ora_add_diagonal.restype = C.c_int
        lib.ora_bsr_spmv.argtypes = [C.c_int64, C.c_int32, _i32p, _i32p, _f64p, _f64p, _f64p]
        lib.ora_bsr_spmv.restype = None
        lib.ora_bsr_to_csr.argtypes = [C.c_int64, C.c_int32, _i32p, _i32p, _f64p, _i32p, _i32p, _f64p,
                                       np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")]
        lib.ora_bsr_to_csr.restype = None
        self.lib = lib

    # ---------------------------------------------------------------- basic operations
    def spmv(self, A, x) -> np.ndarray:
        """y = A x in fp64."""
        x = _f64(x)
        y = np.empty(A.n_rows, dtype=np.float64)
        self.lib.ora_spmv(A.n_rows, _i32(A.row_ptr), _i32(A.col), _f64(A.val), x, y)
        return y

    def dot(self, a, b) -> float:
        a, b = _f64(a), _f64(b)
        return float(self.lib.ora_dot(a.size, a, b))

    def transpose(self, A):
        """CSR of A^T (same class as A, fp64 values)."""
        rpT = np.empty(A.n_cols + 1, dtype=np.int32)
        ciT = np.empty(A.nnz, dtype=np.int32)
        vT = np.empty(A.nnz, dtype=np.float64)
        rc = self.lib.ora_transpose(A.n_rows, A.n_cols, _i32(A.row_ptr), _i32(A.col), _f64(A.val),
                                    rpT, ciT, vT)
        if rc != 0:
            raise MemoryError("oracle transpose")
        return type(A)(A.n_cols, A.n_rows, rpT, ciT, vT)

    def diagonal(self, A) -> np.ndarray:
        d = np.empty(A.n_rows, dtype=np.float64)
        if self.lib.ora_diagonal(A.n_rows, _i32(A.row_ptr), _i32(A.col), _f64(A.val), d) != 0:
            raise ValueError("a row stores no diagonal entry")
        return d

    def grad(self, A, lam, x) -> np.ndarray:
        """dL/dA_ij = -lam_i x_j on A's stored entries."""
        g = np.empty(A.nnz, dtype=np.float64)
        self.lib.ora_pattern_grad(A.n_rows, _i32(A.row_ptr), _i32(A.col), _f64(lam), _f64(x), g)
        return g

    def eigen_grad(self, A, v) -> np.ndarray:
        """d mu / dA_ij = v_i v_j on A's stored entries (v a unit eigenvector of symmetric A)."""
        g = np.empty(A.nnz, dtype=np.float64)
        self.lib.ora_eigen_grad(A.n_rows, _i32(A.row_ptr), _i32(A.col), _f64(v), g)
        return g

    def add_diagonal(self, A, c):
        """A + diag(c) on A's pattern (same class as A, fp64 values)."""
        out = np.empty(A.nnz, dtype=np.float64)
        if self.lib.ora_add_diagonal(A.n_rows, _i32(A.row_ptr), _i32(A.col), _f64(A.val), _f64(c), out) != 0:
            raise ValueError("a row stores no diagonal entry")
        return type(A)(A.n_rows, A.n_cols, _i32(A.row_ptr), _i32(A.col), out)

    # ---------------------------------------------------------------- preconditioners
    def _precond(self, A, kind: str, G=None, eps: float = 0.0):
        keep = []
        P = _Precond()
        if kind == "none":
            P.kind = 0
        elif kind == "jacobi":
            P.kind = 1
            d = self.diagonal(A)
            keep.append(d)
            P.diag = d.ctypes.data
        elif kind == "spai":
            if G is None:
                raise ValueError("SPAI needs G")
            P.kind = 2
            g_rp, g_ci, g_v = _i32(G.row_ptr), _i32(G.col), _f64(G.val)
            Gt = self.transpose(G)
            keep += [g_rp, g_ci, g_v, Gt.row_ptr, Gt.col, Gt.val]
            P.g_rp, P.g_ci, P.g_v = g_rp.ctypes.data, g_ci.ctypes.data, g_v.ctypes.data
            P.gt_rp, P.gt_ci, P.gt_v = Gt.row_ptr.ctypes.data, Gt.col.ctypes.data, Gt.val.ctypes.data
            P.eps = float(eps)
        else:
            raise ValueError(kind)
        return P, keep

    def precond_apply(self, A, r, kind: str, G=None, eps: float = 0.0) -> np.ndarray:
        P, keep = self._precond(A, kind, G, eps)
        r = _f64(r)
        z = np.empty_like(r)
        w = np.empty_like(r)
        self.lib.ora_precond_apply(r.size, C.byref(P), r, z, w)
        return z

    # ---------------------------------------------------------------- solves
    def pcg(self, A, b, precond: str = "jacobi", G=None, eps: float = 0.0, tol: float = 1e-10,
            maxit: Optional[int] = None, fixed_iters: int = 0, history: bool = False,
            store_f32: bool = False, _P=None) -> SolveResult:
        """PCG from x0 = 0; maxit defaults to 10 * n.

        store_f32: the same recurrence with every vector it keeps rounded to binary32 when
        formed (fp64 dot products and scalars) -- the arithmetic of fp32 vector storage, for
        comparing iteration counts with a solver that stores its vectors in fp32."""
        n = A.n_rows
        maxit = 10 * max(n, 1) if maxit is None else int(maxit)
        P, keep = _P if _P is not None else self._precond(A, precond, G, eps)
        b = _f64(b)
        x = np.empty(n, dtype=np.float64)
        it = C.c_int64(0)
        rel = C.c_double(0.0)
        hlen = (fixed_iters if fixed_iters > 0 else maxit) + 1
        hist = np.zeros(hlen, dtype=np.float64) if history else None
        st = self.lib.ora_pcg_ex(n, _i32(A.row_ptr), _i32(A.col), _f64(A.val), C.byref(P), b, x,
                                 float(tol), maxit, int(fixed_iters), 1 if store_f32 else 0,
                                 C.byref(it), C.byref(rel), hist.ctypes.data if history else None)
        if history:
            hist = hist[: it.value + 1]
        return SolveResult(x, int(it.value), float(rel.value), int(st), hist)

    def adjoint(self, A, x, w, precond: str = "jacobi", G=None, eps: float = 0.0,
                tol: float = 1e-10, maxit: Optional[int] = None, store_f32: bool = False) -> AdjointResult:
        """Solve A^T lam = w (w = dL/dx) by PCG; return dL/db = lam and dL/dA on the pattern.

        The transpose is formed explicitly, as the definition states it; M is the same
        preconditioner as the forward solve (for SPD A, A^T = A and M is unchanged).
        """
        At = self.transpose(A)
        P, keep = self._precond(A, precond, G, eps)
        res = self.pcg(At, w, tol=tol, maxit=maxit, store_f32=store_f32, _P=(P, keep))
        g = self.grad(A, res.x, x)
        return AdjointResult(res.x, g, res.iters, res.relres, res.status)

    def nonlinear_adjoint(self, J, A, u, dLdu, precond: str = "jacobi", G=None, eps: float = 0.0,
                          tol: float = 1e-10, maxit: Optional[int] = None, store_f32: bool = False):
        """Backward pass of F(u) = A u + N(u) - b = 0 at its solution u ([TS] Methodology §2,
        Nonlinear Systems): lambda solves J^T lambda = dL/du with the Jacobian J = dF/du
        (PCG on the explicit transpose, preconditioner built on J), then the vector-Jacobian
        product dL/dA_ij = -lambda_i u_j (A's values are parameters) and dL/db = lambda.
        Returns AdjointResult(lam, grad on A's pattern, ...)."""
        Jt = self.transpose(J)
        P, keep = self._precond(J, precond, G, eps)
        res = self.pcg(Jt, dLdu, tol=tol, maxit=maxit, store_f32=store_f32, _P=(P, keep))
        g = self.grad(A, res.x, u)
        return AdjointResult(res.x, g, res.iters, res.relres, res.status)

    # ---------------------------------------------------------------- batches
    def pcg_multi(self, A, B, **kw):
        """Shared-pattern batch: one independent PCG per column of B ([n][k] layout)."""
        B = np.asarray(B)
        k = B.shape[1]
        X = np.empty((A.n_rows, k), dtype=np.float64)
        out = []
        for c in range(k):
            r = self.pcg(A, B[:, c], **kw)
            X[:, c] = r.x
            out.append(r)
        return X, out

    def adjoint_multi(self, A, X, W, **kw):
        """Shared-pattern batched adjoint: Lam[:, c] per RHS, gradient summed over RHS."""
        k = X.shape[1]
        Lam = np.empty((A.n_rows, k), dtype=np.float64)
        g = np.zeros(A.nnz, dtype=np.float64)
        out = []
        for c in range(k):
            r = self.adjoint(A, X[:, c], W[:, c], **kw)
            Lam[:, c] = r.lam
            g = g + r.grad
            out.append(r)
        return Lam, g, out

    # ---------------------------------------------------------------- block sparse rows
    def bsr_spmv(self, A, x) -> np.ndarray:
        """y = A x for a BSR matrix (``A.val`` is [nnzb, b, b]) in fp64."""
        x = _f64(x)
        y = np.empty(A.n_rows, dtype=np.float64)
        self.lib.ora_bsr_spmv(A.n_brows, A.b, _i32(A.row_ptr), _i32(A.col), _f64(A.val).reshape(-1), x, y)
        return y

    def bsr_to_csr(self, A):
        """(scalar CSR of the BSR matrix A with fp64 values, BSR value position of each entry)."""
        from sla_workloads import CSR
        nnz = A.nnzb * A.b * A.b
        rp = np.empty(A.n_rows + 1, dtype=np.int32)
        ci = np.empty(nnz, dtype=np.int32)
        v = np.empty(nnz, dtype=np.float64)
        pos = np.empty(nnz, dtype=np.int64)
        self.lib.ora_bsr_to_csr(A.n_brows, A.b, _i32(A.row_ptr), _i32(A.col), _f64(A.val).reshape(-1),
                                rp, ci, v, pos)
        return CSR(A.n_rows, A.n_rows, rp, ci, v), pos

    def pcg_bsr(self, A, b, **kw) -> SolveResult:
        """PCG on a BSR matrix: the same iteration on its scalar CSR form."""
        return self.pcg(self.bsr_to_csr(A)[0], b, **kw)

    def adjoint_bsr(self, A, x, w, **kw) -> AdjointResult:
        """Adjoint on a BSR matrix; the gradient comes back in BSR value order ([nnzb, b, b])."""
        Ac, pos = self.bsr_to_csr(A)
        r = self.adjoint(Ac, x, w, **kw)
        g = np.empty(pos.size, dtype=np.float64)
        g[pos] = r.grad
        r.grad = g.reshape(A.nnzb, A.b, A.b)
        return r

    @staticmethod
    def system(A, s: int, sys_row_off=None):
        """System s of a block-diagonal list as its own CSR (local column indices).  A matrix
        without its own offsets (a list's SPAI factor) takes the list's `sys_row_off`."""
        off = A.sys_row_off if sys_row_off is None else sys_row_off
        o0, o1 = int(off[s]), int(off[s + 1])
        k0, k1 = int(A.row_ptr[o0]), int(A.row_ptr[o1])
        rp = (A.row_ptr[o0:o1 + 1].astype(np.int64) - k0).astype(np.int32)
        ci = (A.col[k0:k1].astype(np.int64) - o0).astype(np.int32)
        return type(A)(o1 - o0, o1 - o0, rp, ci, np.asarray(A.val[k0:k1]))

    def _system_kw(self, A, s, kw):
        """The solver options for system s: a list's SPAI factor G cut to the system's block."""
        if kw.get("G") is not None:
            kw = dict(kw)
            kw["G"] = self.system(kw["G"], s, A.sys_row_off)
        return kw

    def pcg_list(self, A, b, **kw):
        """Distinct-pattern batch: one PCG per diagonal block; b and x concatenated."""
        x = np.empty(A.n_rows, dtype=np.float64)
        out = []
        for s in range(A.batch):
            o0, o1 = int(A.sys_row_off[s]), int(A.sys_row_off[s + 1])
            r = self.pcg(self.system(A, s), np.asarray(b)[o0:o1], **self._system_kw(A, s, kw))
            x[o0:o1] = r.x
            out.append(r)
        return x, out

    def adjoint_list(self, A, x, w, **kw):
        """Per-system adjoint of a list batch; the gradient is per system, concatenated."""
        lam = np.empty(A.n_rows, dtype=np.float64)
        g = np.empty(A.nnz, dtype=np.float64)
        out = []
        for s in range(A.batch):
            o0, o1 = int(A.sys_row_off[s]), int(A.sys_row_off[s + 1])
            k0, k1 = int(A.row_ptr[o0]), int(A.row_ptr[o1])
            r = self.adjoint(self.system(A, s), np.asarray(x)[o0:o1], np.asarray(w)[o0:o1],
                             **self._system_kw(A, s, kw))
            lam[o0:o1] = r.lam
            g[k0:k1] = r.grad
            out.append(r)
        return lam, g, out


_default: Optional[Oracle] = None


def get() -> Oracle:
    """The oracle built from this directory's oracle.c (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


_omp: Optional[Oracle] = None


def get_omp() -> Oracle:
    """The same source built with OpenMP: independent row / element loops on every host
    core, dot products sequential, results bit-identical to get()'s.  Only the benchmark's
    CPU baseline uses it."""
    global _omp
    if _omp is None:
        _omp = Oracle(_build.build_omp())
    return _omp
