"""Helpers for the GPU parity tests: move seeded workloads onto the device as libsla handles
and compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import differentiable_sparse_linear_b200 as sla

# Tolerances stated for the path: SpMV 1e-12 (fp64) / 1e-5 (fp32); solutions and
# gradients 1e-8 (fp64) / 1e-4 (fp32); iteration counts within 2 %.
SPMV_TOL = {np.float64: 1e-12, np.float32: 1e-5}
SOL_TOL = {np.float64: 1e-8, np.float32: 1e-4}


def tol_key(dtype):
    return np.float64 if np.dtype(dtype) == np.float64 else np.float32


def dev(a, dtype=None):
    """Host array -> CUDA tensor (optionally cast first)."""
    t = torch.from_numpy(np.ascontiguousarray(a if dtype is None else a.astype(dtype)))
    return t.cuda()


def matrix(A, validate=True):
    rp, ci, v = dev(A.row_ptr), dev(A.col), dev(A.val)
    if A.sys_row_off is not None:
        return sla.sla_csr_create_list(list(A.sys_row_off), rp, ci, v, validate=validate)
    return sla.sla_csr_create(rp, ci, v, validate=validate)


def precond(w, Ad):
    if w.precond == "jacobi":
        return sla.sla_precond_jacobi(Ad), None
    Gd = matrix(w.G)
    return sla.sla_precond_spai(Ad, Gd, w.eps), Gd


def rel(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    d = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (d if d > 0 else 1.0))


def relmax(a, b) -> float:
    """Largest element error relative to the largest reference element (catches a single
    wrong row that a 2-norm over millions of rows can hide)."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    if b.size == 0:
        return 0.0
    d = float(np.max(np.abs(b)))
    return float(np.max(np.abs(a - b)) / (d if d > 0 else 1.0))


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.float64)


def iters_close(a: int, b: int) -> bool:
    """Within 2 % of the oracle's count (so below 50 iterations: equal)."""
    return abs(a - b) <= 0.02 * b
