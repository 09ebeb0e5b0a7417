"""Eigenvalue gradient and nonlinear adjoint through the C ABI, against the oracle.

* sla_eigen_grad: Hellmann-Feynman d mu / dA_ij = v_i v_j on the pattern, for the closed-form
  eigenvectors of the 2D Poisson matrices (64^2 fp64 and 1024^2 fp32), one and two vectors;
  sum_k A_k g_k = mu checked on the GPU's output.
* sla_csr_add_diagonal + sla_nonlinear_adjoint: F(u) = A u + u^3 - b = 0 (u from a host
  Newton solve, an input here), J = A + diag(3 u^2) formed on the device, one adjoint PCG
  solve with J and the pattern product dL/dA = -lambda_i u_j.
"""
import numpy as np
import pytest
import scipy.sparse as sp
import scipy.sparse.linalg as spla
import torch

import sla_workloads as W
from gpu_helpers import SOL_TOL, dev, host, iters_close, rel, relmax

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ora():
    import oracle
    return oracle.get()


def _lap_vec(N, j):
    p = np.arange(1, N + 1)
    return np.sin(j * np.pi * p / (N + 1)), 2.0 - 2.0 * np.cos(j * np.pi / (N + 1))


def _poisson_eigvec(N, j, k):
    vj, lj = _lap_vec(N, j)
    vk, lk = _lap_vec(N, k)
    v = np.outer(vj, vk).ravel()
    return v / np.linalg.norm(v), lj + lk


@pytest.mark.parametrize("N,dtype", [(64, np.float64), (1024, np.float32), (13, np.float32)])
def test_eigen_grad_poisson(ora, N, dtype):
    import differentiable_sparse_linear_b200 as sla
    A = W.poisson2d(N, dtype)
    Ad = sla.sla_csr_create(dev(A.row_ptr), dev(A.col), dev(A.val))
    v1, mu1 = _poisson_eigvec(N, 1, 1)
    v2, mu2 = _poisson_eigvec(N, min(3, N), min(5, N))
    for V, mus in ((v1, [mu1]), (np.stack([v1, v2], axis=1), [mu1, mu2])):
        Vt = V.astype(dtype)
        g = host(sla.sla_eigen_grad(Ad, dev(Vt)))
        Vh = Vt.astype(np.float64).reshape(A.n_rows, -1)
        ref = sum(ora.eigen_grad(A, Vh[:, c]) for c in range(Vh.shape[1]))
        bound = 1e-15 if dtype == np.float64 else 1.2e-7
        assert relmax(g, ref) <= bound, relmax(g, ref)
        # homogeneity: sum_k A_k g_k = sum of the eigenvalues, up to the rounding of v and g
        # to the vector type (the sum cancels terms of size sum_k |A_k g_k|, so the bound
        # scales with that, not with the small eigenvalues)
        s = float(A.val.astype(np.float64) @ g)
        s_abs = float(np.abs(A.val.astype(np.float64)) @ np.abs(g))
        assert abs(s - sum(mus)) <= (1e-13 if dtype == np.float64 else 1e-6) * s_abs, (s, mus, s_abs)


def test_eigen_grad_bsr_order(ora):
    """A BSR handle gives the gradient in its value order (the oracle's scalar expansion
    maps back through the expansion positions)."""
    import differentiable_sparse_linear_b200 as sla
    Ab = W.elastic3d_bsr(5, 3, 0.1, np.float64)
    Ad = sla.sla_bsr_create(dev(Ab.row_ptr), dev(Ab.col), dev(Ab.val))
    rng = np.random.default_rng(5)
    v = rng.standard_normal(Ab.n_rows)
    v /= np.linalg.norm(v)
    g = host(sla.sla_eigen_grad(Ad, dev(v)))
    Ac, pos = ora.bsr_to_csr(Ab)
    ref = np.empty(pos.size)
    ref[pos] = ora.eigen_grad(Ac, v)
    assert relmax(g, ref) <= 1e-15


def _semilinear(A, b):
    """u with A u + u^3 = b (host Newton, sparse direct solves): an input of these tests."""
    As = sp.csr_matrix((A.val.astype(np.float64), A.col, A.row_ptr), shape=(A.n_rows, A.n_rows))
    u = spla.spsolve(As.tocsc(), b)
    for _ in range(30):
        F = As @ u + u ** 3 - b
        du = spla.spsolve((As + sp.diags(3 * u ** 2)).tocsc(), F)
        u = u - du
        if np.max(np.abs(du)) <= 1e-15 * max(1.0, np.max(np.abs(u))):
            break
    return u


@pytest.mark.parametrize("cfg,size", [(1, "full"), (1, "tiny"), (2, "small")])
def test_nonlinear_adjoint(ora, cfg, size):
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(cfg, size)
    A = w.A
    dt = w.dtype
    b = w.B.astype(np.float64) * 2.0
    u = _semilinear(A, b).astype(dt)
    rp, ci = dev(A.row_ptr), dev(A.col)
    Ad = sla.sla_csr_create(rp, ci, dev(A.val))
    uu = dev(u)
    c = dev((3.0 * u.astype(np.float64) ** 2).astype(dt))
    jval = torch.empty(A.nnz, dtype=Ad.dtype, device="cuda")
    sla.sla_csr_add_diagonal(Ad, c, jval)
    Jd = sla.sla_csr_create(rp, ci, jval)
    # J's values: one addition per diagonal entry, in A's type
    Jo = ora.add_diagonal(A, (3.0 * u.astype(np.float64) ** 2).astype(dt).astype(np.float64))
    assert relmax(host(jval), Jo.val.astype(dt)) == 0.0
    M = sla.sla_precond_jacobi(Jd)
    wl = dev(w.W)
    lam, g, info = sla.sla_nonlinear_adjoint(Jd, M, Ad, uu, wl, rtol=w.tol)
    torch.cuda.synchronize()
    assert info.status == 0
    # the oracle's own J, stored in A's type as the device stores it
    Jo.val = Jo.val.astype(dt).astype(np.float64)
    ref = ora.nonlinear_adjoint(Jo, A, u.astype(np.float64), w.W, precond="jacobi", tol=w.tol)
    assert ref.status == 0
    cnt = ref
    if dt == np.float32:           # fp32 vectors: the count is decided in fp32 storage on both sides
        cnt = ora.nonlinear_adjoint(Jo, A, u.astype(np.float64), w.W, precond="jacobi", tol=w.tol,
                                    store_f32=True)
    assert iters_close(info.iters, cnt.iters), (info.iters, cnt.iters, ref.iters)
    t = SOL_TOL[np.float64 if dt == np.float64 else np.float32]
    assert rel(host(lam), ref.lam) <= t
    assert rel(host(g), ref.grad) <= t
    assert relmax(host(g), ref.grad) <= 10 * t
    # the product is -lambda_i u_j of the GPU's own lambda, rounded once to A's type
    g2 = ora.grad(A, host(lam), u.astype(np.float64))
    assert relmax(host(g), g2) <= (4e-15 if dt == np.float64 else 4e-7)


def test_add_diagonal_rejects_missing_diagonal():
    import differentiable_sparse_linear_b200 as sla
    rp = torch.tensor([0, 1, 2], dtype=torch.int32, device="cuda")
    ci = torch.tensor([1, 0], dtype=torch.int32, device="cuda")
    v = torch.ones(2, dtype=torch.float64, device="cuda")
    Ad = sla.sla_csr_create(rp, ci, v)
    with pytest.raises(sla.SlaError) as e:
        sla.sla_csr_add_diagonal(Ad, torch.ones(2, dtype=torch.float64, device="cuda"))
    assert e.value.status == sla.SLA_ERR_INVALID_ARG
