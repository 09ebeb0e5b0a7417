"""The inverse-coefficient demo (examples/inverse_conductivity.py) as an end-to-end user of
the differentiable solve: the Adam loop drives the loss and the conductivity error down,
and one gradient dL/dtheta through libsla's solve and adjoint matches the oracle's adjoint
chained through the same assembly map."""
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.join(ROOT, "examples"))
import inverse_conductivity as IC  # noqa: E402

pytestmark = pytest.mark.gpu


def test_adam_loop_recovers_conductivity():
    r = IC.run(N=24, steps=150, lr=0.05)
    assert r["loss"] <= r["loss0"] / 50, (r["loss0"], r["loss"])
    assert r["kappa_err"] <= 0.25 * r["kappa_err0"], (r["kappa_err0"], r["kappa_err"])


def test_gradient_matches_oracle_adjoint():
    import oracle
    ora = oracle.get()
    N = 20
    pb = IC.Problem(N)
    A, ent, node, wt = IC.assembly_terms(N)
    rng = np.random.default_rng(7)
    theta0 = rng.normal(0.0, 0.3, N * N)
    k_true = IC.true_kappa(N)
    # GPU: loss and gradient through the library
    with torch.no_grad():
        U = pb.solve_all(torch.from_numpy(k_true).cuda())
    theta = torch.from_numpy(theta0.copy()).cuda().requires_grad_(True)
    u = pb.solve_all(torch.exp(theta))
    loss = ((u - U) ** 2).sum()
    loss.backward()
    g_gpu = theta.grad.detach().cpu().numpy()
    # oracle: the same loss, adjoint solves, chained through the assembly map on the host
    F = IC.sources(N)

    def vals(k):
        v = np.zeros(A.nnz)
        np.add.at(v, ent, wt * k[node])
        return v

    At = IC.W.CSR(A.n_rows, A.n_cols, A.row_ptr, A.col, vals(k_true))
    Uo = np.stack([ora.pcg(At, F[s], precond="jacobi", tol=1e-12).x for s in range(F.shape[0])])
    k = np.exp(theta0)
    Ak = IC.W.CSR(A.n_rows, A.n_cols, A.row_ptr, A.col, vals(k))
    dv = np.zeros(A.nnz)
    for s in range(F.shape[0]):
        x = ora.pcg(Ak, F[s], precond="jacobi", tol=1e-12).x
        adj = ora.adjoint(Ak, x, 2.0 * (x - Uo[s]), precond="jacobi", tol=1e-12)
        dv += adj.grad
    dk = np.zeros(N * N)
    np.add.at(dk, node, wt * dv[ent])
    g_ora = dk * k
    assert np.linalg.norm(g_gpu - g_ora) / np.linalg.norm(g_ora) <= 1e-6
