"""Inverse coefficient learning: recover a spatially varying conductivity from solutions of
a Poisson equation, with an Adam loop through the differentiable solve.

The application of "torch-sla: Differentiable Sparse Linear Algebra with Adjoint Solvers and
Sparse Tensor Parallelism for PyTorch" (Experimental Results, end-to-end application:
conductivity in a Poisson equation recovered with a standard PyTorch Adam loop, reported at
0.23% relative L2 error).  Here, on synthetic data:

  -div(kappa grad u) = f on the unit square, u = 0 on the boundary, a 5-point finite-volume
  discretisation on an N x N grid of nodes: edge conductivity = mean of its two nodes'
  values (a boundary edge takes its node's value); A(kappa) is SPD for kappa > 0 with the
  2D Poisson pattern, and its values are linear in kappa.

kappa = exp(theta) is learned from S observed solutions u*_s = A(kappa*)^-1 f_s.  Each Adam
step solves A(kappa) u_s = f_s with libsla's PCG through `solve` (autograd: the backward
pass is one adjoint PCG solve and the pattern gradient per source); the assembly
theta -> A's values is ordinary torch code on the GPU (the user's model).

    python examples/inverse_conductivity.py [--N 64] [--steps 400]
"""
from __future__ import annotations

import argparse
import os
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import differentiable_sparse_linear_b200 as sla  # noqa: E402
import sla_workloads as W  # noqa: E402


def assembly_terms(N: int):
    """A's 5-point pattern and the linear map kappa -> values as terms (entry, node, weight):
    values[entry] = sum of weight * kappa[node] over the entry's terms."""
    A = W.poisson2d(N, np.float64)
    n = N * N
    rows = A.rows_of_entries()
    cols = A.col.astype(np.int64)
    ent, node, wt = [], [], []
    off = np.nonzero(rows != cols)[0]
    for e in off:                                   # -(kappa_p + kappa_q) / 2
        ent += [e, e]
        node += [rows[e], cols[e]]
        wt += [-0.5, -0.5]
    diag = np.nonzero(rows == cols)[0]
    for e in diag:
        p = rows[e]
        i, j = divmod(p, N)
        for di, dj in ((-1, 0), (1, 0), (0, -1), (0, 1)):
            ii, jj = i + di, j + dj
            if 0 <= ii < N and 0 <= jj < N:           # interior edge: (kappa_p + kappa_q) / 2
                ent += [e, e]
                node += [p, ii * N + jj]
                wt += [0.5, 0.5]
            else:                                     # boundary edge: kappa_p
                ent += [e]
                node += [p]
                wt += [1.0]
    return A, np.array(ent, np.int64), np.array(node, np.int64), np.array(wt, np.float64)


def true_kappa(N: int) -> np.ndarray:
    x = (np.arange(N) + 1) / (N + 1)
    X, Y = np.meshgrid(x, x, indexing="ij")
    k = 1.0 + 0.8 * np.exp(-((X - 0.35) ** 2 + (Y - 0.6) ** 2) / 0.02) + 0.3 * np.sin(2 * np.pi * X) * np.sin(np.pi * Y)
    return k.ravel()


def sources(N: int, S: int = 4) -> np.ndarray:
    x = (np.arange(N) + 1) / (N + 1)
    X, Y = np.meshgrid(x, x, indexing="ij")
    h2 = 1.0 / (N + 1) ** 2
    fs = [np.ones_like(X), np.sin(np.pi * X) * np.sin(2 * np.pi * Y), np.cos(np.pi * X) + 0.5,
          np.exp(-((X - 0.7) ** 2 + (Y - 0.3) ** 2) / 0.01)]
    return np.stack([h2 * f.ravel() for f in fs[:S]])


class Problem:
    def __init__(self, N: int, device="cuda"):
        A, ent, node, wt = assembly_terms(N)
        self.N, self.n, self.A_host = N, N * N, A
        self.dev = torch.device(device)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(self.dev)
        self.rp, self.ci = t(A.row_ptr), t(A.col)
        self.ent, self.node, self.wt = t(ent), t(node), t(wt)
        self.nnz = A.nnz
        self.val = torch.zeros(self.nnz, dtype=torch.float64, device=self.dev)
        self.mat = sla.sla_csr_create(self.rp, self.ci, self.val)     # values filled per step
        self.M = None
        self.F = t(sources(N))

    def values(self, kappa: torch.Tensor) -> torch.Tensor:
        return torch.zeros(self.nnz, dtype=kappa.dtype, device=self.dev).index_add(0, self.ent, self.wt * kappa[self.node])

    def solve_all(self, kappa: torch.Tensor, rtol: float = 1e-10) -> torch.Tensor:
        """u_s = A(kappa)^-1 f_s for every source, differentiable in kappa."""
        v = self.values(kappa)
        self.val.copy_(v.detach())                   # the handle's value array (borrowed by libsla)
        if self.M is None:
            self.M = sla.sla_precond_jacobi(self.mat)
        else:
            self.M.refresh()
        out = []
        for s in range(self.F.shape[0]):
            out.append(_SolveWithValues.apply(v, self.F[s], self.mat, self.M, rtol))
        return torch.stack(out)


class _SolveWithValues(torch.autograd.Function):
    """solve() with the values coming from the autograd graph of the caller's model."""

    @staticmethod
    def forward(ctx, v, f, mat, M, rtol):
        x, info = sla.sla_pcg_solve(mat, M, f, rtol=rtol)
        if info.status != 0:
            raise RuntimeError(f"solve: {info}")
        ctx.mat, ctx.M, ctx.rtol = mat, M, rtol
        ctx.save_for_backward(x)
        return x

    @staticmethod
    def backward(ctx, gx):
        (x,) = ctx.saved_tensors
        dLdb, dLdA, _ = sla.sla_pcg_adjoint(ctx.mat, ctx.M, x, gx.contiguous(), rtol=ctx.rtol)
        return dLdA, dLdb, None, None, None


def run(N: int = 64, steps: int = 400, lr: float = 0.05, reg: float = 1e-6, device="cuda", log=None):
    pb = Problem(N, device)
    k_true = torch.from_numpy(true_kappa(N)).to(pb.dev)
    with torch.no_grad():
        U = pb.solve_all(k_true)
    theta = torch.zeros(pb.n, dtype=torch.float64, device=pb.dev, requires_grad=True)
    opt = torch.optim.Adam([theta], lr=lr)
    # smoothness penalty on theta over the grid's edges (the data do not fix kappa at the
    # boundary-adjacent nodes tightly)
    Th = torch.arange(pb.n, device=pb.dev).reshape(N, N)
    e_a = torch.cat([Th[:-1, :].reshape(-1), Th[:, :-1].reshape(-1)])
    e_b = torch.cat([Th[1:, :].reshape(-1), Th[:, 1:].reshape(-1)])
    scale = float((U ** 2).sum())
    hist = []
    t0 = time.time()
    for it in range(steps):
        opt.zero_grad()
        u = pb.solve_all(torch.exp(theta))
        data = ((u - U) ** 2).sum() / scale
        loss = data + reg * ((theta[e_a] - theta[e_b]) ** 2).sum()
        loss.backward()
        opt.step()
        with torch.no_grad():
            err = float(torch.linalg.norm(torch.exp(theta) - k_true) / torch.linalg.norm(k_true))
        hist.append((float(loss), err))
        if log and (it % 50 == 0 or it == steps - 1):
            log(f"step {it:4d}  loss {float(loss):.3e}  kappa rel L2 error {err:.4%}")
    return {"N": N, "steps": steps, "seconds": time.time() - t0, "loss0": hist[0][0], "loss": hist[-1][0],
            "kappa_err0": hist[0][1], "kappa_err": hist[-1][1], "history": hist, "theta": theta.detach()}


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--N", type=int, default=64)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--lr", type=float, default=0.05)
    a = ap.parse_args()
    r = run(a.N, a.steps, a.lr, log=print)
    print(f"N={r['N']} steps={r['steps']} in {r['seconds']:.1f} s: loss {r['loss0']:.3e} -> {r['loss']:.3e}, "
          f"kappa relative L2 error {r['kappa_err0']:.3%} -> {r['kappa_err']:.3%}")
