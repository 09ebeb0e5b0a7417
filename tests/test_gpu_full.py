"""Parity at the full workload sizes, in the configuration bench.py times.

The oracle's iteration counts and its solution, adjoint and gradient at sampled indices
come from tests/golden/full_<cfg>.json (written by tests/golden/make_golden.py, which calls
only the oracle).  Properties that hold at any size are checked on the whole vectors: the
true residual b - A x (oracle SpMV in fp64) and the adjoint identity w.x = lambda.b.
"""
import json
import os

import numpy as np
import pytest
import torch

import sla_workloads as W
from gpu_helpers import SOL_TOL, dev, host, iters_close, matrix, precond, rel

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden(cfg):
    path = os.path.join(HERE, "golden", f"full_{cfg}.json")
    if not os.path.exists(path):
        pytest.skip(f"{path} not generated")
    with open(path) as f:
        return json.load(f)


@pytest.fixture(scope="module")
def ora():
    import oracle
    return oracle.get()


def _solve(w, Ad, M, vf64):
    import differentiable_sparse_linear_b200 as sla
    vt = np.float64 if vf64 else w.dtype
    b, wl = dev(w.B, vt), dev(w.W, vt)
    if w.A.sys_row_off is not None or w.nrhs > 1:
        x, fi = sla.sla_pcg_solve_batched(Ad, M, b, rtol=w.tol, vector_f64=vf64)
        lam, g, ai = sla.sla_pcg_adjoint_batched(Ad, M, x, wl, rtol=w.tol, vector_f64=vf64)
    else:
        x, f1 = sla.sla_pcg_solve(Ad, M, b, rtol=w.tol, vector_f64=vf64)
        lam, g, a1 = sla.sla_pcg_adjoint(Ad, M, x, wl, rtol=w.tol, vector_f64=vf64)
        fi, ai = [f1], [a1]
    torch.cuda.synchronize()
    return x, lam, g, fi, ai


CASES = [(1, False), (2, False), (3, False), (4, False), (5, False), (5, True)]


@pytest.mark.parametrize("cfg,vf64", CASES)
def test_full_size_parity(ora, cfg, vf64):
    gold = _golden(cfg)
    w = W.workload(cfg, "full")
    assert w.A.nnz == gold["nnz"]
    Ad = matrix(w.A)
    M, _G = precond(w, Ad)
    x, lam, g, fi, ai = _solve(w, Ad, M, vf64)
    assert all(i.status == 0 for i in fi + ai)
    # iteration counts: within 2 % (pure-fp32 vectors on the power-law SPAI system: 5 %,
    # the delay fp32 storage of the Krylov vectors causes there)
    loose = cfg == 5 and not vf64
    for got, ref in zip([i.iters for i in fi] + [i.iters for i in ai], gold["fwd_iters"] + gold["adj_iters"]):
        ok = abs(got - ref) <= max(1, 0.05 * ref) if loose else iters_close(got, ref)
        assert ok, (got, ref)
    tol = SOL_TOL[np.float64 if (vf64 or w.dtype == np.float64) else np.float32]
    tol = max(tol, 10 * w.tol) if vf64 else tol
    rows, ents = gold["rows"], gold["entries"]
    xs = host(x).reshape(w.A.n_rows, -1)[rows]
    ls = host(lam).reshape(w.A.n_rows, -1)[rows]
    assert rel(xs, np.asarray(gold["x"])) <= tol
    assert rel(ls, np.asarray(gold["lam"])) <= tol
    assert rel(host(g)[ents], np.asarray(gold["grad"])) <= tol
    assert abs(np.linalg.norm(host(x)) - gold["x_norm"]) <= tol * gold["x_norm"]
    # size-independent checks on the whole vectors
    xb = host(x).reshape(w.A.n_rows, -1)
    lb = host(lam).reshape(w.A.n_rows, -1)
    B = w.B.astype(np.float64).reshape(w.A.n_rows, -1)
    Wt = w.W.astype(np.float64).reshape(w.A.n_rows, -1)
    for c in range(B.shape[1]):
        res = np.linalg.norm(B[:, c] - ora.spmv(w.A, xb[:, c])) / np.linalg.norm(B[:, c])
        assert res <= (10 * w.tol if (w.dtype == np.float64 or vf64) else 5e-3), res
        L = float(Wt[:, c] @ xb[:, c])
        assert abs(float(lb[:, c] @ B[:, c]) - L) <= (1e-7 if (w.dtype == np.float64 or vf64) else 1e-3) * max(1.0, abs(L))
