"""Parity at the full workload sizes, in the configuration bench.py times.

The oracle's iteration counts (fp64, and for fp32-vector workloads also its fp32-storage
mode) and its solution, adjoint and gradient at 131072 sampled values each come from
tests/golden/full_<cfg>.{json,npz} (written by tests/golden/make_golden.py, which calls
only the oracle; the sample positions are recomputed from its seeds here).  Properties that
hold at any size are checked on the whole vectors: the true residual b - A x (oracle SpMV
in fp64), the adjoint identity w.x = lambda.b, the gradient's homogeneity identity
sum_k A_k g_k = -L over every stored entry, and g_k = -lambda_row(k) x_col(k) for every k.
"""
import json
import os
import sys

import numpy as np
import pytest
import torch

import sla_workloads as W
from gpu_helpers import SOL_TOL, dev, host, iters_close, matrix, precond, rel, relmax

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))
import make_golden as MG  # noqa: E402  (sample positions only; no oracle call)


def _golden(cfg):
    path = os.path.join(HERE, "golden", f"full_{cfg}.json")
    npz = os.path.join(HERE, "golden", f"full_{cfg}.npz")
    if not (os.path.exists(path) and os.path.exists(npz)):
        pytest.skip(f"{path} not generated")
    with open(path) as f:
        gold = json.load(f)
    arr = np.load(npz)
    return gold, {k: arr[k] for k in arr.files}


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
    gold, arr = _golden(cfg)
    w = W.workload(cfg, "full")
    A = w.A
    assert A.nnz == gold["nnz"]
    Ad = matrix(A)
    M, _G = precond(w, Ad)
    x, lam, g, fi, ai = _solve(w, Ad, M, vf64)
    assert all(i.status == 0 for i in fi + ai)
    # iteration counts within 2 % of the oracle taking the stopping decision in the same
    # vector precision (fp32 vectors: the oracle's fp32-storage mode)
    pure32 = w.dtype == np.float32 and not vf64
    f_ref = gold["fwd_iters_f32"] if pure32 else gold["fwd_iters"]
    a_ref = gold["adj_iters_f32"] if pure32 else gold["adj_iters"]
    for got, ref in zip([i.iters for i in fi] + [i.iters for i in ai], f_ref + a_ref):
        assert iters_close(got, ref), (got, ref)
    tol = SOL_TOL[np.float64 if (vf64 or w.dtype == np.float64) else np.float32]
    tol = max(tol, 10 * w.tol) if vf64 else tol
    rows = MG.row_sample(w, cfg)
    ents = MG.entry_sample(w, cfg)
    assert rows.size == gold["n_rows_sampled"] and ents.size == gold["n_entries_sampled"]
    xh = host(x).reshape(A.n_rows, -1)
    lh = host(lam).reshape(A.n_rows, -1)
    gh = host(g).reshape(-1)
    for name, got, ref in (("x", xh[rows], arr["x"]), ("lam", lh[rows], arr["lam"]),
                           ("grad", gh[ents], arr["grad"])):
        assert rel(got, ref) <= tol, (name, rel(got, ref))
        assert relmax(got, ref) <= 10 * tol, (name, relmax(got, ref))
    assert abs(np.linalg.norm(xh) - gold["x_norm"]) <= tol * gold["x_norm"]
    # size-independent checks on the whole vectors
    B = w.B.astype(np.float64).reshape(A.n_rows, -1)
    Wt = w.W.astype(np.float64).reshape(A.n_rows, -1)
    tight = w.dtype == np.float64 or vf64
    L_tot, bound = 0.0, 0.0
    for c in range(B.shape[1]):
        r_true = B[:, c] - ora.spmv(A, xh[:, c])
        r_adj = Wt[:, c] - ora.spmv(A, lh[:, c])
        res = np.linalg.norm(r_true) / np.linalg.norm(B[:, c])
        assert res <= (10 * w.tol if tight else 5e-3), res
        L = float(Wt[:, c] @ xh[:, c])
        assert abs(float(lh[:, c] @ B[:, c]) - L) <= (1e-7 if tight else 1e-3) * max(1.0, abs(L))
        L_tot += L
        # A symmetric: sum_k A_k (-lambda_i x_j) + w.x = (w - A lambda).x
        bound += np.linalg.norm(xh[:, c]) * np.linalg.norm(r_adj)
    # over every stored entry, in fp64: sum_k A_k g_k = -L up to the adjoint residual and
    # the rounding of each g_k to A's type
    s_ag = float(A.val.astype(np.float64) @ gh)
    s_abs = float(np.abs(A.val.astype(np.float64)) @ np.abs(gh))
    rnd = (1e-13 if w.dtype == np.float64 else 1e-6) * s_abs
    assert abs(s_ag + L_tot) <= 1.01 * bound + rnd, (s_ag, -L_tot, bound, rnd)
    # every stored entry: g_k = -sum_c lambda_c,row(k) x_c,col(k), rounded once to A's type
    g2 = np.zeros(A.nnz, dtype=np.float64)
    rr = A.rows_of_entries()
    cc = A.col.astype(np.int64)
    for c in range(B.shape[1]):
        g2 -= lh[rr, c] * xh[cc, c]
    assert relmax(gh, g2) <= (4e-15 if w.dtype == np.float64 else 4e-7), relmax(gh, g2)
