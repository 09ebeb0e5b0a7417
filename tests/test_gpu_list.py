"""Lists of independent systems (SparseTensorList batches): the SPAI preconditioner with a
block-diagonal factor, systems too large for shared memory (vectors in a workspace), and
the checks that guard them -- against the oracle solving each system on its own."""
import numpy as np
import pytest
import torch

import sla_workloads as W
from gpu_helpers import SOL_TOL, dev, host, iters_close, matrix, rel, relmax

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ora():
    import oracle
    return oracle.get()


def _list(nsys, n, dtype, seed):
    A = W.random_spd_list(nsys, n, seed=seed, dtype=dtype)
    A.sys_row_off = np.asarray(A.sys_row_off)
    rng = np.random.default_rng(seed + 1)
    b = rng.uniform(-1, 1, A.n_rows).astype(dtype)
    w = rng.uniform(-1, 1, A.n_rows).astype(dtype)
    return A, b, w


@pytest.mark.parametrize("nsys,n,dtype,precond", [
    (24, 512, np.float64, "spai"), (7, 1024, np.float32, "spai"),        # shared memory
    (5, 6000, np.float64, "jacobi"), (5, 6000, np.float64, "spai"),      # workspace (fp64)
    (4, 7000, np.float32, "jacobi"), (3, 9000, np.float32, "none"),      # workspace (fp32)
])
def test_list_solve_adjoint(ora, nsys, n, dtype, precond):
    import differentiable_sparse_linear_b200 as sla
    A, b, w = _list(nsys, n, dtype, 60 + n % 97)
    Ad = matrix(A)
    G = None
    if precond == "spai":
        G = W.spai_factor_G(A, seed=61)
        M = sla.sla_precond_spai(Ad, matrix(G), 3e-3)
    elif precond == "jacobi":
        M = sla.sla_precond_jacobi(Ad)
    else:
        M = None
    tol = 1e-10 if dtype == np.float64 else 1e-6
    kw = dict(precond=precond, G=G, eps=3e-3, tol=tol)
    X, infos = sla.sla_pcg_solve_batched(Ad, M, dev(b), rtol=tol)
    xo, outs = ora.pcg_list(A, b, **kw)
    f32 = dtype == np.float32
    _, c32 = ora.pcg_list(A, b, store_f32=True, **kw) if f32 else (None, outs)
    for i, o, c in zip(infos, outs, c32):
        assert i.status == 0 and o.status == 0 and i.engine == "list"
        assert iters_close(i.iters, c.iters), (i.iters, c.iters, o.iters)
    t = SOL_TOL[dtype]
    assert rel(host(X), xo) <= t and relmax(host(X), xo) <= 10 * t
    Lam, g, ainf = sla.sla_pcg_adjoint_batched(Ad, M, X, dev(w), rtol=tol)
    lo, go, aouts = ora.adjoint_list(A, xo, w, **kw)
    assert all(a.status == 0 for a in ainf)
    assert rel(host(Lam), lo) <= t and rel(host(g), go) <= t


def test_list_spai_factor_must_be_block_diagonal():
    import differentiable_sparse_linear_b200 as sla
    A, b, _ = _list(3, 64, np.float64, 70)
    Ad = matrix(A)
    n = A.n_rows
    # a lower-triangular factor reaching across the first two systems
    rp = np.concatenate([[0], np.cumsum(np.where(np.arange(n) == 70, 2, 1))]).astype(np.int32)
    col = []
    for i in range(n):
        if i == 70:
            col += [3, 70]
        else:
            col.append(i)
    G = W.CSR(n, n, rp, np.asarray(col, np.int32), np.ones(len(col)))
    with pytest.raises(sla.SlaError) as e:
        sla.sla_precond_spai(Ad, matrix(G), 3e-3)
    assert e.value.status == sla.SLA_ERR_INVALID_ARG


def test_noalloc_refuses_workspace_sized_lists():
    import differentiable_sparse_linear_b200 as sla
    A, b, _ = _list(2, 6000, np.float64, 71)
    Ad = matrix(A)
    with pytest.raises(sla.SlaError) as e:
        sla.sla_pcg_solve_batched_noalloc(Ad, sla.sla_precond_jacobi(Ad), dev(b))
    assert e.value.status == sla.SLA_ERR_UNSUPPORTED
