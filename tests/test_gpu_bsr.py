"""Block sparse row (BSR) matrices through the C ABI against the oracle: SpMV for block sizes
2-4 with empty, short and long block rows; PCG solve and adjoint (Jacobi and SPAI with a
CSR factor); multi-RHS; lockstep iterates; the calls a BSR handle refuses."""
import numpy as np
import pytest

import sla_workloads as W
from gpu_helpers import SOL_TOL, SPMV_TOL, dev, host, iters_close, matrix, rel, tol_key

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ora():
    import oracle
    return oracle.get()


def bsr(A, validate=True):
    import differentiable_sparse_linear_b200 as sla
    return sla.sla_bsr_create(dev(A.row_ptr), dev(A.col), dev(A.val), validate=validate)


def _lens(n, seed):
    lens = np.random.default_rng(seed).integers(0, 6, size=n)
    lens[::11] = 0                       # empty block rows
    lens[[3, n // 2]] = [min(n, 300), 40]  # block rows for whole warps and 16-lane groups
    return lens


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("b", [2, 3, 4])
def test_bsr_spmv(ora, b, dtype):
    import differentiable_sparse_linear_b200 as sla
    A = W.random_bsr(700, b, _lens(700, b), 60 + b, dtype)
    Ad = bsr(A)
    assert Ad.n == A.n_rows and Ad.nnz == A.nnz
    x = np.random.default_rng(7).uniform(-1, 1, A.n_rows).astype(dtype)
    y = sla.sla_spmv(Ad, dev(x))
    assert rel(host(y), ora.bsr_spmv(A, x)) <= SPMV_TOL[tol_key(dtype)]


@pytest.mark.parametrize("k", [2, 3, 4])
def test_bsr_spmv_multi(ora, k):
    import differentiable_sparse_linear_b200 as sla
    A = W.random_bsr(500, 3, _lens(500, 5), 70, np.float32)
    X = np.random.default_rng(8).uniform(-1, 1, (A.n_rows, k)).astype(np.float32)
    Y = sla.sla_spmv_multi(bsr(A), dev(X))
    ref = np.stack([ora.bsr_spmv(A, X[:, c]) for c in range(k)], axis=1)
    assert rel(host(Y), ref) <= SPMV_TOL[np.float32]


@pytest.mark.parametrize("b,N,dtype", [(3, 16, np.float32), (2, 10, np.float64), (4, 8, np.float32),
                                       (3, 5, np.float64)])
def test_bsr_solve_adjoint(ora, b, N, dtype):
    import differentiable_sparse_linear_b200 as sla
    A = W.elastic3d_bsr(N, b, 0.1, dtype)
    n = A.n_rows
    bv = W.rhs_normal(11, n, dtype)
    wv = W.rhs_uniform(12, n, dtype=dtype)
    tol = 1e-10 if dtype == np.float64 else 1e-6
    Ad = bsr(A)
    M = sla.sla_precond_jacobi(Ad)
    x, info = sla.sla_pcg_solve(Ad, M, dev(bv), rtol=tol)
    ref = ora.pcg_bsr(A, bv, precond="jacobi", tol=tol)
    # fp32 vectors: the stopping decision is compared in fp32 storage on both sides
    f32 = dtype == np.float32
    cnt = ora.pcg_bsr(A, bv, precond="jacobi", tol=tol, store_f32=True) if f32 else ref
    assert info.status == 0 and info.engine == "graph"
    assert iters_close(info.iters, cnt.iters), (info.iters, cnt.iters, ref.iters)
    assert rel(host(x), ref.x) <= SOL_TOL[tol_key(dtype)]
    lam, g, ainf = sla.sla_pcg_adjoint(Ad, M, x, dev(wv), rtol=tol)
    adj = ora.adjoint_bsr(A, ref.x, wv, precond="jacobi", tol=tol)
    acnt = ora.adjoint_bsr(A, cnt.x, wv, precond="jacobi", tol=tol, store_f32=True) if f32 else adj
    assert ainf.status == 0 and iters_close(ainf.iters, acnt.iters), (ainf.iters, acnt.iters, adj.iters)
    assert rel(host(lam), adj.lam) <= SOL_TOL[tol_key(dtype)]
    assert rel(host(g).reshape(A.val.shape), adj.grad) <= SOL_TOL[tol_key(dtype)]
    # the gradient is -lam_i x_j of the GPU's own lam and x, in block order
    Ac, pos = ora.bsr_to_csr(A)
    g2 = np.empty(A.nnz)
    g2[pos] = ora.grad(Ac, host(lam), host(x))
    assert rel(host(g), g2) <= (1e-15 if dtype == np.float64 else 1e-7)


@pytest.mark.parametrize("k", [1, 4, 9])
def test_bsr_lockstep(ora, k):
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(6, "small")
    Ad = bsr(w.A)
    M = sla.sla_precond_jacobi(Ad)
    x, info = sla.sla_pcg_solve(Ad, M, dev(w.B), rtol=1e-300, maxit=k)
    assert info.status == sla.SLA_NOT_CONVERGED and info.iters == k
    ref = ora.pcg_bsr(w.A, w.B, precond="jacobi", fixed_iters=k)
    assert rel(host(x), ref.x) <= 1e-5


def test_bsr_with_spai(ora):
    """BSR A with the SPAI preconditioner of a CSR factor G on A's scalar pattern."""
    import differentiable_sparse_linear_b200 as sla
    A = W.elastic3d_bsr(8, 3, 0.1, np.float32)
    Ac, _ = ora.bsr_to_csr(A)
    Ac32 = W.CSR(Ac.n_rows, Ac.n_cols, Ac.row_ptr, Ac.col, Ac.val.astype(np.float32))
    G = W.spai_factor_G(Ac32, seed=13, dtype=np.float32)
    Ad = bsr(A)
    M = sla.sla_precond_spai(Ad, matrix(G), 3e-3)
    bv = W.rhs_normal(14, A.n_rows, np.float32)
    x, info = sla.sla_pcg_solve(Ad, M, dev(bv, np.float64), rtol=1e-6, vector_f64=True)
    ref = ora.pcg(Ac, bv, precond="spai", G=G, eps=3e-3, tol=1e-6)
    assert info.status == 0 and iters_close(info.iters, ref.iters), (info.iters, ref.iters)
    assert rel(host(x), ref.x) <= 1e-5


@pytest.mark.parametrize("nrhs", [2, 3, 4])
def test_bsr_multi_rhs(ora, nrhs):
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(6, "tiny")
    Ad = bsr(w.A)
    M = sla.sla_precond_jacobi(Ad)
    B = W.rhs_normal(15 + nrhs, (w.A.n_rows, nrhs), np.float64)
    X, infos = sla.sla_pcg_solve_batched(Ad, M, dev(B), rtol=1e-6, vector_f64=True)
    Xo, outs = ora.pcg_multi(ora.bsr_to_csr(w.A)[0], B, precond="jacobi", tol=1e-6)
    for c in range(nrhs):
        assert infos[c].status == 0 and iters_close(infos[c].iters, outs[c].iters)
    assert rel(host(X), Xo) <= 1e-5
    Wt = W.rhs_uniform(16, (w.A.n_rows, nrhs), dtype=np.float64)
    Lam, g, _ = sla.sla_pcg_adjoint_batched(Ad, M, X, dev(Wt), rtol=1e-6, vector_f64=True)
    Lo, go, _ = ora.adjoint_multi(ora.bsr_to_csr(w.A)[0], Xo, Wt, precond="jacobi", tol=1e-6)
    _, pos = ora.bsr_to_csr(w.A)
    gb = np.empty(w.A.nnz)
    gb[pos] = go
    assert rel(host(Lam), Lo) <= SOL_TOL[np.float32]
    assert rel(host(g), gb) <= SOL_TOL[np.float32]


def test_bsr_refusals():
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(6, "tiny")
    Ad = bsr(w.A)
    M = sla.sla_precond_jacobi(Ad)
    with pytest.raises(sla.SlaError) as e:                      # more than 4 right-hand sides
        sla.sla_pcg_solve_batched(Ad, M, dev(np.ones((w.A.n_rows, 5), np.float32)), rtol=1e-6)
    assert e.value.status == sla.SLA_ERR_INVALID_ARG
    with pytest.raises(sla.SlaError) as e:                      # the persistent engine is CSR-only
        sla.sla_pcg_solve(Ad, M, dev(w.B), rtol=1e-6, engine="persistent")
    assert e.value.status == sla.SLA_ERR_INVALID_ARG
    with pytest.raises(sla.SlaError) as e:                      # G must be CSR
        sla.sla_precond_spai(Ad, Ad, 3e-3)
    assert e.value.status == sla.SLA_ERR_INVALID_ARG
    bad = W.BSR(w.A.n_brows, 3, w.A.row_ptr, w.A.col.copy(), w.A.val)
    bad.col[1] = w.A.n_brows                                    # block column out of range
    with pytest.raises(sla.SlaError) as e:
        bsr(bad)
    assert e.value.status == sla.SLA_ERR_INVALID_CSR
    one = W.BSR(1, 2, np.array([0, 1], np.int32), np.array([0], np.int32),
                np.array([[[2.0, 0.5], [0.5, 1.0]]], np.float64))
    Od = bsr(one)
    x, info = sla.sla_pcg_solve(Od, sla.sla_precond_jacobi(Od), dev(np.array([1.0, 2.0])), rtol=1e-12)
    assert info.status == 0
    assert rel(host(x), np.linalg.solve(one.val[0], [1.0, 2.0])) <= 1e-12
