"""PCG forward and adjoint parity with the oracle through the C ABI, on the seeded workload
recipes at sizes the oracle finishes in seconds (several tiles, ragged tails), plus
lockstep iterates, status codes and the autograd wrapper."""
import numpy as np
import pytest
import torch

import sla_workloads as W
from gpu_helpers import SOL_TOL, dev, host, iters_close, matrix, precond, rel, relmax, tol_key

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ora():
    import oracle
    return oracle.get()


def _ora_kw(w):
    return dict(precond=w.precond, G=w.G, eps=w.eps, tol=w.tol)


# (config, size, fp64 vectors with an fp32 matrix)
SINGLE = [(1, "tiny", False), (1, "small", False), (2, "tiny", False), (2, "small", False),
          (2, "small", True), (5, "tiny", False), (5, "small", False), (5, "tiny", True),
          (5, "small", True)]


def _vecs(w, vf64):
    return np.float64 if vf64 else w.dtype


def _store_f32(w, vf64):
    """fp32 vectors: the oracle's count reference is its fp32-storage mode, so the stopping
    decision is taken in the precision the solver stores its vectors in."""
    return w.dtype == np.float32 and not vf64


@pytest.mark.parametrize("engine", ["auto", "graph"])
@pytest.mark.parametrize("cfg,size,vf64", SINGLE)
def test_forward_parity(ora, cfg, size, vf64, engine):
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(cfg, size)
    Ad = matrix(w.A)
    M, _G = precond(w, Ad)
    x, info = sla.sla_pcg_solve(Ad, M, dev(w.B, _vecs(w, vf64)), rtol=w.tol, vector_f64=vf64,
                                engine=engine)
    if engine == "graph":
        assert info.engine == "graph"
    ref = ora.pcg(w.A, w.B, **_ora_kw(w))
    cnt = ora.pcg(w.A, w.B, store_f32=True, **_ora_kw(w)) if _store_f32(w, vf64) else ref
    assert info.status == 0 and ref.status == 0 and cnt.status == 0
    assert iters_close(info.iters, cnt.iters), (info.iters, cnt.iters, ref.iters)
    assert info.relres <= w.tol
    tol_sol = SOL_TOL[np.float64 if (vf64 or w.dtype == np.float64) else np.float32]
    tol_sol = max(tol_sol, 10 * w.tol if vf64 else 0)
    assert rel(host(x), ref.x) <= tol_sol
    assert relmax(host(x), ref.x) <= 10 * tol_sol
    # the true residual of the GPU solution, computed by the oracle's SpMV
    true = np.linalg.norm(w.B.astype(np.float64) - ora.spmv(w.A, host(x))) / np.linalg.norm(w.B)
    assert true <= (10 * w.tol if w.dtype == np.float64 else 1e-3)


@pytest.mark.parametrize("engine", ["auto", "graph"])
@pytest.mark.parametrize("cfg,size,vf64", SINGLE)
def test_adjoint_parity(ora, cfg, size, vf64, engine):
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(cfg, size)
    Ad = matrix(w.A)
    M, _G = precond(w, Ad)
    x, _ = sla.sla_pcg_solve(Ad, M, dev(w.B, _vecs(w, vf64)), rtol=w.tol, vector_f64=vf64, engine=engine)
    lam, g, info = sla.sla_pcg_adjoint(Ad, M, x, dev(w.W, _vecs(w, vf64)), rtol=w.tol, vector_f64=vf64,
                                       engine=engine)
    xo = ora.pcg(w.A, w.B, **_ora_kw(w)).x
    ref = ora.adjoint(w.A, xo, w.W, **_ora_kw(w))
    if _store_f32(w, vf64):
        x32 = ora.pcg(w.A, w.B, store_f32=True, **_ora_kw(w)).x
        cnt = ora.adjoint(w.A, x32, w.W, store_f32=True, **_ora_kw(w))
    else:
        cnt = ref
    assert info.status == 0
    assert iters_close(info.iters, cnt.iters), (info.iters, cnt.iters, ref.iters)
    t = SOL_TOL[tol_key(w.dtype)]
    assert rel(host(lam), ref.lam) <= t
    assert rel(host(g), ref.grad) <= t
    assert relmax(host(lam), ref.lam) <= 10 * t
    assert relmax(host(g), ref.grad) <= 10 * t
    # the gradient is -lam_i x_j of the GPU's own lam and x, rounded once to A's type
    g2 = ora.grad(w.A, host(lam), host(x))
    assert rel(host(g), g2) <= (1e-15 if w.dtype == np.float64 else 1e-7)


@pytest.mark.parametrize("engine", ["auto", "graph"])
@pytest.mark.parametrize("k", [1, 2, 5, 17])
@pytest.mark.parametrize("cfg,vf64", [(1, False), (2, False), (5, False), (5, True)])
def test_lockstep_iterates(ora, cfg, vf64, k, engine):
    """Both sides run exactly k iterations; the iterates agree (no stopping-rule effects)."""
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(cfg, "small")
    Ad = matrix(w.A)
    M, _G = precond(w, Ad)
    x, info = sla.sla_pcg_solve(Ad, M, dev(w.B, _vecs(w, vf64)), rtol=1e-300, maxit=k, vector_f64=vf64,
                                engine=engine)
    assert info.status == sla.SLA_NOT_CONVERGED and info.iters == k
    ref = ora.pcg(w.A, w.B, precond=w.precond, G=w.G, eps=w.eps, fixed_iters=k)
    bound = 1e-11 if (w.dtype == np.float64 or vf64) else 1e-5
    assert rel(host(x), ref.x) <= bound
    assert abs(info.relres - ref.relres) <= bound * max(1.0, ref.relres) * 10


@pytest.mark.parametrize("size", ["tiny", "small"])
def test_multi_rhs_parity(ora, size):
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(3, size)
    Ad = matrix(w.A)
    M, _ = precond(w, Ad)
    X, infos = sla.sla_pcg_solve_batched(Ad, M, dev(w.B), rtol=w.tol)
    Xo, outs = ora.pcg_multi(w.A, w.B, **_ora_kw(w))
    X32, c32 = ora.pcg_multi(w.A, w.B, store_f32=True, **_ora_kw(w))   # fp32 vectors: counts in fp32 storage
    for c in range(w.nrhs):
        assert infos[c].status == 0
        assert iters_close(infos[c].iters, c32[c].iters), (c, infos[c].iters, c32[c].iters, outs[c].iters)
        assert rel(host(X)[:, c], Xo[:, c]) <= SOL_TOL[np.float32]
    Lam, G, ainf = sla.sla_pcg_adjoint_batched(Ad, M, X, dev(w.W), rtol=w.tol)
    Lo, go, aouts = ora.adjoint_multi(w.A, Xo, w.W, **_ora_kw(w))
    _, _, a32 = ora.adjoint_multi(w.A, X32, w.W, store_f32=True, **_ora_kw(w))
    for c in range(w.nrhs):
        assert iters_close(ainf[c].iters, a32[c].iters), (c, ainf[c].iters, a32[c].iters, aouts[c].iters)
    assert rel(host(Lam), Lo) <= SOL_TOL[np.float32]
    assert rel(host(G), go) <= SOL_TOL[np.float32]


@pytest.mark.parametrize("nrhs", [1, 3, 5, 16])
def test_batched_equals_single(nrhs):
    """Each column of a shared-pattern batch equals its own single solve (per-RHS freeze)."""
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(1, "small")
    Ad = matrix(w.A)
    M = sla.sla_precond_jacobi(Ad)
    rng = np.random.default_rng(nrhs)
    B = rng.uniform(-1, 1, size=(w.A.n_rows, nrhs))
    B[:, 0] *= 1e-3                                      # different convergence histories
    X, infos = sla.sla_pcg_solve_batched(Ad, M, dev(B), rtol=1e-10)
    for c in range(nrhs):
        x1, i1 = sla.sla_pcg_solve(Ad, M, dev(np.ascontiguousarray(B[:, c])), rtol=1e-10)
        assert infos[c].iters == i1.iters
        assert rel(host(X)[:, c], host(x1)) <= 1e-13


@pytest.mark.parametrize("size", ["tiny", "small"])
def test_list_parity(ora, size):
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(4, size)
    Ad = matrix(w.A)
    M = sla.sla_precond_jacobi(Ad)
    x, infos = sla.sla_pcg_solve_batched(Ad, M, dev(w.B), rtol=w.tol)
    xo, outs = ora.pcg_list(w.A, w.B, precond="jacobi", tol=w.tol)
    assert len(infos) == w.A.batch
    for s in range(w.A.batch):
        assert infos[s].status == 0
        assert iters_close(infos[s].iters, outs[s].iters), (s, infos[s].iters, outs[s].iters)
    assert rel(host(x), xo) <= SOL_TOL[np.float64]
    lam, g, ainf = sla.sla_pcg_adjoint_batched(Ad, M, x, dev(w.W), rtol=w.tol)
    lo, go, aouts = ora.adjoint_list(w.A, xo, w.W, precond="jacobi", tol=w.tol)
    for s in range(w.A.batch):
        assert iters_close(ainf[s].iters, aouts[s].iters)
    assert rel(host(lam), lo) <= SOL_TOL[np.float64]
    assert rel(host(g), go) <= SOL_TOL[np.float64]


def test_no_preconditioner(ora):
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(1, "small")
    Ad = matrix(w.A)
    x, info = sla.sla_pcg_solve(Ad, None, dev(w.B), rtol=1e-10)
    ref = ora.pcg(w.A, w.B, precond="none", tol=1e-10)
    assert iters_close(info.iters, ref.iters)
    assert rel(host(x), ref.x) <= 1e-8


def test_status_codes():
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(1, "small")
    Ad = matrix(w.A)
    M = sla.sla_precond_jacobi(Ad)
    n = w.A.n_rows
    # b = 0: x = 0 after 0 iterations
    x, info = sla.sla_pcg_solve(Ad, M, torch.zeros(n, dtype=torch.float64, device="cuda"))
    assert info.status == 0 and info.iters == 0 and not x.any()
    # maxit reached
    x, info = sla.sla_pcg_solve(Ad, M, dev(w.B), rtol=1e-15, maxit=3)
    assert info.status == sla.SLA_NOT_CONVERGED and info.iters == 3
    # indefinite matrix: breakdown, reported, no hang
    ind = W.CSR(2, 2, np.array([0, 1, 2], np.int32), np.array([0, 1], np.int32), np.array([1.0, -1.0]))
    Ai = matrix(ind)
    x, info = sla.sla_pcg_solve(Ai, None, dev(np.array([1.0, 1.0])))
    assert info.status == sla.SLA_BREAKDOWN
    # Jacobi needs a positive diagonal
    with pytest.raises(sla.SlaError):
        sla.sla_precond_jacobi(Ai)
    # NaN in b: breakdown, not a hang
    b = dev(w.B).clone()
    b[5] = float("nan")
    x, info = sla.sla_pcg_solve(Ad, M, b)
    assert info.status == sla.SLA_BREAKDOWN
    # preconditioner of another matrix
    A2 = matrix(w.A)
    with pytest.raises(sla.SlaError):
        sla.sla_pcg_solve(A2, M, dev(w.B))


def test_repeat_solves_reuse_plan():
    """The captured graph is replayed: repeated calls give identical results."""
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(2, "small")
    Ad = matrix(w.A)
    M, _G = precond(w, Ad)
    x1, i1 = sla.sla_pcg_solve(Ad, M, dev(w.B))
    x2, i2 = sla.sla_pcg_solve(Ad, M, dev(w.B))
    assert i1.iters == i2.iters and torch.equal(x1, x2)
    ws = sla.sla_workspace_bytes(Ad, M, 1)
    assert 0 < ws < 16 * w.A.n_rows * 4 + (4 << 20)   # O(n), independent of iterations


def test_autograd_solve(ora):
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(1, "small")
    rp, ci = dev(w.A.row_ptr), dev(w.A.col)
    val = dev(w.A.val).requires_grad_(True)
    A = sla.sla_csr_create(rp, ci, val.detach())
    A.val = val
    M = sla.sla_precond_jacobi(A)
    b = dev(w.B).requires_grad_(True)
    x = sla.solve(A, b, M, rtol=1e-12)
    loss = (dev(w.W) * x).sum()
    loss.backward()
    xo = ora.pcg(w.A, w.B, "jacobi", tol=1e-12).x
    ref = ora.adjoint(w.A, xo, w.W, "jacobi", tol=1e-12)
    assert rel(host(b.grad), ref.lam) <= 1e-8
    assert rel(host(val.grad), ref.grad) <= 1e-8


@pytest.mark.parametrize("order", ["A", "G", "M"])
def test_handle_destruction_any_order(order):
    """Handles may be destroyed in any order; a preconditioner whose G is gone is refused."""
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(2, "tiny")
    Ad = matrix(w.A)
    M, Gd = precond(w, Ad)
    sla.sla_pcg_solve(Ad, M, dev(w.B))
    if order == "A":
        Ad.close()
        with pytest.raises(sla.SlaError):
            M.refresh()
        M.close()
        Gd.close()
    elif order == "G":
        Gd.close()
        with pytest.raises(sla.SlaError):
            sla.sla_pcg_solve(Ad, M, dev(w.B))
        Ad.close()
        M.close()
    else:
        M.close()
        x, info = sla.sla_pcg_solve(Ad, None, dev(w.B))
        assert info.status == 0
        Gd.close()
        Ad.close()


def _mixed_length_spd(n=6000, hubs=150, seed=11):
    """fp32 SPD matrix whose row lengths fill every lane-group length bin: ordinary rows link
    to 0-40 others, mostly hub rows (1 to ~45 entries per row); the hub rows collect a few
    hundred entries each."""
    rng = np.random.default_rng(seed)
    deg = rng.choice([0, 1, 2, 3, 6, 12, 25, 40], size=n, p=[.2, .2, .15, .15, .1, .1, .06, .04])
    lo, hi = [], []
    for i in range(hubs, n):
        d = int(deg[i])
        if d == 0:
            continue
        js = np.where(rng.random(d) < 0.8, rng.integers(0, hubs, d), rng.integers(0, n, d))
        js = js[js != i]
        lo.append(np.minimum(js, i))
        hi.append(np.maximum(js, i))
    lo = np.concatenate(lo).astype(np.int64)
    hi = np.concatenate(hi).astype(np.int64)
    key = np.unique(lo * n + hi)
    return W._assemble_symmetric(key // n, key % n, n, seed, 0.1, np.float32)


@pytest.mark.parametrize("nrhs", [1, 2, 3, 4, 8])
def test_mixed_row_lengths_multi_rhs(ora, nrhs):
    """The long-row engines (lane groups up to 4 right-hand sides, row tiles above) on a
    SPAI-preconditioned matrix whose rows fill every length bin, from 1 entry to hundreds:
    lockstep iterates, then converged solve and adjoint against the oracle."""
    import differentiable_sparse_linear_b200 as sla
    A = _mixed_length_spd()
    lens = np.diff(A.row_ptr)
    assert lens.min() == 1 and lens.max() > 128
    G = W.spai_factor_G(A, seed=12)
    eps = 3e-3
    kw = dict(precond="spai", G=G, eps=eps)
    Ad, Gd = matrix(A), matrix(G)
    M = sla.sla_precond_spai(Ad, Gd, eps)
    B = np.random.default_rng(13).standard_normal((A.n_rows, nrhs)).astype(np.float32)
    k = 7
    X, infos = sla.sla_pcg_solve_batched(Ad, M, dev(B), rtol=1e-300, maxit=k)
    assert all(i.engine == "graph" and i.iters == k for i in infos)
    Xo, _ = ora.pcg_multi(A, B, fixed_iters=k, **kw)
    assert rel(host(X), Xo) <= 1e-5
    # converged, fp64 vectors: the iteration counts match the oracle's
    X, infos = sla.sla_pcg_solve_batched(Ad, M, dev(B, np.float64), rtol=1e-6, vector_f64=True)
    Xo, outs = ora.pcg_multi(A, B, tol=1e-6, **kw)
    for c in range(nrhs):
        assert infos[c].status == 0
        assert iters_close(infos[c].iters, outs[c].iters), (c, infos[c].iters, outs[c].iters)
    assert rel(host(X), Xo) <= 1e-5
    Wt = np.random.default_rng(14).uniform(-1, 1, size=(A.n_rows, nrhs))
    Lam, g, ainf = sla.sla_pcg_adjoint_batched(Ad, M, X, dev(Wt), rtol=1e-6, vector_f64=True)
    Lo, go, aouts = ora.adjoint_multi(A, Xo, Wt, tol=1e-6, **kw)
    for c in range(nrhs):
        assert iters_close(ainf[c].iters, aouts[c].iters)
    assert rel(host(Lam), Lo) <= SOL_TOL[np.float32]
    assert rel(host(g), go) <= SOL_TOL[np.float32]
