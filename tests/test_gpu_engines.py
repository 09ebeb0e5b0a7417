"""The two solve engines (graph of fused kernels; one persistent cooperative kernel): which
one runs, that they agree with each other and with the oracle, and the persistent
kernel's phase accounting."""
import numpy as np
import pytest

import sla_workloads as W
from gpu_helpers import SOL_TOL, dev, host, iters_close, matrix, precond, rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ora():
    import oracle
    return oracle.get()


def _solve(sla, w, Ad, M, engine, vf64=False):
    vt = np.float64 if vf64 else w.dtype
    if w.nrhs > 1:
        X, infos = sla.sla_pcg_solve_batched(Ad, M, dev(w.B, vt), rtol=w.tol, engine=engine, vector_f64=vf64)
        return X, infos
    x, info = sla.sla_pcg_solve(Ad, M, dev(w.B, vt), rtol=w.tol, engine=engine, vector_f64=vf64)
    return x, [info]


@pytest.mark.parametrize("cfg,size,vf64,want", [
    (1, "small", False, "persistent"),    # fp64 Jacobi, 5-point rows
    (2, "small", False, "persistent"),    # fp32 SPAI: A, G, G^T all short-row
    (2, "small", True, "persistent"),     # fp32 matrix, fp64 vectors
    (3, "small", False, "persistent"),    # 8 right-hand sides, 7-point rows
    (5, "small", False, "graph"),         # power-law rows: the persistent engine does not apply
])
def test_engine_choice(cfg, size, vf64, want):
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(cfg, size)
    Ad = matrix(w.A)
    M, _G = precond(w, Ad)
    _, infos = _solve(sla, w, Ad, M, "auto", vf64)
    assert all(i.engine == want for i in infos), [i.engine for i in infos]
    _, infos = _solve(sla, w, Ad, M, "graph", vf64)
    assert all(i.engine == "graph" for i in infos)
    if want == "graph":
        with pytest.raises(sla.SlaError) as e:
            _solve(sla, w, Ad, M, "persistent", vf64)
        assert e.value.status == sla.SLA_ERR_INVALID_ARG


def test_list_engine_reported():
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(4, "tiny")
    Ad = matrix(w.A)
    M = sla.sla_precond_jacobi(Ad)
    _, infos = sla.sla_pcg_solve_batched(Ad, M, dev(w.B), rtol=w.tol)
    assert all(i.engine == "list" for i in infos)


@pytest.mark.parametrize("cfg,size,vf64", [(1, "tiny", False), (1, "small", False), (2, "tiny", False),
                                           (2, "small", False), (2, "small", True), (3, "tiny", False),
                                           (3, "small", False)])
def test_engines_agree(ora, cfg, size, vf64):
    """Same iterates up to the summation order of the dot products: iteration counts within
    one, solutions within the solve tolerance class; the persistent result also against
    the oracle."""
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(cfg, size)
    Ad = matrix(w.A)
    M, _G = precond(w, Ad)
    xp, ip = _solve(sla, w, Ad, M, "persistent", vf64)
    xg, ig = _solve(sla, w, Ad, M, "graph", vf64)
    assert all(i.engine == "persistent" for i in ip)
    for a, b in zip(ip, ig):
        assert a.status == 0 and b.status == 0
        assert abs(a.iters - b.iters) <= 1, (a.iters, b.iters)
    f64 = vf64 or w.dtype == np.float64
    # both stop at relative residual w.tol; the summation orders differ, so the iterates
    # agree to the solve tolerance, not to rounding
    assert rel(host(xp), host(xg)) <= (max(1e-9, 10 * w.tol) if f64 else 1e-4)
    kw = dict(precond=w.precond, G=w.G, eps=w.eps, tol=w.tol)
    if w.nrhs > 1:
        xo, outs = ora.pcg_multi(w.A, w.B, **kw)
        its = [o.iters for o in outs]
    else:
        ref = ora.pcg(w.A, w.B, **kw)
        xo, its = ref.x, [ref.iters]
    for a, it in zip(ip, its):
        assert iters_close(a.iters, it), (a.iters, it)
    tol = SOL_TOL[np.float64 if f64 else np.float32]
    assert rel(host(xp).reshape(xo.shape), xo) <= max(tol, 10 * w.tol if vf64 else 0)


def test_persistent_adjoint_and_gradient(ora):
    """Adjoint solve and pattern gradient through the persistent engine (SPAI, fp32)."""
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(2, "small")
    Ad = matrix(w.A)
    M, _G = precond(w, Ad)
    x, fi = sla.sla_pcg_solve(Ad, M, dev(w.B), rtol=w.tol, engine="persistent")
    lam, g, ai = sla.sla_pcg_adjoint(Ad, M, x, dev(w.W), rtol=w.tol, engine="persistent")
    assert fi.engine == ai.engine == "persistent"
    kw = dict(precond=w.precond, G=w.G, eps=w.eps, tol=w.tol)
    xo = ora.pcg(w.A, w.B, **kw).x
    ref = ora.adjoint(w.A, xo, w.W, **kw)
    assert iters_close(ai.iters, ref.iters)
    assert rel(host(lam), ref.lam) <= SOL_TOL[np.float32]
    assert rel(host(g), ref.grad) <= SOL_TOL[np.float32]


@pytest.mark.parametrize("cfg", [1, 2])
def test_phase_counts(cfg):
    """Phase accounting of the persistent kernel: the initial pass runs one x/r update (and,
    with SPAI, one z phase); Jacobi: an iteration that converges stops after its x/r update;
    SPAI: the z phase runs before the residual test of the x/r update is read, so every
    iteration runs all three."""
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(cfg, "small")
    Ad = matrix(w.A)
    M, _G = precond(w, Ad)
    _, info = sla.sla_pcg_solve(Ad, M, dev(w.B), rtol=w.tol, engine="persistent")
    ms, cnt = sla.sla_pcg_phase_times(Ad, M)
    k = info.iters
    if w.precond == "spai":
        assert cnt == [k, k + 1, k + 1, 0]
    else:
        assert cnt == [k, 0, 0, k + 1]
    for t, c in zip(ms, cnt):
        assert (t > 0) == (c > 0)
    # after a graph-engine solve there are no phase times to report
    sla.sla_pcg_solve(Ad, M, dev(w.B), rtol=w.tol, engine="graph")
    with pytest.raises(sla.SlaError):
        sla.sla_pcg_phase_times(Ad, M)


def test_persistent_edge_systems():
    """One-block grids and systems smaller than a tile: n = 1, 2 and a ragged 37-row chain."""
    import differentiable_sparse_linear_b200 as sla
    for n in (1, 2, 37):
        rows = [[(i, 4.0)] + ([(i - 1, -1.0)] if i > 0 else []) + ([(i + 1, -1.0)] if i + 1 < n else [])
                for i in range(n)]
        rp, ci, va = [0], [], []
        for r in rows:
            for j, v in sorted((j, v) for j, v in r):
                ci.append(j)
                va.append(v)
            rp.append(len(ci))
        A = W.CSR(n, n, np.array(rp, np.int32), np.array(ci, np.int32), np.array(va))
        Ad = matrix(A)
        M = sla.sla_precond_jacobi(Ad)
        b = np.linspace(-1.0, 1.0, n) + 0.5
        x, info = sla.sla_pcg_solve(Ad, M, dev(b), rtol=1e-12, engine="persistent")
        assert info.status == 0 and info.engine == "persistent"
        dense = np.zeros((n, n))
        for i in range(n):
            for k in range(rp[i], rp[i + 1]):
                dense[i, ci[k]] = va[k]
        assert rel(host(x), np.linalg.solve(dense, b)) <= 1e-10
