"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each ``check_*`` takes an ``oracle.Oracle`` and raises AssertionError on failure.  The pin
tests run them on the oracle as built; the planted-mistake tests run them on copies of the
oracle with one plausible mistake each and require that some check fails.

What pins what:
  * SpMV       -- closed-form eigenpairs of the 1D/2D/3D Dirichlet Laplacians (the 2D one
                  is the Poisson model problem of the torch-sla page's experiments); a dense
                  matvec (numpy) on random rectangular matrices.
  * transpose  -- dense transpose.
  * PCG        -- the defining optimality of CG: the k-th iterate is the A-norm-optimal
                  point of the Krylov space K_k(M^-1 A, M^-1 b) (Galerkin condition), built
                  here with dense QR and a dense solve; one-step convergence on an
                  eigenvector; m-step termination for m distinct eigenvalues; agreement
                  with a dense LU solve; invariance under scaling of b; status codes.
  * SPAI apply -- the dense product (G G^T + eps I) r.
  * adjoint    -- A lam = w; w.x = lam.b; sum A_ij g_ij = -L; central finite differences
                  of L = w.A^-1 b (dense LU) in single stored entries and in b.
  * fp32 storage -- a hand-worked 2 x 2 case in which binary32 storage of q ends CG one
                  step early with x exact; bit-exact agreement where every vector is exact
                  in binary32; returned iterates are binary32 values and track the fp64
                  recurrence to rounding for the first steps.
  * eigenvalue gradient -- the closed-form 2D Poisson eigenpairs (v_i v_j and
                  sum A_k g_k = mu) and central differences of a dense eigenvalue.
  * nonlinear adjoint -- central differences of L = w.u for A u + u^3 = b solved by dense
                  Newton, in single stored entries and in b; A + diag(c) against dense.
  * BSR        -- a dense matrix assembled block by block (numpy) for the block SpMV and the
                  scalar CSR expansion; closed-form eigenpairs of L (x) S + shift I (the
                  block vector problem) for the SpMV and one-step PCG; central finite
                  differences of L in single block entries for the gradient in block order.
"""
from __future__ import annotations

import numpy as np

import sla_workloads as W

TOL_TIGHT = 1e-13


# ------------------------------------------------------------------------------ helpers
def dense(A) -> np.ndarray:
    D = np.zeros((A.n_rows, A.n_cols), dtype=np.float64)
    rows = A.rows_of_entries()
    D[rows, A.col.astype(np.int64)] = A.val.astype(np.float64)
    return D


def csr_from_dense(D: np.ndarray) -> W.CSR:
    n_rows, n_cols = D.shape
    rp = [0]
    ci, v = [], []
    for i in range(n_rows):
        nz = np.nonzero(D[i])[0]
        ci.extend(nz.tolist())
        v.extend(D[i, nz].tolist())
        rp.append(len(ci))
    return W.CSR(n_rows, n_cols, np.array(rp, np.int32), np.array(ci, np.int32),
                 np.array(v, np.float64))


def random_sparse(rng, n_rows, n_cols, density=0.3) -> np.ndarray:
    D = rng.uniform(-1, 1, size=(n_rows, n_cols))
    D[rng.uniform(size=D.shape) > density] = 0.0
    return D


def random_spd(n: int, seed: int) -> W.CSR:
    """Small SPD matrix with a random pattern and a non-constant diagonal."""
    A = W.random_spd_list(1, n, pairs_per_row=2.0, shift=0.5, seed=seed, dtype=np.float64)
    A.sys_row_off = None
    return A


def rel(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def lap_eig_1d(N, j):
    p = np.arange(1, N + 1)
    return np.sin(j * np.pi * p / (N + 1)), 2.0 - 2.0 * np.cos(j * np.pi / (N + 1))


def dense_minv(ora, A, kind, G=None, eps=0.0) -> np.ndarray:
    n = A.n_rows
    if kind == "none":
        return np.eye(n)
    if kind == "jacobi":
        return np.diag(1.0 / np.diag(dense(A)))
    Gd = dense(G)
    return Gd @ Gd.T + eps * np.eye(n)


# ------------------------------------------------------------------------------ SpMV
def check_spmv_closed_form(ora):
    # 1D: tridiag(-1, 2, -1), eigenvalue 2 - 2cos(j pi/(N+1))
    N = 37
    A = W.poisson1d(N)
    for j in (1, 5, 36):
        v, lam = lap_eig_1d(N, j)
        assert rel(ora.spmv(A, v), lam * v) < 1e-12, "1D Laplacian eigenpair"
    # 2D: 5-point, eigenvalue 4 - 2cos(j pi/(N+1)) - 2cos(k pi/(N+1)), v = v_j (x) v_k
    N = 19
    A = W.poisson2d(N)
    for j, k in ((1, 1), (3, 7), (19, 2)):
        vj, lj = lap_eig_1d(N, j)
        vk, lk = lap_eig_1d(N, k)
        v = np.outer(vj, vk).ravel()
        assert rel(ora.spmv(A, v), (lj + lk) * v) < 1e-12, "2D Poisson eigenpair"
    # 3D heat step: A = I + dt L7, eigenvalue 1 + dt (sum of three 1D eigenvalues)
    N, dt = 9, 0.1
    A = W.heat3d(N, dt, np.float64)
    for j, k, l in ((1, 1, 1), (2, 5, 9)):
        vj, lj = lap_eig_1d(N, j)
        vk, lk = lap_eig_1d(N, k)
        vl, ll = lap_eig_1d(N, l)
        v = np.einsum("a,b,c->abc", vj, vk, vl).ravel()
        assert rel(ora.spmv(A, v), (1 + dt * (lj + lk + ll)) * v) < 1e-12, "3D heat eigenpair"


def check_spmv_dense(ora):
    rng = np.random.default_rng(11)
    for shape in ((30, 30), (20, 33), (41, 7)):
        D = random_sparse(rng, *shape)
        D[3, :] = 0.0                       # an empty row
        A = csr_from_dense(D)
        x = rng.standard_normal(shape[1])
        assert rel(ora.spmv(A, x), D @ x) < 1e-14, f"SpMV vs dense {shape}"


def check_transpose(ora):
    rng = np.random.default_rng(12)
    D = random_sparse(rng, 17, 23, 0.35)
    At = ora.transpose(csr_from_dense(D))
    assert At.n_rows == 23 and At.n_cols == 17
    assert np.array_equal(dense(At), D.T), "transpose vs dense"
    for i in range(At.n_rows):
        seg = At.col[At.row_ptr[i]:At.row_ptr[i + 1]]
        assert np.all(np.diff(seg) > 0), "transpose keeps columns ascending"


def check_spai_apply(ora):
    rng = np.random.default_rng(13)
    A = random_spd(30, 101)
    G = W.spai_factor_G(A, seed=7, dtype=np.float64)
    r = rng.standard_normal(A.n_rows)
    for eps in (3e-3, 0.25):
        z = ora.precond_apply(A, r, "spai", G=G, eps=eps)
        Gd = dense(G)
        assert rel(z, (Gd @ Gd.T + eps * np.eye(A.n_rows)) @ r) < 1e-14, "SPAI apply vs dense"
    zj = ora.precond_apply(A, r, "jacobi")
    assert rel(zj, r / np.diag(dense(A))) < 1e-15, "Jacobi apply vs dense"


# ------------------------------------------------------------------------------ PCG
def check_pcg_krylov_optimal(ora):
    """x_k is the Galerkin (A-norm optimal) point of K_k(M^-1 A, M^-1 b), for k = 1..5."""
    rng = np.random.default_rng(14)
    A = random_spd(14, 202)
    Ad = dense(A)
    G = W.spai_factor_G(A, seed=9, dtype=np.float64)
    b = rng.standard_normal(A.n_rows)
    for kind in ("none", "jacobi", "spai"):
        Minv = dense_minv(ora, A, kind, G, 0.01)
        v = Minv @ b
        basis = []
        for k in range(1, 6):
            basis.append(v / np.linalg.norm(v))
            v = Minv @ (Ad @ basis[-1])
            Q, _ = np.linalg.qr(np.array(basis).T)
            x_ref = Q @ np.linalg.solve(Q.T @ Ad @ Q, Q.T @ b)
            res = ora.pcg(A, b, precond=kind, G=G, eps=0.01, fixed_iters=k)
            assert res.iters == k
            assert rel(res.x, x_ref) < 1e-10, f"{kind}: iterate {k} is not Krylov-optimal"
            true_rel = np.linalg.norm(b - Ad @ res.x) / np.linalg.norm(b)
            assert abs(res.relres - true_rel) <= 1e-12, f"{kind}: recursive residual drifts at {k}"


def check_pcg_eigvec_one_step(ora):
    N = 16
    A = W.poisson2d(N)
    vj, lj = lap_eig_1d(N, 3)
    vk, lk = lap_eig_1d(N, 5)
    b = np.outer(vj, vk).ravel()
    res = ora.pcg(A, b, "jacobi", tol=1e-12)
    assert res.iters == 1, f"eigenvector rhs needs one step, took {res.iters}"
    assert rel(res.x, b / (lj + lk)) < 1e-13, "x = v / lambda"


def check_pcg_m_distinct(ora):
    N = 16
    A = W.poisson2d(N)
    pairs = [(1, 1), (1, 2), (2, 3), (4, 4), (7, 9)]        # distinct eigenvalues
    lams = []
    b = np.zeros(N * N)
    for c, (j, k) in enumerate(pairs):
        vj, lj = lap_eig_1d(N, j)
        vk, lk = lap_eig_1d(N, k)
        lams.append(lj + lk)
        b += (1.0 + c) * np.outer(vj, vk).ravel()
    assert len(set(np.round(lams, 12))) == len(pairs)
    res = ora.pcg(A, b, "jacobi", tol=1e-10)
    assert res.iters == len(pairs), f"{len(pairs)} distinct eigenvalues, {res.iters} steps"


def check_pcg_dense_solve(ora):
    rng = np.random.default_rng(15)
    for n, seed in ((8, 1), (33, 2), (64, 3)):
        A = random_spd(n, 300 + seed)
        Ad = dense(A)
        G = W.spai_factor_G(A, seed=seed, dtype=np.float64)
        b = rng.uniform(-1, 1, n)
        x_ref = np.linalg.solve(Ad, b)
        kappa = np.linalg.cond(Ad)
        for kind in ("none", "jacobi", "spai"):
            res = ora.pcg(A, b, precond=kind, G=G, eps=3e-3, tol=1e-12)
            assert res.status == 0, f"{kind} n={n} status {res.status}"
            assert res.iters <= n + 5, f"{kind} n={n}: {res.iters} steps"
            assert rel(res.x, x_ref) < 10 * kappa * 1e-12, f"{kind} n={n} vs dense solve"


def check_pcg_scaling(ora):
    A = random_spd(40, 404)
    b = np.random.default_rng(16).standard_normal(40)
    r1 = ora.pcg(A, b, "jacobi", tol=1e-9)
    r2 = ora.pcg(A, 1e6 * b, "jacobi", tol=1e-9)
    assert r1.iters == r2.iters, "the stopping test is relative to ||b||"
    assert rel(r2.x, 1e6 * r1.x) < 1e-12


def check_pcg_status(ora):
    A = W.poisson2d(12)
    n = A.n_rows
    res = ora.pcg(A, np.zeros(n), "jacobi", tol=1e-10)
    assert res.status == 0 and res.iters == 0 and not res.x.any(), "b = 0 gives x = 0, 0 steps"
    b = np.random.default_rng(17).uniform(-1, 1, n)
    res = ora.pcg(A, b, "jacobi", tol=1e-14, maxit=3)
    assert res.status == 1 and res.iters == 3, "maxit reached -> not converged"
    ind = csr_from_dense(np.diag([1.0, -1.0]))
    res = ora.pcg(ind, np.array([1.0, 1.0]), "none", tol=1e-10)
    assert res.status == 2, "p.q = 0 on an indefinite matrix -> breakdown"


# ------------------------------------------------------------------------------ adjoint
def _loss_dense(Ad, b, w):
    return float(w @ np.linalg.solve(Ad, b))


def check_adjoint_identities(ora):
    rng = np.random.default_rng(18)
    for A in (W.poisson2d(14), random_spd(50, 505)):
        n = A.n_rows
        b = rng.uniform(-1, 1, n)
        w = rng.uniform(-1, 1, n)
        fw = ora.pcg(A, b, "jacobi", tol=1e-13)
        adj = ora.adjoint(A, fw.x, w, "jacobi", tol=1e-13)
        L = float(w @ fw.x)
        assert rel(ora.spmv(A, adj.lam), w) < 1e-12, "A^T lam = w"
        assert abs(float(adj.lam @ b) - L) <= 1e-10 * max(1.0, abs(L)), "lam.b = w.x"
        s = float(np.sum(A.val.astype(np.float64) * adj.grad))
        assert abs(s + L) <= 1e-10 * max(1.0, abs(L)), "sum A_ij g_ij = -L"


def check_grad_fd(ora):
    """Central differences of L = w.A^-1 b in single stored entries (dense LU)."""
    rng = np.random.default_rng(19)
    A = random_spd(15, 606)
    Ad = dense(A)
    b = rng.uniform(-1, 1, 15)
    w = rng.uniform(-1, 1, 15)
    fw = ora.pcg(A, b, "jacobi", tol=1e-14)
    adj = ora.adjoint(A, fw.x, w, "jacobi", tol=1e-14)
    rows = A.rows_of_entries()
    picks = rng.choice(A.nnz, size=12, replace=False)
    for kk in picks:
        i, j = int(rows[kk]), int(A.col[kk])
        h = 1e-6 * max(1.0, abs(Ad[i, j]))
        Ap = Ad.copy(); Ap[i, j] += h
        Am = Ad.copy(); Am[i, j] -= h
        fd = (_loss_dense(Ap, b, w) - _loss_dense(Am, b, w)) / (2 * h)
        assert abs(adj.grad[kk] - fd) <= 1e-7 * max(1.0, abs(fd)), f"dL/dA[{i},{j}]"
    for i in rng.choice(15, size=5, replace=False):
        h = 1e-6
        bp = b.copy(); bp[i] += h
        bm = b.copy(); bm[i] -= h
        fd = (_loss_dense(Ad, bp, w) - _loss_dense(Ad, bm, w)) / (2 * h)
        assert abs(adj.lam[i] - fd) <= 1e-7 * max(1.0, abs(fd)), f"dL/db[{i}]"


def check_grad_fd_symmetric(ora):
    """A symmetric perturbation of (i,j) and (j,i), L evaluated by tight CG, matches g_ij + g_ji."""
    rng = np.random.default_rng(20)
    A = W.poisson2d(8)
    n = A.n_rows
    b = rng.uniform(-1, 1, n)
    w = rng.uniform(-1, 1, n)
    fw = ora.pcg(A, b, "jacobi", tol=1e-14)
    adj = ora.adjoint(A, fw.x, w, "jacobi", tol=1e-14)
    rows = A.rows_of_entries()
    index = {(int(rows[k]), int(A.col[k])): k for k in range(A.nnz)}
    for (i, j) in ((0, 1), (9, 17), (30, 30)):
        h = 1e-5
        def L_of(delta):
            B = W.CSR(A.n_rows, A.n_cols, A.row_ptr, A.col, A.val.astype(np.float64).copy())
            B.val[index[(i, j)]] += delta
            if i != j:
                B.val[index[(j, i)]] += delta
            return float(w @ ora.pcg(B, b, "jacobi", tol=1e-14).x)
        fd = (L_of(h) - L_of(-h)) / (2 * h)
        g = adj.grad[index[(i, j)]] + (adj.grad[index[(j, i)]] if i != j else 0.0)
        assert abs(g - fd) <= 1e-6 * max(1.0, abs(fd)), f"symmetric dL/dA[{i},{j}]"


def check_list_blocks(ora):
    A = W.random_spd_list(4, 30, seed=21, dtype=np.float64)
    Ad = dense(A)
    b = np.random.default_rng(22).uniform(-1, 1, A.n_rows)
    x, out = ora.pcg_list(A, b, precond="jacobi", tol=1e-13)
    assert all(r.status == 0 for r in out)
    assert rel(x, np.linalg.solve(Ad, b)) < 1e-10, "block-diagonal list vs dense solve"
    # with a block-diagonal SPAI factor, cut to each system: the same solution, and every
    # system's iterates are those of its own SPAI solve
    A.sys_row_off = np.asarray(A.sys_row_off)
    G = W.spai_factor_G(A, seed=23)
    xs, outs = ora.pcg_list(A, b, precond="spai", G=G, eps=3e-3, tol=1e-13)
    assert all(r.status == 0 for r in outs)
    assert rel(xs, np.linalg.solve(Ad, b)) < 1e-10, "SPAI list vs dense solve"
    o0, o1 = int(A.sys_row_off[2]), int(A.sys_row_off[3])
    Gs = ora.system(G, 2, A.sys_row_off)
    assert np.allclose(dense(Gs), dense(G)[o0:o1, o0:o1], rtol=0, atol=0)


# ------------------------------------------------------------------------------ BSR
def dense_bsr(A) -> np.ndarray:
    """Dense matrix of a BSR matrix, placed block by block."""
    b = A.b
    D = np.zeros((A.n_rows, A.n_rows), dtype=np.float64)
    for I in range(A.n_brows):
        for k in range(int(A.row_ptr[I]), int(A.row_ptr[I + 1])):
            J = int(A.col[k])
            D[I * b:(I + 1) * b, J * b:(J + 1) * b] = A.val[k].astype(np.float64)
    return D


def check_bsr_spmv_dense(ora):
    for b, seed in ((1, 41), (2, 42), (3, 43), (4, 44)):
        lens = np.random.default_rng(seed).integers(0, 5, size=37)
        lens[[3, 20]] = [0, 30]
        A = W.random_bsr(37, b, lens, seed, np.float64)
        D = dense_bsr(A)
        x = np.random.default_rng(seed + 100).uniform(-1, 1, A.n_rows)
        assert rel(ora.bsr_spmv(A, x), D @ x) < TOL_TIGHT, f"BSR SpMV, b = {b}"
        Ac, pos = ora.bsr_to_csr(A)
        assert np.array_equal(dense(Ac), D), f"BSR -> CSR expansion, b = {b}"
        assert np.array_equal(np.sort(pos), np.arange(A.nnz)), "BSR positions are a permutation"
        assert np.array_equal(Ac.val, A.val.reshape(-1)[pos].astype(np.float64)), "BSR positions"


def _elastic_eigvec(N, b, jkl, m):
    """Eigenvector v_jkl (x) s_m of L (x) S on the N^3 grid, and its eigenvalue factors."""
    ax = np.arange(1, N + 1)
    v = np.einsum("i,j,k->ijk", *[np.sin(j * np.pi * ax / (N + 1)) for j in jkl]).reshape(-1)
    lam = sum(2.0 - 2.0 * np.cos(j * np.pi / (N + 1)) for j in jkl)
    s = np.sin(m * np.pi * np.arange(1, b + 1) / (b + 1))
    mu = 1.0 + np.cos(m * np.pi / (b + 1))
    return np.kron(v, s), lam, mu


def check_bsr_closed_form(ora):
    for b in (2, 3):
        N, shift = 4, 0.1
        A = W.elastic3d_bsr(N, b, shift, np.float64)
        for jkl, m in (((1, 1, 1), 1), ((2, 3, 1), b), ((4, 2, 3), 2)):
            u, lam, mu = _elastic_eigvec(N, b, jkl, m)
            ev = lam * mu + shift
            assert rel(ora.bsr_spmv(A, u), ev * u) < TOL_TIGHT, f"BSR eigenpair b={b} {jkl} {m}"
            # constant diagonal (6 + shift): Jacobi is a multiple of I, CG stops in one step
            r = ora.pcg_bsr(A, u, precond="jacobi", tol=1e-12)
            assert r.status == 0 and r.iters == 1, f"one-step PCG on a BSR eigenvector ({r.iters})"
            assert rel(r.x, u / ev) < 1e-12


def check_bsr_grad_fd(ora):
    A = W.elastic3d_bsr(2, 2, 0.3, np.float64)
    D = dense_bsr(A)
    rng = np.random.default_rng(45)
    bvec = rng.uniform(-1, 1, A.n_rows)
    w = rng.uniform(-1, 1, A.n_rows)
    x = np.linalg.solve(D, bvec)
    adj = ora.adjoint_bsr(A, x, w, precond="jacobi", tol=1e-14)
    assert adj.grad.shape == A.val.shape
    for k, r, c in ((0, 0, 1), (3, 1, 0), (int(A.nnzb) - 1, 1, 1)):
        I = int(np.searchsorted(A.row_ptr, k, side="right")) - 1
        i, j = I * A.b + r, int(A.col[k]) * A.b + c
        h = 1e-6 * max(1.0, abs(D[i, j]))
        Dp, Dm = D.copy(), D.copy()
        Dp[i, j] += h
        Dm[i, j] -= h
        fd = (w @ np.linalg.solve(Dp, bvec) - w @ np.linalg.solve(Dm, bvec)) / (2 * h)
        assert abs(adj.grad[k, r, c] - fd) <= 1e-7 * max(1.0, abs(fd)), f"BSR dL/dA block {k} ({r},{c})"


# ------------------------------------------------------------------ fp32-storage mode
def check_store_f32_worked_2x2(ora):
    """A hand-worked case where binary32 storage of q = A p changes the iteration count.

    A = diag(1, 1 + d) with d = 1e-9 (below half an fp32 ulp of 1), b = (1, 1), plain CG,
    tol 1e-12.  fp64: q = (1, 1 + d), alpha = 2 / (2 + d), the residual after one step is
    about d / 2 > tol, and CG ends at step 2 (two distinct eigenvalues).  fp32 storage: q
    rounds to (1, 1), so alpha = 1, r = 0 and the solve ends after ONE step with x = (1, 1)
    exactly."""
    d = 1e-9
    A = csr_from_dense(np.diag([1.0, 1.0 + d]))
    b = np.array([1.0, 1.0])
    r64 = ora.pcg(A, b, precond="none", tol=1e-12)
    r32 = ora.pcg(A, b, precond="none", tol=1e-12, store_f32=True)
    assert r64.status == 0 and r64.iters == 2, (r64.status, r64.iters)
    assert abs(r64.x[1] - 1.0 / (1.0 + d)) <= 1e-15
    assert r32.status == 0 and r32.iters == 1, (r32.status, r32.iters)
    assert r32.x[0] == 1.0 and r32.x[1] == 1.0 and r32.relres == 0.0


def check_store_f32_exact_case(ora):
    """Where every stored vector is exact in binary32 the two modes agree bit for bit:
    Jacobi on a diagonal matrix with power-of-two entries and small-integer b converges in
    one step to x = b / diag, exactly."""
    diag = np.array([1.0, 2.0, 4.0, 8.0, 0.5, 16.0])
    A = csr_from_dense(np.diag(diag))
    b = np.array([3.0, -2.0, 5.0, 1.0, -7.0, 12.0])
    r64 = ora.pcg(A, b, precond="jacobi", tol=1e-12)
    r32 = ora.pcg(A, b, precond="jacobi", tol=1e-12, store_f32=True)
    assert r64.iters == r32.iters == 1
    assert np.array_equal(r32.x, b / diag) and np.array_equal(r64.x, r32.x)


def check_store_f32_rounds_and_tracks(ora):
    """On the power-law SPAI recipe: every iterate the fp32-storage mode returns is a binary32
    value (the fp64 mode's are not), and for the first steps its iterates stay within fp32
    rounding distance of the fp64 recurrence's (the same method, only the storage differs)."""
    w = W.workload(5, "tiny")
    kw = dict(precond="spai", G=w.G, eps=w.eps)
    for k in (1, 2, 3, 5):
        x64 = ora.pcg(w.A, w.B, fixed_iters=k, **kw).x
        x32 = ora.pcg(w.A, w.B, fixed_iters=k, store_f32=True, **kw).x
        assert np.array_equal(x32, x32.astype(np.float32).astype(np.float64))
        assert not np.array_equal(x64, x64.astype(np.float32).astype(np.float64))
        d = np.linalg.norm(x32 - x64) / np.linalg.norm(x64)
        assert 0.0 < d <= 1e-5 * k, (k, d)
    # converged: the same solution to the fp32 tolerance
    a = ora.pcg(w.A, w.B, tol=w.tol, **kw)
    b = ora.pcg(w.A, w.B, tol=w.tol, store_f32=True, **kw)
    assert a.status == b.status == 0
    assert np.linalg.norm(a.x - b.x) / np.linalg.norm(a.x) <= 1e-5


# ------------------------------------------------------------------ eigenvalue gradient
def check_eigen_grad_closed_form(ora):
    """2D Poisson eigenpair in closed form: g_k = v_i v_j for the unit eigenvector, and by
    homogeneity of the eigenvalue in A, sum_k A_k g_k = v^T A v = mu."""
    N = 17
    A = W.poisson2d(N)
    for j, k in ((1, 1), (4, 9), (17, 3)):
        vj, lj = lap_eig_1d(N, j)
        vk, lk = lap_eig_1d(N, k)
        v = np.outer(vj, vk).ravel()
        v /= np.linalg.norm(v)
        g = ora.eigen_grad(A, v)
        rows = A.rows_of_entries()
        assert np.allclose(g, v[rows] * v[A.col.astype(np.int64)], rtol=0, atol=1e-16)
        mu = lj + lk
        assert abs(float(A.val.astype(np.float64) @ g) - mu) <= 1e-12 * mu, "sum A_k g_k = mu"


def check_eigen_grad_fd(ora):
    """Central differences of a simple eigenvalue of a random SPD matrix in single stored
    entries (each perturbation breaks the symmetry; the eigenvalue of the perturbed matrix
    comes from a dense non-symmetric eigensolver)."""
    rng = np.random.default_rng(29)
    A = random_spd(14, 707)
    Ad = dense(A)
    mus, vecs = np.linalg.eigh(Ad)
    m = 6
    assert min(mus[m] - mus[m - 1], mus[m + 1] - mus[m]) > 1e-3
    v = vecs[:, m]
    g = ora.eigen_grad(A, v)
    rows = A.rows_of_entries()
    for kk in rng.choice(A.nnz, size=14, replace=False):
        i, j = int(rows[kk]), int(A.col[kk])
        h = 1e-6
        Ap = Ad.copy(); Ap[i, j] += h
        Am = Ad.copy(); Am[i, j] -= h
        ep = np.linalg.eigvals(Ap); em = np.linalg.eigvals(Am)
        fp = float(np.real(ep[np.argmin(np.abs(ep - mus[m]))]))
        fm = float(np.real(em[np.argmin(np.abs(em - mus[m]))]))
        fd = (fp - fm) / (2 * h)
        assert abs(g[kk] - fd) <= 1e-7, f"d mu / dA[{i},{j}]: {g[kk]} vs {fd}"


# ------------------------------------------------------------------ nonlinear adjoint
def _newton_cubic(Ad, b, iters=60):
    """Solve A u + u^3 = b by dense Newton to machine precision."""
    u = np.linalg.solve(Ad, b)
    for _ in range(iters):
        F = Ad @ u + u ** 3 - b
        du = np.linalg.solve(Ad + np.diag(3 * u ** 2), F)
        u = u - du
        if np.max(np.abs(du)) <= 1e-16 * max(1.0, np.max(np.abs(u))):
            break
    return u


def check_nonlinear_adjoint_fd(ora):
    """F(u) = A u + u^3 - b = 0, L = w.u: the adjoint through J = A + diag(3 u^2) gives
    dL/db = lambda and dL/dA_ij = -lambda_i u_j; central differences of L (dense Newton
    solves) in single stored entries and in b."""
    rng = np.random.default_rng(31)
    A = random_spd(12, 808)
    Ad = dense(A)
    b = rng.uniform(-1, 1, 12)
    w = rng.uniform(-1, 1, 12)
    u = _newton_cubic(Ad, b)
    J = ora.add_diagonal(A, 3 * u ** 2)
    assert np.allclose(dense(J), Ad + np.diag(3 * u ** 2), rtol=0, atol=1e-15)
    res = ora.nonlinear_adjoint(J, A, u, w, precond="jacobi", tol=1e-14)
    assert res.status == 0
    L = lambda Ax, bx: float(w @ _newton_cubic(Ax, bx))
    rows = A.rows_of_entries()
    for kk in rng.choice(A.nnz, size=10, replace=False):
        i, j = int(rows[kk]), int(A.col[kk])
        h = 1e-6
        Ap = Ad.copy(); Ap[i, j] += h
        Am = Ad.copy(); Am[i, j] -= h
        fd = (L(Ap, b) - L(Am, b)) / (2 * h)
        assert abs(res.grad[kk] - fd) <= 1e-7 * max(1.0, abs(fd)), f"dL/dA[{i},{j}]"
    for i in rng.choice(12, size=5, replace=False):
        h = 1e-6
        bp = b.copy(); bp[i] += h
        bm = b.copy(); bm[i] -= h
        fd = (L(Ad, bp) - L(Ad, bm)) / (2 * h)
        assert abs(res.lam[i] - fd) <= 1e-7 * max(1.0, abs(fd)), f"dL/db[{i}]"


ALL_CHECKS = [
    check_spmv_closed_form, check_spmv_dense, check_transpose, check_spai_apply,
    check_pcg_krylov_optimal, check_pcg_eigvec_one_step, check_pcg_m_distinct,
    check_pcg_dense_solve, check_pcg_scaling, check_pcg_status, check_adjoint_identities,
    check_grad_fd, check_grad_fd_symmetric, check_list_blocks,
    check_bsr_spmv_dense, check_bsr_closed_form, check_bsr_grad_fd,
    check_store_f32_worked_2x2, check_store_f32_exact_case, check_store_f32_rounds_and_tracks,
    check_eigen_grad_closed_form, check_eigen_grad_fd, check_nonlinear_adjoint_fd,
]
