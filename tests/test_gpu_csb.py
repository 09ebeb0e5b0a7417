"""The column-sorted segment engine (the long-row SpMV of single-right-hand-side solves) on
patterns made to reach its edge cases: columns 70000 apart inside one segment (chunks cut
early: the in-chunk column offset is 16 bits), a hub row of 3000 entries, empty-neighbour
rows, many segments with a ragged last one, fp32 and fp64.  Lockstep iterates after k
steps, then a converged solve and adjoint, against the oracle."""
import numpy as np
import pytest

import sla_workloads as W
from gpu_helpers import SOL_TOL, dev, host, iters_close, matrix, rel, relmax

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ora():
    import oracle
    return oracle.get()


def _wide_spd(n, dtype):
    rng = np.random.default_rng(91)
    jump = 70001 if n > 140002 else n // 2         # columns further apart than 16 bits reach
    i = np.arange(n - 1, dtype=np.int64)
    lo = [i, i[: n - jump]]                        # chain and a wide jump
    hi = [i + 1, i[: n - jump] + jump]
    hub = 12345
    others = rng.choice(np.setdiff1d(np.arange(n), [hub]), size=3000, replace=False).astype(np.int64)
    lo.append(np.minimum(others, hub))
    hi.append(np.maximum(others, hub))
    a = rng.integers(0, n, 20000)
    b = rng.integers(0, n, 20000)
    keep = a != b
    lo.append(np.minimum(a, b)[keep])
    hi.append(np.maximum(a, b)[keep])
    key = np.unique(np.concatenate(lo) * n + np.concatenate(hi))
    A = W._assemble_symmetric(key // n, key % n, n, 17, 0.5, dtype)
    assert np.diff(A.row_ptr).max() > 3000
    return A


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_csb_lockstep_and_solve(ora, dtype):
    import differentiable_sparse_linear_b200 as sla
    n = 150001
    A = _wide_spd(n, dtype)
    Ad = matrix(A)
    M = sla.sla_precond_jacobi(Ad)
    b = W.rhs_normal(92, n, dtype)
    w = W.rhs_uniform(93, n, dtype=dtype)
    tight = 1e-11 if dtype == np.float64 else 1e-5
    for k in (1, 4, 9):
        x, info = sla.sla_pcg_solve(Ad, M, dev(b), rtol=1e-300, maxit=k, engine="graph")
        assert info.iters == k and info.status == sla.SLA_NOT_CONVERGED
        ref = ora.pcg(A, b, precond="jacobi", fixed_iters=k)
        assert rel(host(x), ref.x) <= tight, (k, rel(host(x), ref.x))
        assert relmax(host(x), ref.x) <= 10 * tight
    tol = 1e-10 if dtype == np.float64 else 1e-6
    x, info = sla.sla_pcg_solve(Ad, M, dev(b), rtol=tol)
    ref = ora.pcg(A, b, precond="jacobi", tol=tol)
    cnt = ora.pcg(A, b, precond="jacobi", tol=tol, store_f32=True) if dtype == np.float32 else ref
    assert info.status == 0 and iters_close(info.iters, cnt.iters), (info.iters, cnt.iters, ref.iters)
    assert rel(host(x), ref.x) <= SOL_TOL[dtype]
    lam, g, ainfo = sla.sla_pcg_adjoint(Ad, M, x, dev(w), rtol=tol)
    adj = ora.adjoint(A, ref.x, w, precond="jacobi", tol=tol)
    assert ainfo.status == 0
    assert rel(host(lam), adj.lam) <= SOL_TOL[dtype] and rel(host(g), adj.grad) <= SOL_TOL[dtype]


def test_csb_values_follow_in_place_changes(ora):
    """The sorted copy's values are gathered from the CSR values at every solve."""
    import differentiable_sparse_linear_b200 as sla
    A = _wide_spd(150001, np.float64)
    val = dev(A.val)
    Ad = sla.sla_csr_create(dev(A.row_ptr), dev(A.col), val)
    M = sla.sla_precond_jacobi(Ad)
    b = W.rhs_normal(94, A.n_rows, np.float64)
    x1, _ = sla.sla_pcg_solve(Ad, M, dev(b), rtol=1e-10)
    val.mul_(2.0)                                    # A -> 2A in place: x -> x / 2
    M.refresh()
    x2, _ = sla.sla_pcg_solve(Ad, M, dev(b), rtol=1e-10)
    assert rel(host(x2), host(x1) / 2.0) <= 1e-8


@pytest.mark.parametrize("cfg,size", [(5, "small"), (5, "tiny")])
def test_static_values_spmv(ora, cfg, size):
    """sla_spmv of a SLA_STATIC_VALUES handle reads the column-sorted value copy; after the
    values change in place, sla_csr_values_changed makes the next product use the new ones."""
    import differentiable_sparse_linear_b200 as sla
    from gpu_helpers import SPMV_TOL
    w = W.workload(cfg, size)
    A = w.A
    val = dev(A.val)
    As = sla.sla_csr_create(dev(A.row_ptr), dev(A.col), val, static_values=True)
    Ad = sla.sla_csr_create(dev(A.row_ptr), dev(A.col), val)
    x = W.rhs_normal(95, A.n_rows, w.dtype)
    ref = ora.spmv(A, x)
    ys = host(sla.sla_spmv(As, dev(x)))
    yd = host(sla.sla_spmv(Ad, dev(x)))
    assert rel(ys, ref) <= SPMV_TOL[w.dtype] and rel(yd, ref) <= SPMV_TOL[w.dtype]
    val.mul_(-0.5)
    sla.sla_csr_values_changed(As)
    ys2 = host(sla.sla_spmv(As, dev(x)))
    assert rel(ys2, -0.5 * ref) <= SPMV_TOL[w.dtype]


def _fx_slack(A, x):
    """2^-50 of max_i sum_j |a_ij| x max_j |x_j|: the fixed-point sums round every term once,
    to 2^-63 of their segment's bound (largest row sum of |a_ij| times max |x_j|), so a row
    of m <= 8192 terms is off by at most 2^-50 of it."""
    rows = np.add.reduceat(np.abs(A.val.astype(np.float64)), A.row_ptr[:-1]) * (np.diff(A.row_ptr) > 0)
    return 2.0 ** -50 * float(rows.max()) * float(np.max(np.abs(x.astype(np.float64))))


def test_fixed_point_sums_reproducible_and_rounded(ora):
    """fp32 products of the segment engine sum exact integers on a per-segment scale: two
    launches give identical bits, and each row is the fp64 row sum rounded to fp32 up to an
    error far below the fp32 rounding of a typical row."""
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(5, "small")
    A = w.A
    As = sla.sla_csr_create(dev(A.row_ptr), dev(A.col), dev(A.val), static_values=True)
    x = W.rhs_normal(96, A.n_rows, np.float32)
    y1 = host(sla.sla_spmv(As, dev(x)))
    y2 = host(sla.sla_spmv(As, dev(x)))
    assert np.array_equal(y1.view(np.uint32), y2.view(np.uint32))
    ref = ora.spmv(A, x)
    ulp = np.spacing(np.abs(ref.astype(np.float32))).astype(np.float64)
    err = np.abs(y1.astype(np.float64) - ref)
    assert np.all(err <= 0.5 * ulp + _fx_slack(A, x))


def test_fixed_point_wide_range(ora):
    """Operands spanning the fp32 range (1e-30 .. 1e30): no term or word overflows, every
    row stays finite, and rows are exact to 2^-50 of the largest |A||x| scale."""
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(5, "tiny")
    A = w.A
    As = sla.sla_csr_create(dev(A.row_ptr), dev(A.col), dev(A.val), static_values=True)
    rng = np.random.default_rng(97)
    x = (rng.standard_normal(A.n_rows) * 10.0 ** rng.uniform(-30, 30, A.n_rows)).astype(np.float32)
    y = host(sla.sla_spmv(As, dev(x))).astype(np.float64)
    ref = ora.spmv(A, x)
    ulp = np.spacing(np.abs(ref.astype(np.float32))).astype(np.float64)
    assert np.all(np.isfinite(y))
    assert np.all(np.abs(y - ref) <= 0.5 * ulp + _fx_slack(A, x))


@pytest.mark.parametrize("bad", [np.nan, np.inf])
def test_nonfinite_operand_reaches_the_result(ora, bad):
    """A NaN or Inf in the operand makes the fixed-point bound unusable: the product falls
    back to fp64 sums, so the rows that read it are not finite and the others are exact."""
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(5, "tiny")
    A = w.A
    As = sla.sla_csr_create(dev(A.row_ptr), dev(A.col), dev(A.val), static_values=True)
    x = W.rhs_normal(98, A.n_rows, np.float32)
    j = A.n_rows // 3
    x[j] = bad
    y = host(sla.sla_spmv(As, dev(x)))
    reads = np.zeros(A.n_rows, bool)
    rows = np.repeat(np.arange(A.n_rows), np.diff(A.row_ptr))
    reads[rows[A.col == j]] = True
    assert reads.any() and not np.isfinite(y[reads]).any()
    xs = x.copy()
    xs[j] = 0.0
    ref = ora.spmv(A, xs)
    assert rel(y[~reads], ref[~reads]) <= 1e-6


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_csb_small_dense_solve(ora, dtype):
    """A dense 20 x 20 SPD system: every row is long, so the solve runs on the column-sorted
    copy with one segment per row group smaller than a warp (padding rows fall back to row
    0); lockstep iterates and the converged solve against the oracle."""
    import differentiable_sparse_linear_b200 as sla
    rng = np.random.default_rng(99)
    n = 20
    B = rng.standard_normal((n, n))
    D = B @ B.T + n * np.eye(n)
    rp = np.arange(0, n * n + 1, n, dtype=np.int32)
    col = np.tile(np.arange(n, dtype=np.int32), n)
    A = W.CSR(n, n, rp, col, D.ravel().astype(dtype))
    Ad = matrix(A)
    M = sla.sla_precond_jacobi(Ad)
    b = rng.standard_normal(n).astype(dtype)
    tight = 1e-11 if dtype == np.float64 else 1e-5
    for k in (1, 3):
        x, info = sla.sla_pcg_solve(Ad, M, dev(b), rtol=1e-300, maxit=k, engine="graph")
        ref = ora.pcg(A, b, precond="jacobi", fixed_iters=k)
        assert info.iters == k and rel(host(x), ref.x) <= tight, (k, rel(host(x), ref.x))
    tol = 1e-10 if dtype == np.float64 else 1e-6
    x, info = sla.sla_pcg_solve(Ad, M, dev(b), rtol=tol, engine="graph")
    ref = ora.pcg(A, b, precond="jacobi", tol=tol)
    assert info.status == 0 and rel(host(x), ref.x) <= SOL_TOL[dtype]
