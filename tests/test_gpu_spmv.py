"""SpMV parity with the oracle through the C ABI: every workload recipe, multi-RHS blocks,
ragged tiles, long rows, empty rows and degenerate sizes."""
import numpy as np
import pytest

import sla_workloads as W
from gpu_helpers import SPMV_TOL, dev, host, matrix, rel, tol_key

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ora():
    import oracle
    return oracle.get()


def _x(n, k, dtype, seed):
    rng = np.random.default_rng(seed)
    shape = (n,) if k == 1 else (n, k)
    return rng.uniform(-1, 1, size=shape).astype(dtype)


def _ref(ora, A, x):
    if x.ndim == 1:
        return ora.spmv(A, x)
    return np.stack([ora.spmv(A, x[:, c]) for c in range(x.shape[1])], axis=1)


@pytest.mark.parametrize("cfg,size", [(c, s) for c in (1, 2, 3, 4, 5) for s in ("tiny", "small")])
def test_spmv_workloads(ora, cfg, size):
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(cfg, size)
    A = w.A
    Ad = matrix(A)
    x = _x(A.n_rows, 1, w.dtype, 7)
    y = sla.sla_spmv(Ad, dev(x))
    assert rel(host(y), _ref(ora, A, x)) <= SPMV_TOL[tol_key(w.dtype)]


@pytest.mark.parametrize("k", [1, 2, 3, 8, 16])
@pytest.mark.parametrize("cfg", [1, 3, 5])
def test_spmv_multi(ora, cfg, k):
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(cfg, "small")
    A = w.A
    Ad = matrix(A)
    X = _x(A.n_rows, k, w.dtype, 8 + k)
    if k == 1:
        X = X.reshape(-1, 1)
    Y = sla.sla_spmv_multi(Ad, dev(X))
    assert rel(host(Y), _ref(ora, A, X)) <= SPMV_TOL[tol_key(w.dtype)]


def _special(kind, dtype):
    rng = np.random.default_rng(3)
    if kind == "long_rows":       # rows far longer than a tile, plus short rows around them
        n = 9000
        lens = rng.integers(0, 6, size=n)
        lens[[5, 4000, 8999]] = [5000, 2047, 8999]
    elif kind == "empty_rows":
        n = 3001
        lens = rng.integers(0, 4, size=n)
        lens[::7] = 0
    elif kind == "one_row":
        n = 1
        lens = np.array([1])
    elif kind == "dense_row_block":
        n = 700
        lens = np.full(n, 700)
    elif kind == "dense_small":       # fewer rows than a warp's lanes, all long
        n = 20
        lens = np.full(n, 20)
    rp = np.zeros(n + 1, np.int64)
    np.cumsum(lens, out=rp[1:])
    col = np.concatenate([np.sort(rng.choice(n, size=l, replace=False)) if l else np.zeros(0, np.int64)
                          for l in lens]).astype(np.int32)
    val = rng.uniform(-1, 1, size=col.size).astype(dtype)
    return W.CSR(n, n, rp.astype(np.int32), col, val)


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("kind", ["long_rows", "empty_rows", "one_row", "dense_row_block", "dense_small"])
@pytest.mark.parametrize("static", [False, True])
def test_spmv_edge_patterns(ora, kind, dtype, static):
    """static=True: long-row single-vector products run on the column-sorted copy (its
    padding rows, segments smaller than a warp, fixed-point sums for fp32)."""
    import differentiable_sparse_linear_b200 as sla
    A = _special(kind, dtype)
    Ad = (sla.sla_csr_create(dev(A.row_ptr), dev(A.col), dev(A.val), static_values=True) if static
          else matrix(A))
    for k in (1, 4):
        X = _x(A.n_rows, k, dtype, 11)
        if k == 1:
            y = sla.sla_spmv(Ad, dev(X))
        else:
            y = sla.sla_spmv_multi(Ad, dev(X))
        assert rel(host(y), _ref(ora, A, X)) <= SPMV_TOL[tol_key(dtype)], (kind, k)


def test_spmv_empty_matrix():
    import torch
    import differentiable_sparse_linear_b200 as sla
    rp = torch.zeros(1, dtype=torch.int32, device="cuda")
    ci = torch.zeros(0, dtype=torch.int32, device="cuda")
    v = torch.zeros(0, dtype=torch.float64, device="cuda")
    A = sla.sla_csr_create(rp, ci, v)
    y = sla.sla_spmv(A, torch.zeros(0, dtype=torch.float64, device="cuda"))
    assert y.numel() == 0


def test_invalid_patterns_rejected():
    import torch
    import differentiable_sparse_linear_b200 as sla
    def mk(rp, ci):
        return (torch.tensor(rp, dtype=torch.int32, device="cuda"),
                torch.tensor(ci, dtype=torch.int32, device="cuda"),
                torch.ones(len(ci), dtype=torch.float64, device="cuda"))
    for rp, ci in (([0, 2, 1, 3], [0, 1, 2]),          # decreasing row_ptr
                   ([0, 2, 3, 4], [1, 0, 1, 2]),       # unsorted row
                   ([0, 2, 3, 4], [0, 0, 1, 2]),       # duplicate
                   ([0, 1, 2, 3], [0, 1, 3]),          # column out of range
                   ([1, 2, 3, 4], [0, 1, 2])):         # row_ptr[0] != 0
        with pytest.raises(sla.SlaError) as e:
            sla.sla_csr_create(*mk(rp, ci))
        assert e.value.status == sla.SLA_ERR_INVALID_CSR


@pytest.mark.parametrize("k", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("cfg,size", [(1, "small"), (2, "small"), (3, "small"), (2, "tiny"), (5, "small")])
def test_spmv_static_values(ora, cfg, size, k):
    """Handles with SLA_STATIC_VALUES: short rows read the sliced copy (whole-row operand
    accesses when the block is [n][k] with k a power of two), long rows the column-sorted
    copy (one column); a change of the values is picked up after sla_csr_values_changed."""
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(cfg, size)
    A = w.A
    val = dev(A.val)
    As = sla.sla_csr_create(dev(A.row_ptr), dev(A.col), val, static_values=True)
    X = _x(A.n_rows, k, w.dtype, 30 + k)
    Y = sla.sla_spmv(As, dev(X)) if k == 1 else sla.sla_spmv_multi(As, dev(X))
    ref = _ref(ora, A, X)
    assert rel(host(Y), ref) <= SPMV_TOL[tol_key(w.dtype)]
    val.mul_(3.0)
    sla.sla_csr_values_changed(As)
    Y = sla.sla_spmv(As, dev(X)) if k == 1 else sla.sla_spmv_multi(As, dev(X))
    assert rel(host(Y), 3.0 * ref) <= SPMV_TOL[tol_key(w.dtype)]
