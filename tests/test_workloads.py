"""The seeded synthetic inputs: sizes, symmetry, dominance and the SPAI factor's structure."""
import numpy as np
import pytest

import sla_workloads as W
from oracle_checks import dense


def test_stencil_sizes_match_closed_counts():
    # 5-point on N x N: 5N^2 - 4N entries; 7-point on N^3: 7N^3 - 6N^2
    for N in (3, 7, 64):
        assert W.poisson2d(N).nnz == 5 * N * N - 4 * N
    assert W.poisson2d(64).nnz == 20224
    for N in (3, 10):
        assert W.heat3d(N).nnz == 7 * N ** 3 - 6 * N ** 2


def test_poisson_values_and_order():
    A = W.poisson2d(5)
    D = dense(A)
    assert np.allclose(np.diag(D), 4.0)
    assert np.array_equal(D, D.T)
    off = D - np.diag(np.diag(D))
    assert set(np.unique(off)) <= {0.0, -1.0}
    for i in range(A.n_rows):
        seg = A.col[A.row_ptr[i]:A.row_ptr[i + 1]]
        assert np.all(np.diff(seg) > 0)


def test_heat_diagonal():
    A = W.heat3d(4, 0.1, np.float64)
    D = dense(A)
    assert np.allclose(np.diag(D), 1.6) and np.array_equal(D, D.T)
    assert set(np.unique(D - np.diag(np.diag(D)))) <= {0.0, -0.1}


@pytest.mark.parametrize("make", [
    lambda: W.random_spd_list(3, 50, seed=5),
    lambda: W.powerlaw_spd(400, seed=6, dtype=np.float32),
])
def test_random_spd_symmetric_dominant(make):
    A = make()
    D = dense(A)
    assert np.array_equal(D, D.T)
    d = np.diag(D)
    off = np.abs(D).sum(axis=1) - np.abs(d)
    assert np.all(d > off), "strict diagonal dominance of the stored matrix"
    assert np.all(D - np.diag(d) <= 0)
    for i in range(A.n_rows):
        seg = A.col[A.row_ptr[i]:A.row_ptr[i + 1]]
        assert np.all(np.diff(seg) > 0), "ascending, no duplicates"


def test_list_blocks_are_diagonal():
    A = W.random_spd_list(4, 30, seed=7)
    D = dense(A)
    for s in range(4):
        lo, hi = s * 30, (s + 1) * 30
        D[lo:hi, lo:hi] = 0
    assert not D.any(), "no entry outside the diagonal blocks"
    assert list(A.sys_row_off) == [0, 30, 60, 90, 120]


def test_powerlaw_degree_law():
    A = W.powerlaw_spd(20000, seed=8)
    deg = np.diff(A.row_ptr)
    assert deg.min() >= 5 and deg.max() <= 4096 + 1 + deg.max()  # drawn degree >= 4, plus diagonal
    assert 40 < deg.mean() < 60, "literal recipe gives about 51 stored entries per row"
    assert deg.max() > 1000, "heavy rows present"


def test_spai_factor_structure():
    A = W.poisson2d(6, np.float32)
    G = W.spai_factor_G(A, seed=2)
    Gd = dense(G)
    assert np.array_equal(Gd, np.tril(Gd))
    assert np.allclose(np.diag(Gd), (1.0 / np.sqrt(4.0)), rtol=1e-7)
    strict = Gd[np.tril_indices(36, -1)]
    pattern = dense(A)[np.tril_indices(36, -1)] != 0
    assert np.all(strict[~pattern] == 0)
    assert np.all(np.abs(strict[pattern]) <= 0.1 / 2.0 + 1e-7)
    assert G.val.dtype == np.float32


def test_determinism():
    a = W.workload(5, "tiny")
    b = W.workload(5, "tiny")
    assert np.array_equal(a.A.col, b.A.col) and np.array_equal(a.A.val, b.A.val)
    assert np.array_equal(a.G.val, b.G.val) and np.array_equal(a.B, b.B)


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5, 6])
def test_workload_recipes_small(cfg):
    w = W.workload(cfg, "small")
    assert w.A.val.dtype == w.dtype
    assert w.B.dtype == w.dtype and w.W.dtype == w.dtype
    assert w.B.shape[0] == w.A.n_rows
    assert (w.G is not None) == (w.precond == "spai")
    if cfg == 3:
        assert w.B.shape == (w.A.n_rows, 8)


@pytest.mark.parametrize("b", [2, 3, 4])
def test_elastic_bsr_structure(b):
    """The block vector problem: 7-point block pattern (7N^3 - 6N^2 blocks), symmetric, SPD,
    row-major blocks with -S off the diagonal and 6 S + shift I on it."""
    from oracle_checks import dense_bsr
    N = 4
    A = W.elastic3d_bsr(N, b, 0.1, np.float64)
    assert A.n_rows == N ** 3 * b and A.nnzb == 7 * N ** 3 - 6 * N ** 2
    assert np.all(np.diff(A.row_ptr) >= 4)
    for I in range(A.n_brows):
        cols = A.col[A.row_ptr[I]:A.row_ptr[I + 1]]
        assert np.all(np.diff(cols) > 0) and I in cols
    S = W.coupling_block(b)
    rows = np.repeat(np.arange(A.n_brows), np.diff(A.row_ptr))
    diag = rows == A.col
    assert np.allclose(A.val[~diag], -S) and np.allclose(A.val[diag], 6 * S + 0.1 * np.eye(b))
    D = dense_bsr(A)
    assert np.array_equal(D, D.T)
    assert np.linalg.eigvalsh(D).min() > 0


def test_random_bsr_lengths():
    lens = np.array([0, 3, 1, 0, 6, 2])
    A = W.random_bsr(6, 3, lens, 9, np.float32)
    assert np.array_equal(np.diff(A.row_ptr), lens) and A.val.shape == (lens.sum(), 3, 3)
    for I in range(6):
        cols = A.col[A.row_ptr[I]:A.row_ptr[I + 1]]
        assert np.all(np.diff(cols) > 0) and np.all((cols >= 0) & (cols < 6))


def test_bench_stream_bytes():
    """bench.py's matrix-stream byte count: CSR values + indices + row pointers; BSR one index
    and b*b values per block + block row pointers."""
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    A = W.elastic3d_bsr(5, 3, 0.1, np.float32)
    assert bench.stream_bytes(A, 4) == A.nnzb * (9 * 4 + 4) + (A.n_brows + 1) * 4
    C = W.poisson2d(9, np.float32)
    assert bench.stream_bytes(C, 4) == C.nnz * 8 + (C.n_rows + 1) * 4
