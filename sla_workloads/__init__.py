"""Seeded synthetic inputs for the sparse SPD solve: matrices, SPAI factors and right-hand sides.

This module is the one piece shared by the CPU oracle and the CUDA path.  It builds the
inputs only: CSR patterns and values, the synthetic SPAI factor G, right-hand sides and
loss weights.  It holds none of the method's arithmetic (no SpMV, no CG step, no
preconditioner apply, no gradient).

Workload recipes (sizes, value laws and seeds) follow the five synthetic cases that
stand in for the pages' benchmarks:

* 2D Poisson, 5-point stencil, Dirichlet boundary, diagonal 4, off-diagonals -1: the
  model problem of "torch-sla: Differentiable Sparse Linear Algebra with Adjoint Solvers
  and Sparse Tensor Parallelism for PyTorch", Experimental Results (2D Poisson
  benchmarks).
* Implicit heat step A = I + dt*L on a 3D grid, L the unscaled 7-point Laplacian.
* Many small random SPD systems (the distinct-pattern batch of the same page,
  Methodology §1, SparseTensorList).
* A power-law random SPD system (the "Synthetic System" of "Learning Sparse Approximate
  Inverse Preconditioners for Conjugate Gradient Solvers on GPUs", Key results).
* The SPAI factor G with A's lower-triangular pattern (same page, Approach:
  M^-1 = G G^T + eps I, G sharing A's sparsity), here synthetic rather than learned.
* A vector-valued 3D problem stored in 3 x 3 blocks (BSR), standing in for the same page's
  hyperelasticity benchmark; block sparse storage as "Efficient Sparse Matrix Algebra in
  Python for Mathematics" describes it (Key sparse formats and memory tradeoffs).

Random draws use numpy's PCG64 ``default_rng``.  Off-diagonal values of the random SPD
matrices come from the SplitMix64 mixing function (Steele, Lea and Flood, "Fast
Splittable Pseudorandom Number Generators", OOPSLA 2014) applied to the unordered pair
(min(i,j), max(i,j)), so A_ij = A_ji holds by construction without a lookup.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

__all__ = [
    "CSR", "BSR", "Workload", "coupling_block", "elastic3d_bsr", "random_bsr", "splitmix64", "hash_uniform01", "sorted_unique",
    "poisson2d", "heat3d", "random_spd_list", "powerlaw_spd", "spai_factor_G",
    "rhs_uniform", "rhs_normal", "workload", "CONFIG_NAMES",
]


@dataclass
class CSR:
    """Compressed sparse row matrix: int32 row_ptr (n_rows+1), int32 col (nnz), val (nnz)."""
    n_rows: int
    n_cols: int
    row_ptr: np.ndarray
    col: np.ndarray
    val: np.ndarray
    # Block-diagonal "list" of independent systems: row offsets of each system (int64,
    # batch+1).  Column indices stay global, inside the owning system's row range.
    sys_row_off: Optional[np.ndarray] = None

    @property
    def nnz(self) -> int:
        return int(self.row_ptr[-1])

    @property
    def batch(self) -> int:
        return 1 if self.sys_row_off is None else len(self.sys_row_off) - 1

    def rows_of_entries(self) -> np.ndarray:
        return np.repeat(np.arange(self.n_rows, dtype=np.int64), np.diff(self.row_ptr))


@dataclass
class BSR:
    """Block sparse row matrix: a CSR pattern of b x b dense blocks.

    int32 row_ptr (n_brows+1) and col (nnzb) index blocks; val is [nnzb, b, b], each block
    row-major, so scalar entry (I*b + r, col[k]*b + c) is val[k, r, c].
    """
    n_brows: int
    b: int
    row_ptr: np.ndarray
    col: np.ndarray
    val: np.ndarray

    @property
    def n_rows(self) -> int:
        return self.n_brows * self.b

    @property
    def n_cols(self) -> int:
        return self.n_rows

    @property
    def nnzb(self) -> int:
        return int(self.row_ptr[-1])

    @property
    def nnz(self) -> int:
        return self.nnzb * self.b * self.b

    @property
    def batch(self) -> int:
        return 1

    sys_row_off = None


@dataclass
class Workload:
    """One synthetic problem: A, optional SPAI factor G, right-hand sides B and loss weights W.

    B and W are [n][nrhs] row-major (interleaved); nrhs == 1 gives plain vectors.
    """
    name: str
    A: CSR
    B: np.ndarray
    W: np.ndarray
    tol: float
    precond: str                     # "jacobi" or "spai"
    G: Optional[CSR] = None
    eps: float = 0.0
    dtype: type = np.float64
    info: dict = field(default_factory=dict)

    @property
    def nrhs(self) -> int:
        return 1 if self.B.ndim == 1 else self.B.shape[1]


# ----------------------------------------------------------------------------------------
# Counter-based hashing (SplitMix64 finaliser) and helpers
# ----------------------------------------------------------------------------------------
_M64 = np.uint64(0xFFFFFFFFFFFFFFFF)


def splitmix64(x: np.ndarray) -> np.ndarray:
    """SplitMix64 output function applied to counters x (uint64, wrapping arithmetic)."""
    z = np.asarray(x, dtype=np.uint64) + np.uint64(0x9E3779B97F4A7C15)
    z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def hash_uniform01(seed: int, keys: np.ndarray) -> np.ndarray:
    """Uniform doubles in [0, 1): top 53 bits of SplitMix64(seed * 2^48 + key)."""
    ctr = np.asarray(keys, dtype=np.uint64) + (np.uint64(seed) << np.uint64(48))
    return (splitmix64(ctr) >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def sorted_unique(a: np.ndarray) -> np.ndarray:
    """Sorted distinct values of an integer array (sort, then drop repeats)."""
    s = np.sort(a, kind="quicksort")
    if s.size == 0:
        return s
    keep = np.empty(s.size, dtype=bool)
    keep[0] = True
    np.not_equal(s[1:], s[:-1], out=keep[1:])
    return s[keep]


def _csr_from_sorted_keys(keys: np.ndarray, n: int) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """row_ptr, col, row for entries given as sorted distinct keys row*n + col."""
    rows = keys // n
    cols = (keys - rows * n).astype(np.int32)
    counts = np.bincount(rows, minlength=n)
    row_ptr = np.zeros(n + 1, dtype=np.int64)
    np.cumsum(counts, out=row_ptr[1:])
    if row_ptr[-1] >= 2**31:
        raise ValueError("nnz does not fit int32 indices")
    return row_ptr.astype(np.int32), cols, rows


# ----------------------------------------------------------------------------------------
# Stencil matrices
# ----------------------------------------------------------------------------------------
def _stencil_csr(shape: tuple[int, ...], diag: float, off: float, dtype) -> CSR:
    """Constant-coefficient (2*ndim+1)-point stencil on a grid, natural (row-major) order.

    Neighbours outside the grid are dropped (Dirichlet).  Columns in each row ascend.
    """
    dims = len(shape)
    n = int(np.prod(shape))
    idx = np.arange(n, dtype=np.int64)
    coords = np.unravel_index(idx, shape)
    strides = [int(np.prod(shape[d + 1:])) for d in range(dims)]
    # offsets in ascending order: -stride_0 ... -stride_last, 0, +stride_last ... +stride_0
    offs = []
    for d in range(dims):
        offs.append((d, -1))
    offs.append((None, 0))
    for d in reversed(range(dims)):
        offs.append((d, +1))
    # ascending column order needs offsets sorted by value: -s0 < -s1 < ... < 0 < ... < s0
    offs_sorted = sorted(offs, key=lambda t: 0 if t[0] is None else t[1] * strides[t[0]])
    present = []
    cols = []
    for d, s in offs_sorted:
        if d is None:
            present.append(np.ones(n, dtype=bool))
            cols.append(idx)
        else:
            c = coords[d] + s
            ok = (c >= 0) & (c < shape[d])
            present.append(ok)
            cols.append(idx + s * strides[d])
    present = np.stack(present, axis=1)           # [n, 2*dims+1]
    cols = np.stack(cols, axis=1)
    is_diag = np.zeros_like(present)
    is_diag[:, dims] = True
    counts = present.sum(axis=1)
    row_ptr = np.zeros(n + 1, dtype=np.int64)
    np.cumsum(counts, out=row_ptr[1:])
    col = cols[present].astype(np.int32)
    val = np.where(is_diag[present], diag, off).astype(dtype)
    return CSR(n, n, row_ptr.astype(np.int32), col, val)


def poisson2d(N: int, dtype=np.float64) -> CSR:
    """N x N grid, 5-point Laplacian with Dirichlet boundary: diagonal 4, neighbours -1."""
    return _stencil_csr((N, N), 4.0, -1.0, dtype)


def poisson1d(N: int, dtype=np.float64) -> CSR:
    """1D Dirichlet Laplacian tridiag(-1, 2, -1)."""
    return _stencil_csr((N,), 2.0, -1.0, dtype)


def heat3d(N: int, dt: float = 0.1, dtype=np.float32) -> CSR:
    """Implicit heat step A = I + dt*L, L the unscaled 7-point Laplacian (diag 6, off -1)."""
    return _stencil_csr((N, N, N), 1.0 + 6.0 * dt, -dt, dtype)


def coupling_block(b: int) -> np.ndarray:
    """The b x b SPD coupling S = tridiag(1/2, 1, 1/2), eigenvalues 1 + cos(m pi / (b+1))."""
    S = np.eye(b)
    for r in range(b - 1):
        S[r, r + 1] = S[r + 1, r] = 0.5
    return S


def elastic3d_bsr(N: int, b: int = 3, shift: float = 0.1, dtype=np.float32) -> BSR:
    """Vector-valued 3D model problem in b x b blocks: A = L (x) S + shift*I on an N^3 grid.

    L is the unscaled 7-point Dirichlet Laplacian (diagonal 6, neighbours -1), S the SPD
    coupling above, so a node couples its b unknowns to each neighbour's through -S and
    its own through 6 S + shift I -- the block structure of a vector PDE (the pages'
    hyperelasticity benchmark has 3 unknowns per node).  A is SPD: its eigenvalues are
    lambda_L * mu_S + shift.
    """
    P = _stencil_csr((N, N, N), 6.0, -1.0, np.float64)
    S = coupling_block(b)
    rows = P.rows_of_entries()
    val = P.val[:, None, None] * S[None, :, :]
    diag = rows == P.col.astype(np.int64)
    val[diag] += shift * np.eye(b)[None, :, :]
    return BSR(P.n_rows, b, P.row_ptr, P.col, val.astype(dtype))


def random_bsr(n_brows: int, b: int, lens: np.ndarray, seed: int, dtype=np.float32) -> BSR:
    """Unstructured BSR pattern (block row I holds lens[I] distinct block columns, ascending)
    with values U[-1, 1]: SpMV and layout tests, not a solvable system."""
    rng = np.random.default_rng(seed)
    rp = np.zeros(n_brows + 1, dtype=np.int64)
    np.cumsum(lens, out=rp[1:])
    col = np.concatenate([np.sort(rng.choice(n_brows, size=int(l), replace=False)) if l else
                          np.zeros(0, np.int64) for l in lens]).astype(np.int32)
    val = rng.uniform(-1, 1, size=(col.size, b, b)).astype(dtype)
    return BSR(n_brows, b, rp.astype(np.int32), col, val)


# ----------------------------------------------------------------------------------------
# Random SPD matrices
# ----------------------------------------------------------------------------------------
def _spd_values_from_pairs(key_n: int, seed: int, shift: float, dtype,
                           rows_off: np.ndarray, cols_off: np.ndarray, n_rows: int):
    """Off-diagonal values -U[0,1) from the unordered pair hash; diagonal = sum|off| + shift.

    The diagonal is summed (in fp64) from the off-diagonals as stored in ``dtype``, then
    rounded to ``dtype``, so strict diagonal dominance holds for the stored matrix.
    """
    lo = np.minimum(rows_off, cols_off)
    hi = np.maximum(rows_off, cols_off)
    u = hash_uniform01(seed, lo * key_n + hi)
    off_vals = (-u).astype(dtype)
    rowsum = np.bincount(rows_off, weights=np.abs(off_vals.astype(np.float64)), minlength=n_rows)
    diag_vals = (rowsum + shift).astype(dtype)
    return off_vals, diag_vals


def _assemble_symmetric(pair_lo: np.ndarray, pair_hi: np.ndarray, n: int, seed: int,
                        shift: float, dtype, key_n: int | None = None) -> CSR:
    """CSR of the symmetric matrix with the given distinct unordered off-diagonal pairs."""
    key_n = n if key_n is None else key_n
    keys = np.concatenate([pair_lo * n + pair_hi, pair_hi * n + pair_lo,
                           np.arange(n, dtype=np.int64) * (n + 1)])
    keys = np.sort(keys, kind="quicksort")
    row_ptr, col, rows = _csr_from_sorted_keys(keys, n)
    del keys
    cols64 = col.astype(np.int64)
    is_diag = rows == cols64
    off = ~is_diag
    off_vals, diag_vals = _spd_values_from_pairs(key_n, seed, shift, dtype,
                                                 rows[off], cols64[off], n)
    val = np.empty(rows.size, dtype=dtype)
    val[off] = off_vals
    val[is_diag] = diag_vals            # exactly one diagonal per row, in row order
    return CSR(n, n, row_ptr, col, val)


def random_spd_list(nsys: int, n: int, pairs_per_row: float = 7.5, shift: float = 0.1,
                    seed: int = 3, dtype=np.float64) -> CSR:
    """Block-diagonal batch of ``nsys`` independent SPD systems of size n.

    Each system draws round(n*pairs_per_row) unordered pairs {i != j} uniformly, drops
    repeats, mirrors them and adds the diagonal (about 16 stored entries per row for the
    default).  Values: A_ij = A_ji ~ -U[0,1); A_ii = sum_j |A_ij| + shift.  Patterns differ
    between systems.  Column indices are global (system s owns rows/cols
    [s*n, (s+1)*n)).
    """
    rng = np.random.default_rng(seed)
    m = int(round(n * pairs_per_row))
    i = rng.integers(0, n, size=(nsys, m), dtype=np.int64)
    j = rng.integers(0, n - 1, size=(nsys, m), dtype=np.int64)
    j += (j >= i)                                  # uniform over j != i
    lo = np.minimum(i, j)
    hi = np.maximum(i, j)
    sys = np.arange(nsys, dtype=np.int64)[:, None]
    N = nsys * n
    base = sys * n
    pk = sorted_unique(((lo + base) * N + (hi + base)).ravel())
    plo = pk // N
    phi = pk - plo * N
    A = _assemble_symmetric(plo, phi, N, seed, shift, dtype)
    A.sys_row_off = np.arange(nsys + 1, dtype=np.int64) * n
    return A


def _zipf_truncated(rng, n: int, exponent: float, dmin: int, dmax: int) -> np.ndarray:
    """n draws of P(d) ~ d^-exponent restricted to [dmin, dmax] by rejection."""
    out = np.empty(n, dtype=np.int64)
    filled = 0
    while filled < n:
        want = n - filled
        draw = rng.zipf(exponent, size=max(8 * want, 1024))
        ok = draw[(draw >= dmin) & (draw <= dmax)]
        take = min(ok.size, want)
        out[filled:filled + take] = ok[:take]
        filled += take
    return out


def powerlaw_spd(n: int, exponent: float = 2.0, dmin: int = 4, dmax: int = 4096,
                 shift: float = 1e-2, seed: int = 5000, dtype=np.float32) -> CSR:
    """Symmetric SPD matrix with power-law row degrees (load-balance stress case).

    Row i draws d_i ~ Zipf(exponent) truncated to [dmin, dmax] (rejection), then d_i
    distinct neighbours j != i uniformly; the pattern is the union with its transpose plus
    the diagonal.  Values: A_ij = A_ji ~ -U[0,1); A_ii = sum_j |A_ij| + shift.
    """
    rng = np.random.default_rng(seed)
    deg = np.minimum(_zipf_truncated(rng, n, exponent, dmin, dmax), n - 1)
    rows = np.repeat(np.arange(n, dtype=np.int64), deg)
    cols = rng.integers(0, n - 1, size=rows.size, dtype=np.int64)
    cols += (cols >= rows)
    keys = sorted_unique(rows * n + cols)
    del rows, cols
    for _ in range(64):                            # redraw neighbours lost to repeats
        have = np.bincount(keys // n, minlength=n)
        miss = deg - have
        if not miss.any():
            break
        r2 = np.repeat(np.arange(n, dtype=np.int64), miss)
        c2 = rng.integers(0, n - 1, size=r2.size, dtype=np.int64)
        c2 += (c2 >= r2)
        keys = sorted_unique(np.concatenate([keys, r2 * n + c2]))
    r = keys // n
    c = keys - r * n
    del keys
    pk = sorted_unique(np.minimum(r, c) * n + np.maximum(r, c))
    del r, c
    plo = pk // n
    phi = pk - plo * n
    del pk
    A = _assemble_symmetric(plo, phi, n, seed, shift, dtype)
    return A


# ----------------------------------------------------------------------------------------
# Synthetic SPAI factor
# ----------------------------------------------------------------------------------------
def spai_factor_G(A: CSR, seed: int, scale: float = 0.1, dtype=None) -> CSR:
    """G on the lower-triangular pattern of A (diagonal included).

    G_ii = 1/sqrt(A_ii) (fp64, then rounded to dtype); G_ij = u_ij/sqrt(A_ii) for j < i with
    u_ij ~ U[-scale, scale] drawn in CSR order of G's strictly-lower entries.
    """
    dtype = A.val.dtype if dtype is None else dtype
    rows = A.rows_of_entries()
    col = A.col.astype(np.int64)
    keep = col <= rows
    g_rows = rows[keep]
    g_col = A.col[keep]
    diag_mask = col == rows
    a_diag = np.zeros(A.n_rows, dtype=np.float64)
    a_diag[rows[diag_mask]] = A.val[diag_mask].astype(np.float64)
    if np.any(a_diag <= 0):
        raise ValueError("SPAI factor needs a positive diagonal in every row")
    inv_sqrt = 1.0 / np.sqrt(a_diag)
    is_d = g_col.astype(np.int64) == g_rows
    rng = np.random.default_rng(seed)
    u = rng.uniform(-scale, scale, size=int((~is_d).sum()))
    gval = np.empty(g_rows.size, dtype=np.float64)
    gval[is_d] = inv_sqrt[g_rows[is_d]]
    gval[~is_d] = u * inv_sqrt[g_rows[~is_d]]
    counts = np.bincount(g_rows, minlength=A.n_rows)
    rp = np.zeros(A.n_rows + 1, dtype=np.int64)
    np.cumsum(counts, out=rp[1:])
    return CSR(A.n_rows, A.n_cols, rp.astype(np.int32), g_col.astype(np.int32), gval.astype(dtype))


# ----------------------------------------------------------------------------------------
# Right-hand sides
# ----------------------------------------------------------------------------------------
def rhs_uniform(seed: int, shape, lo: float = -1.0, hi: float = 1.0, dtype=np.float64) -> np.ndarray:
    return np.random.default_rng(seed).uniform(lo, hi, size=shape).astype(dtype)


def rhs_normal(seed: int, shape, dtype=np.float64) -> np.ndarray:
    return np.random.default_rng(seed).standard_normal(size=shape).astype(dtype)


# ----------------------------------------------------------------------------------------
# The five synthetic workloads and their scaled-down forms
# ----------------------------------------------------------------------------------------
CONFIG_NAMES = {
    1: "poisson2d_64_f64_jacobi",
    2: "poisson2d_1024_f32_spai",
    3: "heat3d_128_f32_jacobi_8rhs",
    4: "spd_list_4096x1024_f64_jacobi",
    5: "powerlaw_4M_f32_spai",
    6: "elastic3d_128_bsr3_f32_jacobi",
}


def workload(cfg: int, size: str = "full") -> Workload:
    """Build synthetic workload ``cfg`` (1..6; 6 is the block-sparse (BSR) vector problem).

    size="full" gives the stated sizes.  size="small" keeps each recipe (pattern law,
    value law, precision, preconditioner, tolerance, seeds) at a size the fp64 oracle
    finishes in seconds.  size="tiny" is smaller still, for exhaustive CPU checks.
    size="medium" (workload 5 only) is a quarter of the full system -- still larger than
    a GPU's L2 but a few hundred MB on the device -- for profiler captures.
    """
    if size == "medium" and cfg != 5:
        raise ValueError("size 'medium' is defined for workload 5 only")
    small = size not in ("full", "medium")
    tiny = size == "tiny"
    if cfg == 1:
        N = 64 if not tiny else 12
        A = poisson2d(N, np.float64)
        n = A.n_rows
        return Workload(CONFIG_NAMES[1] if not small else f"poisson2d_{N}_f64_jacobi", A,
                        rhs_uniform(0, n, dtype=np.float64), rhs_uniform(1, n, dtype=np.float64),
                        1e-10, "jacobi", dtype=np.float64, info={"grid": N})
    if cfg == 2:
        N = 1024 if not small else (96 if not tiny else 12)
        A = poisson2d(N, np.float32)
        n = A.n_rows
        G = spai_factor_G(A, seed=2, dtype=np.float32)
        return Workload(CONFIG_NAMES[2] if not small else f"poisson2d_{N}_f32_spai", A,
                        rhs_normal(2001, n, np.float32), rhs_uniform(2002, n, dtype=np.float32),
                        1e-6, "spai", G=G, eps=3e-3, dtype=np.float32, info={"grid": N})
    if cfg == 3:
        N = 128 if not small else (20 if not tiny else 6)
        A = heat3d(N, 0.1, np.float32)
        n = A.n_rows
        k = 8
        return Workload(CONFIG_NAMES[3] if not small else f"heat3d_{N}_f32_jacobi_8rhs", A,
                        rhs_uniform(3001, (n, k), 0.0, 1.0, np.float32),
                        rhs_normal(3002, (n, k), np.float32),
                        1e-6, "jacobi", dtype=np.float32, info={"grid": N, "dt": 0.1})
    if cfg == 4:
        nsys, n = (4096, 1024) if not small else ((24, 1024) if not tiny else (5, 40))
        A = random_spd_list(nsys, n, seed=3, dtype=np.float64)
        N = A.n_rows
        return Workload(CONFIG_NAMES[4] if not small else f"spd_list_{nsys}x{n}_f64_jacobi", A,
                        rhs_uniform(4001, N, dtype=np.float64), rhs_uniform(4002, N, dtype=np.float64),
                        1e-10, "jacobi", dtype=np.float64, info={"nsys": nsys, "n": n})
    if cfg == 5:
        n = (4194304 if size == "full" else 1048576) if not small else (49152 if not tiny else 600)
        A = powerlaw_spd(n, seed=5000, dtype=np.float32)
        G = spai_factor_G(A, seed=5003, dtype=np.float32)
        return Workload(CONFIG_NAMES[5] if size == "full" else f"powerlaw_{n}_f32_spai", A,
                        rhs_normal(5001, n, np.float32), rhs_uniform(5002, n, dtype=np.float32),
                        1e-6, "spai", G=G, eps=3e-3, dtype=np.float32, info={"n": n})
    if cfg == 6:
        N = 128 if not small else (16 if not tiny else 5)
        A = elastic3d_bsr(N, 3, 0.1, np.float32)
        n = A.n_rows
        return Workload(CONFIG_NAMES[6] if not small else f"elastic3d_{N}_bsr3_f32_jacobi", A,
                        rhs_normal(6001, n, np.float32), rhs_uniform(6002, n, dtype=np.float32),
                        1e-6, "jacobi", dtype=np.float32, info={"grid": N, "block": 3})
    raise ValueError(f"unknown workload {cfg}")
