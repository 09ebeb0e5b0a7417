/*
 * fp64 CPU oracle for the preconditioned conjugate-gradient solve of a sparse SPD system
 * and its adjoint.  TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
 * benchmark's CPU-baseline leg call it; the CUDA library never does, and the two share no
 * code.  Everything here is plain, sequential fp64 arithmetic in the order the method's
 * definition gives; no blocking, fusion or reordering.
 *
 * Sources (page title, section):
 *  [TS]   "torch-sla: Differentiable Sparse Linear Algebra with Adjoint Solvers and Sparse
 *         Tensor Parallelism for PyTorch" -- Methodology §1 (the PyTorch-native iterative
 *         backend, Jacobi preconditioned; limitations paragraph), Methodology §2 "Linear
 *         Systems" (adjoint: solve A^T lambda = dL/dx, gradient -lambda_i x_j on the pattern).
 *  [SPAI] "Learning Sparse Approximate Inverse Preconditioners for Conjugate Gradient
 *         Solvers on GPUs" -- Approach (M^-1 = G G^T + eps I, G on A's pattern, two SpMVs
 *         per CG step) and the epsilon ablation (default eps = 3e-3).
 *
 * Readings where the pages are silent (listed with the design notes):
 *  - x0 = 0; the stopping test is ||r_k||_2 / ||b||_2 <= tol on the recursively updated
 *    residual, taken right after the x/r update; the iteration count is the number of
 *    products q = A p in the loop.
 *  - The PCG recurrence is the standard Hestenes-Stiefel form.
 *  - Breakdown: p.q <= 0 or not finite, or r.z <= 0 or not finite for a residual that has
 *    not met the tolerance (A or M not SPD).
 *  - Every pin of these functions lives in the tests; none is "parity unpinned".
 *
 * Threads: build.py also compiles this same source with OpenMP (liboracle_omp.so), used
 * only to time the CPU baseline on every host core.  The pragmas below split loops whose
 * iterations are independent (rows of a product, elements of a vector update) over
 * threads; dot products and norms stay sequential, so both builds give identical bits.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORA_CONVERGED 0
#define ORA_NOT_CONVERGED 1
#define ORA_BREAKDOWN 2

/* y = A x: for each row, the sum over its stored entries of A_ij * x_j, in storage order. */
void ora_spmv(int64_t n_rows, const int32_t *row_ptr, const int32_t *col, const double *val,
              const double *x, double *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n_rows; ++i) {
        double s = 0.0;
        for (int64_t k = row_ptr[i]; k < row_ptr[i + 1]; ++k)
            s += val[k] * x[col[k]];
        y[i] = s;
    }
}

/* Inner product, summed left to right. */
double ora_dot(int64_t n, const double *a, const double *b)
{
    double s = 0.0;
    for (int64_t i = 0; i < n; ++i)
        s += a[i] * b[i];
    return s;
}

/* CSR of A^T (n_cols rows): count the entries of each column, prefix-sum the counts,
 * then drop every entry (i, j, v) into row j of the transpose in increasing i. */
int ora_transpose(int64_t n_rows, int64_t n_cols, const int32_t *rp, const int32_t *ci,
                  const double *v, int32_t *rpT, int32_t *ciT, double *vT)
{
    int64_t nnz = rp[n_rows];
    int64_t *fill = (int64_t *)calloc((size_t)n_cols + 1, sizeof(int64_t));
    if (!fill)
        return -1;
    for (int64_t k = 0; k < nnz; ++k)
        fill[ci[k] + 1] += 1;
    for (int64_t j = 0; j < n_cols; ++j)
        fill[j + 1] += fill[j];
    for (int64_t j = 0; j <= n_cols; ++j)
        rpT[j] = (int32_t)fill[j];
    for (int64_t i = 0; i < n_rows; ++i)
        for (int64_t k = rp[i]; k < rp[i + 1]; ++k) {
            int64_t dst = fill[ci[k]]++;
            ciT[dst] = (int32_t)i;
            vT[dst] = v[k];
        }
    free(fill);
    return 0;
}

/* diag[i] = A_ii; returns -1 if a row stores no diagonal entry, 0 otherwise. */
int ora_diagonal(int64_t n, const int32_t *rp, const int32_t *ci, const double *v, double *diag)
{
    for (int64_t i = 0; i < n; ++i) {
        int found = 0;
        diag[i] = 0.0;
        for (int64_t k = rp[i]; k < rp[i + 1]; ++k)
            if (ci[k] == i) {
                diag[i] = v[k];
                found = 1;
            }
        if (!found)
            return -1;
    }
    return 0;
}

/* Preconditioner z = M^-1 r.
 *  kind 0: identity (plain CG).
 *  kind 1: Jacobi, z_i = r_i / A_ii  ([TS] Methodology §1: the native backend's Jacobi
 *          preconditioning).
 *  kind 2: SPAI, z = G (G^T r) + eps r  ([SPAI] Approach), G^T held as its own CSR. */
typedef struct {
    int32_t kind;
    int32_t pad;
    const double *diag;
    const int32_t *g_rp;
    const int32_t *g_ci;
    const double *g_v;
    const int32_t *gt_rp;
    const int32_t *gt_ci;
    const double *gt_v;
    double eps;
} ora_precond;

/* Round every entry of v to the nearest binary32 value (kept in a double).  Used only by
 * the fp32-storage mode of the solve below. */
static void ora_round_f32(int64_t n, double *v)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        v[i] = (double)(float)v[i];
}

static void precond_apply(int64_t n, const ora_precond *M, const double *r, double *z, double *work,
                          int store_f32)
{
    if (M == NULL || M->kind == 0) {
        for (int64_t i = 0; i < n; ++i)
            z[i] = r[i];
    } else if (M->kind == 1) {
#pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < n; ++i)
            z[i] = r[i] / M->diag[i];
    } else {
        ora_spmv(n, M->gt_rp, M->gt_ci, M->gt_v, r, work);   /* y = G^T r */
        if (store_f32)
            ora_round_f32(n, work);
        ora_spmv(n, M->g_rp, M->g_ci, M->g_v, work, z);      /* z = G y   */
#pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < n; ++i)
            z[i] = z[i] + M->eps * r[i];                     /* + eps r   */
    }
    if (store_f32)
        ora_round_f32(n, z);
}

void ora_precond_apply(int64_t n, const ora_precond *M, const double *r, double *z, double *work)
{
    precond_apply(n, M, r, z, work, 0);
}

static int ora_finite(double a) { return a == a && a - a == 0.0; }

/* Preconditioned CG for A x = b from x0 = 0 ([TS] Methodology §1; [SPAI] Approach).
 *
 *   r = b, z = M^-1 r, p = z, rho = r.z
 *   repeat:  q = A p;  alpha = rho / (p.q);  x += alpha p;  r -= alpha q;
 *            stop if ||r|| / ||b|| <= tol;
 *            z = M^-1 r;  rho' = r.z;  beta = rho'/rho;  p = z + beta p;  rho = rho'
 *
 * fixed_iters > 0 runs exactly that many iterations and ignores tol (lockstep checks).
 * hist (optional, maxit+1 or fixed_iters+1 doubles) receives ||r_k||/||b|| for k = 0.. .
 * Returns ORA_CONVERGED, ORA_NOT_CONVERGED or ORA_BREAKDOWN; *iters and *relres report
 * the last iteration and its relative recursive residual.
 *
 * store_f32 != 0 is the same recurrence with single-precision vector storage: every vector
 * the iteration keeps (q, x, r, the SPAI intermediate y = G^T r, z and p) is rounded to the
 * nearest binary32 value right after it is formed in fp64; dot products, norms and the
 * scalars stay fp64.  It is the arithmetic of a solver that stores its vectors in fp32 with
 * fp64 reductions, so the stopping decision (an integer: the iteration count) can be taken
 * in that storage precision too. */
int ora_pcg_ex(int64_t n, const int32_t *rp, const int32_t *ci, const double *v,
               const ora_precond *M, const double *b, double *x, double tol, int64_t maxit,
               int64_t fixed_iters, int32_t store_f32, int64_t *iters, double *relres, double *hist)
{
    double *r = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double *z = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double *p = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double *q = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double *w = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    int status = ORA_NOT_CONVERGED;
    int64_t k = 0;
    int64_t limit = fixed_iters > 0 ? fixed_iters : maxit;
    double bnorm, rnorm, rho, rho_new, pq, alpha, beta;

    for (int64_t i = 0; i < n; ++i) {
        x[i] = 0.0;
        r[i] = b[i];
    }
    if (store_f32)
        ora_round_f32(n, r);
    bnorm = sqrt(ora_dot(n, r, r));
    *relres = 0.0;
    if (hist)
        hist[0] = bnorm > 0.0 ? 1.0 : 0.0;
    if (bnorm == 0.0) {
        status = ORA_CONVERGED;
        goto done;
    }
    *relres = 1.0;
    precond_apply(n, M, r, z, w, store_f32);
    for (int64_t i = 0; i < n; ++i)
        p[i] = z[i];
    rho = ora_dot(n, r, z);
    if (!(rho > 0.0) || !ora_finite(rho)) {
        status = ORA_BREAKDOWN;
        goto done;
    }
    while (k < limit) {
        k += 1;
        ora_spmv(n, rp, ci, v, p, q);
        if (store_f32)
            ora_round_f32(n, q);
        pq = ora_dot(n, p, q);
        if (!(pq > 0.0) || !ora_finite(pq)) {
            status = ORA_BREAKDOWN;
            break;
        }
        alpha = rho / pq;
#pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < n; ++i) {
            x[i] = x[i] + alpha * p[i];
            r[i] = r[i] - alpha * q[i];
        }
        if (store_f32) {
            ora_round_f32(n, x);
            ora_round_f32(n, r);
        }
        rnorm = sqrt(ora_dot(n, r, r));
        *relres = rnorm / bnorm;
        if (hist)
            hist[k] = *relres;
        if (fixed_iters <= 0 && *relres <= tol) {
            status = ORA_CONVERGED;
            break;
        }
        if (fixed_iters > 0 && k == fixed_iters) {
            status = ORA_CONVERGED;
            break;
        }
        precond_apply(n, M, r, z, w, store_f32);
        rho_new = ora_dot(n, r, z);
        if (!(rho_new > 0.0) || !ora_finite(rho_new)) {
            status = ORA_BREAKDOWN;
            break;
        }
        beta = rho_new / rho;
#pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < n; ++i)
            p[i] = z[i] + beta * p[i];
        if (store_f32)
            ora_round_f32(n, p);
        rho = rho_new;
    }
done:
    *iters = k;
    free(r);
    free(z);
    free(p);
    free(q);
    free(w);
    return status;
}

/* The fp64 solve (no rounding of the stored vectors). */
int ora_pcg(int64_t n, const int32_t *rp, const int32_t *ci, const double *v,
            const ora_precond *M, const double *b, double *x, double tol, int64_t maxit,
            int64_t fixed_iters, int64_t *iters, double *relres, double *hist)
{
    return ora_pcg_ex(n, rp, ci, v, M, b, x, tol, maxit, fixed_iters, 0, iters, relres, hist);
}

/* Gradient of L with respect to the stored entries of A ([TS] Methodology §2, Linear
 * Systems): for every stored (i, j), dL/dA_ij = -lambda_i * x_j, where A^T lambda = dL/dx.
 * g is aligned with A's value array. */
void ora_pattern_grad(int64_t n_rows, const int32_t *rp, const int32_t *ci, const double *lam,
                      const double *x, double *g)
{
    for (int64_t i = 0; i < n_rows; ++i)
        for (int64_t k = rp[i]; k < rp[i + 1]; ++k)
            g[k] = -lam[i] * x[ci[k]];
}

/* Eigenvalue gradient ([TS] Methodology §2, Eigenvalue Problems, Hellmann-Feynman): for a
 * simple eigenvalue mu of a symmetric A with unit eigenvector v, d mu / d A_ij = v_i v_j,
 * evaluated on every stored (i, j); g is aligned with A's value array. */
void ora_eigen_grad(int64_t n_rows, const int32_t *rp, const int32_t *ci, const double *v, double *g)
{
    for (int64_t i = 0; i < n_rows; ++i)
        for (int64_t k = rp[i]; k < rp[i + 1]; ++k)
            g[k] = v[i] * v[ci[k]];
}

/* out = the values of A + diag(c) on A's pattern (the Jacobian A + diag(N'(u)) of
 * F(u) = A u + N(u) - b, [TS] Methodology §2, Nonlinear Systems).  Returns -1 if a row stores
 * no diagonal entry. */
int ora_add_diagonal(int64_t n_rows, const int32_t *rp, const int32_t *ci, const double *v,
                     const double *c, double *out)
{
    for (int64_t i = 0; i < n_rows; ++i) {
        int found = 0;
        for (int64_t k = rp[i]; k < rp[i + 1]; ++k) {
            out[k] = v[k];
            if (ci[k] == i) {
                out[k] = v[k] + c[i];
                found = 1;
            }
        }
        if (!found)
            return -1;
    }
    return 0;
}

/* Block sparse row (BSR) storage -- [SM] "Efficient Sparse Matrix Algebra in Python for
 * Mathematics", "Key sparse formats and memory tradeoffs" (block sparse layouts store
 * dense blocks) and "Block sparse patterns and sharding strategies" (one index per block).
 * The matrix is a CSR pattern of b x b dense blocks: block row I holds blocks
 * k = rp[I] .. rp[I+1]-1 in block columns ci[k], and block k keeps its b*b values row-major
 * at val[k*b*b].  Scalar entry (I*b + r, ci[k]*b + c) is val[k*b*b + r*b + c].
 *
 * y = A x: scalar row I*b + r is the sum, over the blocks of block row I in storage order
 * and over c = 0 .. b-1, of val[k*b*b + r*b + c] * x[ci[k]*b + c]. */
void ora_bsr_spmv(int64_t n_brows, int32_t b, const int32_t *rp, const int32_t *ci, const double *val,
                  const double *x, double *y)
{
    for (int64_t I = 0; I < n_brows; ++I)
        for (int32_t r = 0; r < b; ++r) {
            double s = 0.0;
            for (int64_t k = rp[I]; k < rp[I + 1]; ++k)
                for (int32_t c = 0; c < b; ++c)
                    s += val[k * b * b + (int64_t)r * b + c] * x[(int64_t)ci[k] * b + c];
            y[I * b + r] = s;
        }
}

/* The same matrix as scalar CSR: scalar row I*b + r lists, for each block k of block row I
 * in storage order, the b entries (r, c) -- ascending columns when the block columns are
 * ascending.  pos[e] is the BSR value position of CSR entry e, so a result on the CSR
 * pattern maps back to BSR order by g_bsr[pos[e]] = g_csr[e]. */
void ora_bsr_to_csr(int64_t n_brows, int32_t b, const int32_t *rp, const int32_t *ci, const double *val,
                    int32_t *out_rp, int32_t *out_ci, double *out_val, int64_t *pos)
{
    int64_t e = 0;
    out_rp[0] = 0;
    for (int64_t I = 0; I < n_brows; ++I)
        for (int32_t r = 0; r < b; ++r) {
            for (int64_t k = rp[I]; k < rp[I + 1]; ++k)
                for (int32_t c = 0; c < b; ++c) {
                    const int64_t p = k * b * b + (int64_t)r * b + c;
                    out_ci[e] = (int32_t)((int64_t)ci[k] * b + c);
                    out_val[e] = val[p];
                    pos[e] = p;
                    ++e;
                }
            out_rp[I * b + r + 1] = (int32_t)e;
        }
}
