// PCG forward/adjoint on one B200: fused SpMV + vector-update kernels, device-side
// convergence, and the whole loop as one CUDA graph with a conditional WHILE node.
//
// Method ("torch-sla: Differentiable Sparse Linear Algebra with Adjoint Solvers and Sparse
// Tensor Parallelism for PyTorch", Methodology §1 native Jacobi-preconditioned CG and §2
// adjoint; "Learning Sparse Approximate Inverse Preconditioners for Conjugate Gradient
// Solvers on GPUs", Approach: M^-1 = G G^T + eps I):
//
//   r = b, z = M^-1 r, p = z, rho = r.z
//   loop: q = A p; alpha = rho/(p.q); x += alpha p; r -= alpha q; stop if ||r||/||b|| <= tol
//         z = M^-1 r; rho' = r.z; beta = rho'/rho; p = z + beta p; rho = rho'
//
// Kernel schedule of one iteration (each kernel streams one CSR matrix at most):
//   Q   : p_new = z + beta p_old (own rows) and q = A p_new, p_new.q      [A]
//         (the gathered operand z_j + beta p_old_j is formed on the fly, so p is never
//          written and re-read in a separate pass; p is double-buffered)
//   Jacobi  U_J : x += alpha p; r -= alpha q; z = D^-1 r; r.r and r.z    [elementwise]
//   SPAI    U_S : r_new = r_old - alpha q (own rows and gathered), x += alpha p,
//                 y = G^T r_new, r_new.r_new                             [G^T]
//           Z   : z = G y + eps r_new, r_new.z                           [G]
// Each kernel's last block reduces the dot products (fp64, fixed order) and updates the
// scalars in PcgState: alpha after Q, the stopping test after U, beta after U_J / Z.
// When every right-hand side has stopped it clears the graph's loop condition.
//
// Matrix values (VM) and vectors (VV) may differ: fp32 values with fp64 vectors is the
// mixed-precision mode.  Products and sums are always formed in fp64.
#include <cuda_runtime.h>

#include <algorithm>

#include "sla_internal.cuh"

namespace sla {

// ------------------------------------------------------------------ set-up kernels
// Pattern check of every row: columns inside [lo, hi) of the row's system, strictly ascending.
__global__ void k_validate(int64_t n, const int32_t *rp, const int32_t *ci, const int64_t *sys_off,
                           int batch, int *err)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        int64_t lo = 0, hi = n;
        if (sys_off) {
            int a = 0, b = batch - 1;
            while (a < b) {  // last system whose start <= i
                const int mid = (a + b + 1) >> 1;
                if (sys_off[mid] <= i)
                    a = mid;
                else
                    b = mid - 1;
            }
            lo = sys_off[a];
            hi = sys_off[a + 1];
        }
        int prev = -1;
        for (int64_t k = rp[i]; k < rp[i + 1]; ++k) {
            const int j = ci[k];
            if (j < lo || j >= hi || j <= prev) {
                atomicOr(err, 1);
                break;
            }
            prev = j;
        }
    }
}


// D^-1 of A in fp64 and, for fp32 matrices, in fp32; a missing or non-positive diagonal
// sets *err.
template <typename VM>
__global__ void k_jacobi_dinv(int64_t n, const int32_t *rp, const int32_t *ci, const VM *val,
                              double *dinv64, float *dinv32, int *err)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        double d = 0.0;
        for (int64_t k = rp[i]; k < rp[i + 1]; ++k)
            if (ci[k] == i)
                d = (double)val[k];
        const double inv = d > 0.0 ? 1.0 / d : 0.0;
        if (!(d > 0.0))
            atomicOr(err, 1);
        dinv64[i] = inv;
        if (dinv32)
            dinv32[i] = (float)inv;
    }
}

// The same for a BSR matrix: the diagonal entries of scalar rows I*b .. I*b + b-1 sit on the
// diagonal of block row I's diagonal block.
template <typename VM>
__global__ void k_bsr_dinv(int64_t nbr, int b, const int32_t *rp, const int32_t *ci, const VM *val,
                           double *dinv64, float *dinv32, int *err)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t I = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; I < nbr; I += stride) {
        int64_t kd = -1;
        for (int64_t k = rp[I]; k < rp[I + 1]; ++k)
            if (ci[k] == I)
                kd = k;
        for (int r = 0; r < b; ++r) {
            const double d = kd >= 0 ? (double)val[kd * b * b + (int64_t)r * b + r] : 0.0;
            const double inv = d > 0.0 ? 1.0 / d : 0.0;
            if (!(d > 0.0))
                atomicOr(err, 1);
            dinv64[I * b + r] = inv;
            if (dinv32)
                dinv32[I * b + r] = (float)inv;
        }
    }
}

template <typename V>
__global__ void k_gather_values(int64_t nnz, const int32_t *perm, const V *src, V *dst)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < nnz; k += stride)
        dst[k] = src[perm[k]];
}

static inline int vec_grid(const sla_csr *A) { return A->num_sms * 8; }

sla_status launch_spmv(const sla_csr *A, int K, const void *x, void *y, cudaStream_t s)
{
    return A->dtype == SLA_F32 ? spmv_ff(A, K, x, y, s) : spmv_dd(A, K, x, y, s);
}

sla_status launch_pattern_grad(const sla_csr *A, int nrhs, int vec64, const void *lam, const void *x,
                               void *g, cudaStream_t s, double scale)
{
    if (A->dtype == SLA_F64)
        return grad_dd(A, nrhs, lam, x, g, scale, s);
    return vec64 ? grad_fd(A, nrhs, lam, x, g, scale, s) : grad_ff(A, nrhs, lam, x, g, scale, s);
}

sla_status launch_validate(const sla_csr *A, int *d_err, cudaStream_t s)
{
    if (A->n == 0)
        return SLA_SUCCESS;
    // the stored pattern: block rows and block columns of a BSR matrix
    k_validate<<<vec_grid(A), 256, 0, s>>>(pattern_rows(A), A->rp, A->ci, A->d_sys_off, A->batch, d_err);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

sla_status launch_jacobi_dinv(const sla_csr *A, void *dinv64, void *dinv32, int *d_err, cudaStream_t s)
{
    if (A->n == 0)
        return SLA_SUCCESS;
    if (A->bdim > 1) {
        if (A->dtype == SLA_F32)
            k_bsr_dinv<float><<<vec_grid(A), 256, 0, s>>>(pattern_rows(A), A->bdim, A->rp, A->ci,
                                                          (const float *)A->val, (double *)dinv64,
                                                          (float *)dinv32, d_err);
        else
            k_bsr_dinv<double><<<vec_grid(A), 256, 0, s>>>(pattern_rows(A), A->bdim, A->rp, A->ci,
                                                           (const double *)A->val, (double *)dinv64,
                                                           nullptr, d_err);
        SLA_CUDA_TRY(cudaGetLastError());
        return SLA_SUCCESS;
    }
    if (A->dtype == SLA_F32)
        k_jacobi_dinv<float><<<vec_grid(A), 256, 0, s>>>(A->n, A->rp, A->ci, (const float *)A->val,
                                                         (double *)dinv64, (float *)dinv32, d_err);
    else
        k_jacobi_dinv<double><<<vec_grid(A), 256, 0, s>>>(A->n, A->rp, A->ci, (const double *)A->val,
                                                          (double *)dinv64, nullptr, d_err);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

sla_status refresh_transpose_values(const sla_csr *G, sla_csr *GT, const int32_t *perm, cudaStream_t s)
{
    if (G->nnz == 0)
        return SLA_SUCCESS;
    if (G->dtype == SLA_F32)
        k_gather_values<float><<<vec_grid(G), 256, 0, s>>>(G->nnz, perm, (const float *)G->val,
                                                           (float *)GT->own_val);
    else
        k_gather_values<double><<<vec_grid(G), 256, 0, s>>>(G->nnz, perm, (const double *)G->val,
                                                            (double *)GT->own_val);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

// Packed values: slot s takes val[perm[s]] (0 for padding slots).
template <typename V>
__global__ void k_pack_values(int64_t n_slots, const int32_t *perm, const V *val, V *out)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_slots; i += stride) {
        const int32_t k = perm[i];
        out[i] = k >= 0 ? val[k] : (V)0;
    }
}

sla_status launch_sell_values(const sla_csr *A, const SellPart *sp, cudaStream_t s)
{
    if (sp->n_slots == 0)
        return SLA_SUCCESS;
    const int grid = (int)std::min<int64_t>(vec_grid(A), (sp->n_slots + 255) / 256);
    if (A->dtype == SLA_F32)
        k_pack_values<float><<<grid, 256, 0, s>>>(sp->n_slots, sp->d_perm, (const float *)A->val,
                                                  (float *)sp->d_val);
    else
        k_pack_values<double><<<grid, 256, 0, s>>>(sp->n_slots, sp->d_perm, (const double *)A->val,
                                                   (double *)sp->d_val);
    SLA_CUDA_TRY(cudaGetLastError());
    const_cast<sla_csr *>(A)->sell_vals_current = 1;
    return SLA_SUCCESS;
}

// ------------------------------------------------------------------ dispatch
sla_status capture_plan_graph(sla_csr *A, Plan *p)
{
    if (A->dtype == SLA_F64)
        return capture_dd(A, p);
    return p->vec64 ? capture_fd(A, p) : capture_ff(A, p);
}

sla_status kernel_times(sla_csr *A, Plan *p, int nrhs, int reps, double *h_ms, cudaStream_t s)
{
    if (A->dtype == SLA_F64)
        return times_dd(A, p, nrhs, reps, h_ms, s);
    return p->vec64 ? times_fd(A, p, nrhs, reps, h_ms, s) : times_ff(A, p, nrhs, reps, h_ms, s);
}

sla_status run_plan(sla_csr *A, Plan *p, int nrhs, const void *B, void *X,
                    const sla_pcg_opts *opts, sla_pcg_info *info, const void *grad_x,
                    void *grad_out, cudaStream_t s)
{
    const bool f64 = A->dtype == SLA_F64 || p->vec64;
    double tol = (opts && opts->rtol > 0) ? opts->rtol : (f64 ? 1e-10 : 1e-6);
    long long n_sys = A->batch > 1 ? A->max_sys_n : A->n;
    long long maxit = (opts && opts->maxit > 0) ? opts->maxit : 10 * std::max<long long>(n_sys, 1);
    const int engine = opts ? opts->engine : SLA_ENGINE_AUTO;
    if (engine < SLA_ENGINE_AUTO || engine > SLA_ENGINE_PERSISTENT)
        return fail(SLA_ERR_INVALID_ARG, "unknown solve engine");
    sla_status st;
    if (A->dtype == SLA_F64)
        st = run_dd(A, p, nrhs, B, X, tol, maxit, engine, s);
    else if (p->vec64)
        st = run_fd(A, p, nrhs, B, X, tol, maxit, engine, s);
    else
        st = run_ff(A, p, nrhs, B, X, tol, maxit, engine, s);
    if (st != SLA_SUCCESS)
        return st;
    if (grad_out)
        SLA_TRY(launch_pattern_grad(A, nrhs, p->vec64, X, grad_x, grad_out, s));
    SLA_CUDA_TRY(cudaMemcpyAsync(p->h_st, p->st, sizeof(PcgState), cudaMemcpyDeviceToHost, s));
    SLA_CUDA_TRY(cudaStreamSynchronize(s));
    if (p->h_st->error)
        return fail(SLA_ERR_CUDA, "a pipeline wait inside a solver kernel ran out of time; results are invalid");
    sla_status worst = SLA_SUCCESS;
    for (int c = 0; c < nrhs; ++c) {
        if (info) {
            info[c].iters = p->h_st->iters[c];
            info[c].relres = p->h_st->relres[c];
            info[c].status = p->h_st->status[c];
            info[c].engine = p->h_st->persistent ? SLA_ENGINE_PERSISTENT : SLA_ENGINE_GRAPH;
        }
        worst = std::max(worst, (sla_status)p->h_st->status[c]);
    }
    return worst;
}

}  // namespace sla
