// Gradients beyond the linear solve, from "torch-sla: Differentiable Sparse Linear Algebra with
// Adjoint Solvers and Sparse Tensor Parallelism for PyTorch", Methodology §2:
//
// * Eigenvalue problems (Hellmann-Feynman): for a simple eigenvalue mu of a symmetric A with
//   unit eigenvector v, d mu / d A_ij = v_i v_j, needed only on A's pattern -- the pattern
//   outer product of the linear adjoint with the sign flipped (sla_eigen_grad).
// * Nonlinear systems F(u, theta) = 0: the backward pass is one linear adjoint solve
//   J^T lambda = dL/du with the Jacobian J = dF/du at the solution, followed by the
//   vector-Jacobian product dL/dtheta = -lambda^T dF/dtheta, whatever the number of
//   nonlinear iterations.  For F = A u + N(u) - b (A on a sparse pattern, N elementwise) the
//   product is the same pattern outer product: dL/dA_ij = -lambda_i u_j and dL/db = lambda
//   (sla_nonlinear_adjoint).  J = A + diag(N'(u)) is formed on A's pattern by
//   sla_csr_add_diagonal.
#include <cuda_runtime.h>

#include <algorithm>

#include "sla.h"
#include "sla_internal.cuh"

namespace sla {

// d_out[row's diagonal entry] += c[row] for every row (d_out holds a copy of A's values).
// Columns are ascending in each row, so the diagonal is found by binary search; a row that
// stores no diagonal entry sets *err.
template <typename V>
__global__ void k_add_diagonal(int64_t n, const int32_t *rp, const int32_t *ci, const V *c, V *out, int *err)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        int64_t lo = rp[i], hi = (int64_t)rp[i + 1] - 1;
        int64_t at = -1;
        while (lo <= hi) {
            const int64_t mid = (lo + hi) >> 1;
            const int32_t col = ci[mid];
            if (col == i) {
                at = mid;
                break;
            }
            if (col < i)
                lo = mid + 1;
            else
                hi = mid - 1;
        }
        if (at < 0)
            atomicOr(err, 1);
        else
            out[at] = out[at] + c[i];
    }
}

}  // namespace sla

using namespace sla;

extern "C" {

sla_status sla_eigen_grad(const sla_csr *A, int32_t nvec, const void *d_V, void *d_g, void *stream)
{
    if (!A)
        return fail(SLA_ERR_INVALID_ARG, "NULL handle");
    if (nvec < 1)
        return fail(SLA_ERR_INVALID_ARG, "nvec must be >= 1");
    if (A->nnz > 0 && (!d_V || !d_g))
        return fail(SLA_ERR_INVALID_ARG, "NULL vector");
    if (A->nnz == 0)
        return SLA_SUCCESS;
    return launch_pattern_grad(A, nvec, 0, d_V, d_V, d_g, (cudaStream_t)stream, +1.0);
}

sla_status sla_csr_add_diagonal(const sla_csr *A, const void *d_c, void *d_val_out, void *stream)
{
    if (!A)
        return fail(SLA_ERR_INVALID_ARG, "NULL handle");
    if (A->bdim > 1)
        return fail(SLA_ERR_UNSUPPORTED, "sla_csr_add_diagonal takes a CSR handle (not BSR)");
    if (A->nnz > 0 && (!d_c || !d_val_out))
        return fail(SLA_ERR_INVALID_ARG, "NULL vector");
    if (A->n == 0)
        return SLA_SUCCESS;
    if (d_val_out == A->val)
        return fail(SLA_ERR_INVALID_ARG, "d_val_out must not be A's own value array");
    cudaStream_t s = (cudaStream_t)stream;
    const size_t vb = A->dtype == SLA_F32 ? 4 : 8;
    SLA_CUDA_TRY(cudaMemcpyAsync(d_val_out, A->val, (size_t)A->nnz * vb, cudaMemcpyDeviceToDevice, s));
    int *d_err = nullptr;
    SLA_CUDA_TRY(cudaMallocAsync((void **)&d_err, sizeof(int), s));
    SLA_CUDA_TRY(cudaMemsetAsync(d_err, 0, sizeof(int), s));
    const int grid = (int)std::min<int64_t>((A->n + 255) / 256, (int64_t)A->num_sms * 8);
    if (A->dtype == SLA_F32)
        k_add_diagonal<float><<<grid, 256, 0, s>>>(A->n, A->rp, A->ci, (const float *)d_c, (float *)d_val_out,
                                                  d_err);
    else
        k_add_diagonal<double><<<grid, 256, 0, s>>>(A->n, A->rp, A->ci, (const double *)d_c,
                                                   (double *)d_val_out, d_err);
    cudaError_t e = cudaGetLastError();
    int h_err = 0;
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(&h_err, d_err, sizeof(int), cudaMemcpyDeviceToHost, s);
    cudaFreeAsync(d_err, s);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(s);
    if (e != cudaSuccess)
        return cuda_fail(e, "sla_csr_add_diagonal");
    if (h_err)
        return fail(SLA_ERR_INVALID_ARG, "a row stores no diagonal entry");
    return SLA_SUCCESS;
}

sla_status sla_nonlinear_adjoint(const sla_csr *J, const sla_precond *M, const sla_csr *A, const void *d_u,
                                 const void *d_dLdu, void *d_lambda, void *d_dLdA,
                                 const sla_pcg_opts *opts, sla_pcg_info *info, void *stream)
{
    if (!J)
        return fail(SLA_ERR_INVALID_ARG, "NULL Jacobian handle");
    if (A && (A->n != J->n || A->dtype != J->dtype || A->batch != J->batch))
        return fail(SLA_ERR_INVALID_ARG, "A and J must have the same size, dtype and batch");
    if (d_dLdA && !A)
        return fail(SLA_ERR_INVALID_ARG, "d_dLdA needs the matrix A whose values are the parameters");
    if (J->n > 0 && d_dLdA && !d_u)
        return fail(SLA_ERR_INVALID_ARG, "NULL solution u");
    // J is SPD, so J^T lambda = dL/du is the same PCG solve as J lambda = dL/du
    sla_status st = sla_pcg_solve(J, M, d_dLdu, d_lambda, opts, info, stream);
    if (st < 0)
        return st;
    if (A && d_dLdA && A->nnz > 0) {
        const int vec64 = (opts && opts->vector_f64 && A->dtype == SLA_F32) ? 1 : 0;
        SLA_TRY(launch_pattern_grad(A, 1, vec64, d_lambda, d_u, d_dLdA, (cudaStream_t)stream, -1.0));
        SLA_CUDA_TRY(cudaStreamSynchronize((cudaStream_t)stream));
    }
    return st;
}

}  // extern "C"
