// The explicit transpose G^T of the SPAI factor, built on the device ([SPAI] "Learning Sparse
// Approximate Inverse Preconditioners for Conjugate Gradient Solvers on GPUs", Approach:
// the apply z = G (G^T r) + eps r is two plain SpMVs once G^T is stored).
//
// Row j of G^T lists the rows i of G that store column j, in increasing i.  G's entries are
// sorted by column with the stable radix sort (radix_sort.cuh): entries of one column keep
// their CSR order, which is increasing row.  perm[t] = position in G of the t-th entry of
// G^T (so a later change of G's values is one gather), col_T[t] = row of that entry in G,
// and row_ptr_T[j] = first sorted position whose column is >= j.
#include <cuda_runtime.h>

#include <algorithm>

#include "sla.h"
#include "sla_internal.cuh"
#include "radix_sort.cuh"

namespace sla {

namespace {

// ri[k] = row of entry k (one warp per row).
__global__ void k_row_of_entry(int64_t n, const int32_t *rp, int32_t *ri)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; i < n; i += warps)
        for (int64_t k = rp[i] + lane; k < rp[i + 1]; k += 32)
            ri[k] = (int32_t)i;
}

// Sort keys (the columns) and values (entry positions); *err = 1 for a column outside
// [0, ncols) (its key is then 0, so the sort still stays inside its buffers).
__global__ void k_transpose_keys(int64_t nnz, int64_t ncols, const int32_t *ci, uint32_t *key, int32_t *val,
                                 int *err)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < nnz; k += stride) {
        int32_t c = ci[k];
        if (c < 0 || c >= ncols) {
            atomicOr(err, 1);
            c = 0;
        }
        key[k] = (uint32_t)c;
        val[k] = (int32_t)k;
    }
}

// row_ptr_T from the sorted columns: every column in (key[t-1], key[t]] starts at t, and the
// columns after the last key start at nnz.
__global__ void k_rp_from_sorted(int64_t nnz, int64_t nrows_t, const uint32_t *key, int32_t *rpT)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < nnz; t += stride) {
        const int64_t c = key[t];
        const int64_t p = t > 0 ? (int64_t)key[t - 1] : -1;
        for (int64_t j = p + 1; j <= c; ++j)
            rpT[j] = (int32_t)t;
        if (t == nnz - 1)
            for (int64_t j = c + 1; j <= nrows_t; ++j)
                rpT[j] = (int32_t)nnz;
    }
}

__global__ void k_gather_rows(int64_t nnz, const int32_t *perm, const int32_t *ri, int32_t *ciT)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < nnz; t += stride)
        ciT[t] = ri[perm[t]];
}

}  // namespace

sla_status device_transpose(const sla_csr *G, int32_t *rpT, int32_t *ciT, int32_t *perm, cudaStream_t s)
{
    const int64_t n = G->n, nnz = G->nnz;
    if (nnz == 0) {
        SLA_CUDA_TRY(cudaMemsetAsync(rpT, 0, sizeof(int32_t) * (size_t)(n + 1), s));
        return SLA_SUCCESS;
    }
    uint32_t *k0 = nullptr, *k1 = nullptr;
    int32_t *v0 = nullptr, *v1 = nullptr, *ri = nullptr;
    int *d_err = nullptr;
    const size_t b4 = sizeof(int32_t) * (size_t)nnz;
    cudaError_t e = cudaMallocAsync((void **)&k0, b4, s);
    if (e == cudaSuccess) e = cudaMallocAsync((void **)&k1, b4, s);
    if (e == cudaSuccess) e = cudaMallocAsync((void **)&v0, b4, s);
    if (e == cudaSuccess) e = cudaMallocAsync((void **)&v1, b4, s);
    if (e == cudaSuccess) e = cudaMallocAsync((void **)&ri, b4, s);
    if (e == cudaSuccess) e = cudaMallocAsync((void **)&d_err, sizeof(int), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_err, 0, sizeof(int), s);
    const int grid = (int)std::min<int64_t>((nnz + 255) / 256, (int64_t)G->num_sms * 16);
    const int rgrid = (int)std::min<int64_t>((n + 7) / 8, (int64_t)G->num_sms * 16);
    uint32_t *ks = nullptr;
    int32_t *vs = nullptr;
    if (e == cudaSuccess) {
        k_transpose_keys<<<grid, 256, 0, s>>>(nnz, n, G->ci, k0, v0, d_err);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess && n > 0) {
        k_row_of_entry<<<std::max(rgrid, 1), 256, 0, s>>>(n, G->rp, ri);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess)
        e = radix_sort_pairs<uint32_t>(k0, v0, k1, v1, nnz, std::max(1, bits_for((uint64_t)std::max<int64_t>(n - 1, 0))),
                                       &ks, &vs, s);
    if (e == cudaSuccess) {
        k_rp_from_sorted<<<grid, 256, 0, s>>>(nnz, n, ks, rpT);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        k_gather_rows<<<grid, 256, 0, s>>>(nnz, vs, ri, ciT);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(perm, vs, b4, cudaMemcpyDeviceToDevice, s);
    int h_err = 0;
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(&h_err, d_err, sizeof(int), cudaMemcpyDeviceToHost, s);
    for (void *p : {(void *)k0, (void *)k1, (void *)v0, (void *)v1, (void *)ri, (void *)d_err})
        if (p)
            cudaFreeAsync(p, s);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(s);
    if (e != cudaSuccess)
        return cuda_fail(e, "G^T on the device");
    if (h_err)
        return fail(SLA_ERR_INVALID_CSR, "G: column index out of range");
    return SLA_SUCCESS;
}

}  // namespace sla
