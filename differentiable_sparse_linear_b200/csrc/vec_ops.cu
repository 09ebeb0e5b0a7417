// Vector steps of one PCG iteration as separate calls, for solvers whose iteration is driven
// from the host between collectives: the row-block distributed PCG of "torch-sla:
// Differentiable Sparse Linear Algebra with Adjoint Solvers and Sparse Tensor Parallelism
// for PyTorch", Methodology §3 (each rank owns a block of rows; halo values are exchanged
// before each product and the scalars of the recurrence are all-reduced).  The fused
// single-GPU engines do the same arithmetic inside their SpMV epilogues.
//
// Dot products are fp64 and deterministic: each block sums a fixed strided share in a fixed
// shuffle order, and one block then sums the block partials in block order.  Vector updates
// use the single-GPU engines' arithmetic: a*b + c with a rounded once to the vector type and
// one fused multiply-add in that type.
#include <cuda_runtime.h>

#include <algorithm>

#include "sla.h"
#include "sla_internal.cuh"

namespace sla {
namespace {

constexpr int VT = 256;
constexpr int MAX_BLOCKS = 1184;     // 148 SMs x 8

template <typename V>
__device__ __forceinline__ V fma_v(double a, V b, V c);
template <>
__device__ __forceinline__ float fma_v<float>(double a, float b, float c) { return __fmaf_rn((float)a, b, c); }
template <>
__device__ __forceinline__ double fma_v<double>(double a, double b, double c) { return __fma_rn(a, b, c); }

// Sum N values over the block in a fixed order; thread 0 returns the totals in v.
template <int N>
__device__ __forceinline__ void block_sum_fixed(double (&v)[N], double *s_red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < N; ++i)
        for (int off = 16; off > 0; off >>= 1)
            v[i] += __shfl_down_sync(0xffffffffu, v[i], off);
    if (lane == 0)
#pragma unroll
        for (int i = 0; i < N; ++i)
            s_red[warp * N + i] = v[i];
    __syncthreads();
    if (threadIdx.x == 0)
#pragma unroll
        for (int i = 0; i < N; ++i) {
            double t = 0.0;
            for (int w = 0; w < VT / 32; ++w)
                t += s_red[w * N + i];
            v[i] = t;
        }
}

template <int N>
__global__ void __launch_bounds__(VT) k_sum_partials(int nb, const double *part, double *out)
{
    __shared__ double s_red[(VT / 32) * N];
    double v[N];
#pragma unroll
    for (int i = 0; i < N; ++i)
        v[i] = 0.0;
    for (int b = threadIdx.x; b < nb; b += VT)
#pragma unroll
        for (int i = 0; i < N; ++i)
            v[i] += part[(size_t)b * N + i];
    block_sum_fixed<N>(v, s_red);
    if (threadIdx.x == 0)
#pragma unroll
        for (int i = 0; i < N; ++i)
            out[i] = v[i];
}

template <typename V>
__global__ void __launch_bounds__(VT) k_dot(int64_t n, const V *x, const V *y, double *part)
{
    __shared__ double s_red[VT / 32];
    double v[1] = {0.0};
    const int64_t stride = (int64_t)gridDim.x * VT;
    for (int64_t i = (int64_t)blockIdx.x * VT + threadIdx.x; i < n; i += stride)
        v[0] += (double)x[i] * (double)y[i];
    block_sum_fixed<1>(v, s_red);
    if (threadIdx.x == 0)
        part[blockIdx.x] = v[0];
}

// x += alpha p; r -= alpha q; z = dinv * r (r when dinv is null); partials r.r, r.z
template <typename V>
__global__ void __launch_bounds__(VT) k_update(int64_t n, double alpha, const V *p, const V *q, V *x, V *r,
                                               const V *dinv, V *z, double *part)
{
    __shared__ double s_red[(VT / 32) * 2];
    double v[2] = {0.0, 0.0};
    const int64_t stride = (int64_t)gridDim.x * VT;
    for (int64_t i = (int64_t)blockIdx.x * VT + threadIdx.x; i < n; i += stride) {
        x[i] = fma_v<V>(alpha, p[i], x[i]);
        const V ri = fma_v<V>(-alpha, q[i], r[i]);
        r[i] = ri;
        const V zi = dinv ? (V)((double)ri * (double)dinv[i]) : ri;
        z[i] = zi;
        v[0] += (double)ri * (double)ri;
        v[1] += (double)ri * (double)zi;
    }
    block_sum_fixed<2>(v, s_red);
    if (threadIdx.x == 0) {
        part[(size_t)blockIdx.x * 2] = v[0];
        part[(size_t)blockIdx.x * 2 + 1] = v[1];
    }
}

template <typename V>
__global__ void k_direction(int64_t n, double beta, const V *z, V *p)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        p[i] = fma_v<V>(beta, p[i], z[i]);
}

template <typename V>
__global__ void k_gather(int64_t n, const int32_t *idx, const V *src, V *dst)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride)
        dst[k] = src[idx[k]];
}

template <typename V>
__global__ void k_scatter_add(int64_t n, const int32_t *idx, const V *src, V *dst)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride) {
        const int32_t j = idx[k];
        dst[j] = dst[j] + src[k];
    }
}

int grid_for(int64_t n) { return (int)std::max<int64_t>(1, std::min<int64_t>((n + VT - 1) / VT, MAX_BLOCKS)); }

sla_status check_dtype(int32_t dtype)
{
    if (dtype != SLA_F32 && dtype != SLA_F64)
        return fail(SLA_ERR_INVALID_ARG, "dtype must be SLA_F32 or SLA_F64");
    return SLA_SUCCESS;
}

// Partials of `nb` blocks, N values each, then their fixed-order sum into d_out.
template <int N, class Launch>
sla_status reduce_into(int nb, double *d_out, cudaStream_t s, Launch launch)
{
    double *part = nullptr;
    SLA_CUDA_TRY(cudaMallocAsync((void **)&part, sizeof(double) * N * (size_t)nb, s));
    launch(part);
    k_sum_partials<N><<<1, VT, 0, s>>>(nb, part, d_out);
    cudaError_t e = cudaGetLastError();
    cudaFreeAsync(part, s);
    if (e != cudaSuccess)
        return cuda_fail(e, "vector reduction");
    return SLA_SUCCESS;
}

}  // namespace
}  // namespace sla

using namespace sla;

extern "C" {

sla_status sla_vec_dot(int32_t dtype, int64_t n, const void *d_x, const void *d_y, double *d_out, void *stream)
{
    SLA_TRY(check_dtype(dtype));
    if (n < 0 || !d_out || (n > 0 && (!d_x || !d_y)))
        return fail(SLA_ERR_INVALID_ARG, "bad size or NULL vector");
    cudaStream_t s = (cudaStream_t)stream;
    const int nb = grid_for(n);
    return reduce_into<1>(nb, d_out, s, [&](double *part) {
        if (dtype == SLA_F32)
            k_dot<float><<<nb, VT, 0, s>>>(n, (const float *)d_x, (const float *)d_y, part);
        else
            k_dot<double><<<nb, VT, 0, s>>>(n, (const double *)d_x, (const double *)d_y, part);
    });
}

sla_status sla_pcg_update(int32_t dtype, int64_t n, double alpha, const void *d_p, const void *d_q, void *d_x,
                          void *d_r, const void *d_dinv, void *d_z, double *d_out2, void *stream)
{
    SLA_TRY(check_dtype(dtype));
    if (n < 0 || !d_out2 || (n > 0 && (!d_p || !d_q || !d_x || !d_r || !d_z)))
        return fail(SLA_ERR_INVALID_ARG, "bad size or NULL vector");
    cudaStream_t s = (cudaStream_t)stream;
    const int nb = grid_for(n);
    return reduce_into<2>(nb, d_out2, s, [&](double *part) {
        if (dtype == SLA_F32)
            k_update<float><<<nb, VT, 0, s>>>(n, alpha, (const float *)d_p, (const float *)d_q, (float *)d_x,
                                              (float *)d_r, (const float *)d_dinv, (float *)d_z, part);
        else
            k_update<double><<<nb, VT, 0, s>>>(n, alpha, (const double *)d_p, (const double *)d_q, (double *)d_x,
                                               (double *)d_r, (const double *)d_dinv, (double *)d_z, part);
    });
}

sla_status sla_pcg_direction(int32_t dtype, int64_t n, double beta, const void *d_z, void *d_p, void *stream)
{
    SLA_TRY(check_dtype(dtype));
    if (n < 0 || (n > 0 && (!d_z || !d_p)))
        return fail(SLA_ERR_INVALID_ARG, "bad size or NULL vector");
    if (n == 0)
        return SLA_SUCCESS;
    cudaStream_t s = (cudaStream_t)stream;
    if (dtype == SLA_F32)
        k_direction<float><<<grid_for(n), VT, 0, s>>>(n, beta, (const float *)d_z, (float *)d_p);
    else
        k_direction<double><<<grid_for(n), VT, 0, s>>>(n, beta, (const double *)d_z, (double *)d_p);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

sla_status sla_vec_gather(int32_t dtype, int64_t n, const int32_t *d_idx, const void *d_src, void *d_dst,
                          void *stream)
{
    SLA_TRY(check_dtype(dtype));
    if (n < 0 || (n > 0 && (!d_idx || !d_src || !d_dst)))
        return fail(SLA_ERR_INVALID_ARG, "bad size or NULL vector");
    if (n == 0)
        return SLA_SUCCESS;
    cudaStream_t s = (cudaStream_t)stream;
    if (dtype == SLA_F32)
        k_gather<float><<<grid_for(n), VT, 0, s>>>(n, d_idx, (const float *)d_src, (float *)d_dst);
    else
        k_gather<double><<<grid_for(n), VT, 0, s>>>(n, d_idx, (const double *)d_src, (double *)d_dst);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

sla_status sla_vec_scatter_add(int32_t dtype, int64_t n, const int32_t *d_idx, const void *d_src, void *d_dst,
                               void *stream)
{
    SLA_TRY(check_dtype(dtype));
    if (n < 0 || (n > 0 && (!d_idx || !d_src || !d_dst)))
        return fail(SLA_ERR_INVALID_ARG, "bad size or NULL vector");
    if (n == 0)
        return SLA_SUCCESS;
    cudaStream_t s = (cudaStream_t)stream;
    if (dtype == SLA_F32)
        k_scatter_add<float><<<grid_for(n), VT, 0, s>>>(n, d_idx, (const float *)d_src, (float *)d_dst);
    else
        k_scatter_add<double><<<grid_for(n), VT, 0, s>>>(n, d_idx, (const double *)d_src, (double *)d_dst);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

}  // extern "C"
