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
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "sla_internal.cuh"
#include "tile_engine.cuh"

namespace sla {

// ------------------------------------------------------------------ scalar finalisation
__device__ __forceinline__ bool finite_d(double a) { return isfinite(a); }

__device__ void signal_if_done(PcgState *st)
{
    int any = 0;
    for (int c = 0; c < st->k; ++c)
        any |= st->active[c];
    if (!any) {
        st->all_done = 1;
        if (st->has_cond)
            cudaGraphSetConditional((cudaGraphConditionalHandle)st->cond_handle, 0u);
    }
}

// After q = A p: alpha = rho / (p.q); p.q <= 0 or non-finite is a breakdown.
__device__ void finalize_alpha(PcgState *st, const double *pq)
{
    if (st->profile)
        return;
    for (int c = 0; c < st->k; ++c) {
        if (!st->active[c])
            continue;
        const double d = pq[c];
        if (!(d > 0.0) || !finite_d(d)) {
            st->status[c] = SLA_BREAKDOWN;
            st->active[c] = 0;
        } else {
            st->alpha[c] = st->rho[c] / d;
        }
    }
    signal_if_done(st);
}

// After the x/r update: stopping test on ||r||/||b|| (initial pass: record ||b||).
__device__ void finalize_residual(PcgState *st, const double *rr)
{
    if (st->profile)
        return;
    for (int c = 0; c < st->k; ++c) {
        if (!st->active[c])
            continue;
        if (st->phase0) {
            const double bn = sqrt(rr[c]);
            st->bnorm[c] = bn;
            st->relres[c] = bn > 0.0 ? 1.0 : 0.0;
            if (!finite_d(bn)) {
                st->status[c] = SLA_BREAKDOWN;
                st->active[c] = 0;
            } else if (bn == 0.0) {
                st->status[c] = SLA_SUCCESS;
                st->active[c] = 0;
            }
        } else {
            st->iters[c] += 1;
            const double rel = sqrt(rr[c]) / st->bnorm[c];
            st->relres[c] = rel;
            if (!finite_d(rel)) {
                st->status[c] = SLA_BREAKDOWN;
                st->active[c] = 0;
            } else if (rel <= st->tol) {
                st->status[c] = SLA_SUCCESS;
                st->active[c] = 0;
            } else if (st->iters[c] >= st->maxit) {
                st->status[c] = SLA_NOT_CONVERGED;
                st->active[c] = 0;
            }
        }
    }
}

// After z = M^-1 r: rho' = r.z, beta = rho'/rho (0 on the initial pass).
__device__ void finalize_beta(PcgState *st, const double *rz)
{
    if (st->profile)
        return;
    for (int c = 0; c < st->k; ++c) {
        if (!st->active[c])
            continue;
        const double v = rz[c];
        if (!(v > 0.0) || !finite_d(v)) {
            st->status[c] = SLA_BREAKDOWN;
            st->active[c] = 0;
            continue;
        }
        st->beta[c] = st->phase0 ? 0.0 : v / st->rho[c];
        st->rho[c] = v;
    }
    st->phase0 = 0;
    signal_if_done(st);
}

// ------------------------------------------------------------------ operations
// y = A x for K right-hand sides with leading dimension ld (columns c >= nc are zero).
template <typename V, int K>
struct OpSpmv {
    static constexpr int NP = 0, NS = 0;
    const V *x;
    V *y;
    int ld, nc;
    __device__ bool skip() const { return false; }
    __device__ void stage(double *) const {}
    __device__ __forceinline__ double operand(int64_t j, int c, const double *) const
    {
        return c < nc ? (double)__ldg(&x[j * ld + c]) : 0.0;
    }
    template <int N>
    __device__ __forceinline__ void emit(int64_t i, const double (&acc)[K], double (&)[N],
                                         const double *) const
    {
#pragma unroll
        for (int c = 0; c < K; ++c)
            if (c < nc)
                y[i * ld + c] = (V)acc[c];
    }
    __device__ void finalize(const double *) const {}
};

// Q: p_new = z + beta p_old, q = A p_new, partial p_new.q
template <typename V, int K>
struct OpQ {
    static constexpr int NP = 1, NS = K;
    const V *z;
    const V *p_old;
    V *p_new;
    V *q;
    PcgState *st;
    __device__ bool skip() const { return *(volatile int *)&st->all_done; }
    __device__ void stage(double *s) const
    {
        for (int c = 0; c < K; ++c)
            s[c] = st->beta[c];
    }
    __device__ __forceinline__ V pnew(int64_t j, int c, const double *s) const
    {
        return (V)__fma_rn(s[c], (double)p_old[j * K + c], (double)z[j * K + c]);
    }
    __device__ __forceinline__ double operand(int64_t j, int c, const double *s) const
    {
        return (double)pnew(j, c, s);
    }
    template <int N>
    __device__ __forceinline__ void emit(int64_t i, const double (&acc)[K], double (&part)[N],
                                         const double *s) const
    {
#pragma unroll
        for (int c = 0; c < K; ++c) {
            const V pn = pnew(i, c, s);
            const V qv = (V)acc[c];
            p_new[i * K + c] = pn;
            q[i * K + c] = qv;
            part[c] += (double)pn * (double)qv;
        }
    }
    __device__ void finalize(const double *sums) const { finalize_alpha(st, sums); }
};

// U_S: r_new = r_old - alpha q, x += alpha p, y = G^T r_new, partial r_new.r_new
template <typename V, int K>
struct OpUS {
    static constexpr int NP = 1, NS = 2 * K;
    const V *r_old;
    const V *q;
    const V *p;
    V *r_new;
    V *x;
    V *y;
    PcgState *st;
    __device__ bool skip() const { return *(volatile int *)&st->all_done; }
    __device__ void stage(double *s) const
    {
        for (int c = 0; c < K; ++c) {
            s[c] = st->alpha[c];
            s[K + c] = st->active[c] ? 1.0 : 0.0;
        }
    }
    __device__ __forceinline__ V rnew(int64_t j, int c, const double *s) const
    {
        const V ro = r_old[j * K + c];
        return s[K + c] != 0.0 ? (V)__fma_rn(-s[c], (double)q[j * K + c], (double)ro) : ro;
    }
    __device__ __forceinline__ double operand(int64_t j, int c, const double *s) const
    {
        return (double)rnew(j, c, s);
    }
    template <int N>
    __device__ __forceinline__ void emit(int64_t i, const double (&acc)[K], double (&part)[N],
                                         const double *s) const
    {
#pragma unroll
        for (int c = 0; c < K; ++c) {
            const V rn = rnew(i, c, s);
            r_new[i * K + c] = rn;
            if (s[K + c] != 0.0)
                x[i * K + c] = (V)__fma_rn(s[c], (double)p[i * K + c], (double)x[i * K + c]);
            y[i * K + c] = (V)acc[c];
            part[c] += (double)rn * (double)rn;
        }
    }
    __device__ void finalize(const double *sums) const
    {
        if (st->profile)
            return;
        finalize_residual(st, sums);
        signal_if_done(st);
    }
};

// Z: z = G y + eps r, partial r.z
template <typename V, int K>
struct OpZ {
    static constexpr int NP = 1, NS = 1;
    const V *y;
    const V *r;
    V *z;
    PcgState *st;
    __device__ bool skip() const { return *(volatile int *)&st->all_done; }
    __device__ void stage(double *s) const { s[0] = st->eps; }
    __device__ __forceinline__ double operand(int64_t j, int c, const double *) const
    {
        return (double)y[j * K + c];
    }
    template <int N>
    __device__ __forceinline__ void emit(int64_t i, const double (&acc)[K], double (&part)[N],
                                         const double *s) const
    {
#pragma unroll
        for (int c = 0; c < K; ++c) {
            const double rv = (double)r[i * K + c];
            const V zv = (V)__fma_rn(s[0], rv, acc[c]);
            z[i * K + c] = zv;
            part[c] += rv * (double)zv;
        }
    }
    __device__ void finalize(const double *sums) const { finalize_beta(st, sums); }
};

// ------------------------------------------------------------------ elementwise kernels
constexpr int VEC_T = 256;

struct UJFinal {
    PcgState *st;
    int K;
    __device__ void finalize(const double *sums) const
    {
        // sums[c] = r.r, sums[K + c] = r.z
        finalize_residual(st, sums);
        finalize_beta(st, sums + K);
    }
};

// U_J: x += alpha p; r -= alpha q; z = D^-1 r; partials r.r, r.z (rows, all K columns)
template <typename V, int K>
__global__ void __launch_bounds__(VEC_T)
k_update_jacobi(int64_t n, V *x, V *r, const V *p, const V *q, V *z, const V *dinv,
                double *partials, PcgState *st)
{
    __shared__ double s_a[K];
    __shared__ double s_on[K];
    __shared__ double s_red[(VEC_T / 32) * 2 * K];
    if (*(volatile int *)&st->all_done)
        return;
    if (threadIdx.x < K) {
        s_a[threadIdx.x] = st->alpha[threadIdx.x];
        s_on[threadIdx.x] = st->active[threadIdx.x] ? 1.0 : 0.0;
    }
    __syncthreads();
    double part[2 * K];
#pragma unroll
    for (int i = 0; i < 2 * K; ++i)
        part[i] = 0.0;
    const int64_t stride = (int64_t)gridDim.x * VEC_T;
    for (int64_t i = (int64_t)blockIdx.x * VEC_T + threadIdx.x; i < n; i += stride) {
        const double di = (double)dinv[i];
#pragma unroll
        for (int c = 0; c < K; ++c) {
            const int64_t e = i * K + c;
            double rv = (double)r[e];
            if (s_on[c] != 0.0) {
                x[e] = (V)__fma_rn(s_a[c], (double)p[e], (double)x[e]);
                const V rn = (V)__fma_rn(-s_a[c], (double)q[e], rv);
                r[e] = rn;
                rv = (double)rn;
            }
            const V zv = (V)(rv * di);
            z[e] = zv;
            part[c] += rv * rv;
            part[K + c] += rv * (double)zv;
        }
    }
    UJFinal fin{st, K};
    grid_reduce_finalize<VEC_T, 2 * K>(part, partials, st, fin, s_red);
}

// Reset the state and load the right-hand sides: r = b (padded to K columns), x = p = q = 0.
template <typename V, int K>
__global__ void k_init(int64_t n, int nrhs, const V *B, V *x, V *r, V *p, V *q, V *z, V *y,
                       PcgState *st, double tol, long long maxit, double eps,
                       unsigned long long cond, int has_cond)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * K; e += stride) {
        const int64_t i = e / K;
        const int c = (int)(e - i * K);
        r[e] = c < nrhs ? B[i * nrhs + c] : (V)0;
        x[e] = (V)0;
        p[e] = (V)0;
        q[e] = (V)0;
        z[e] = (V)0;
        if (y)
            y[e] = (V)0;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        for (int c = 0; c < KMAX; ++c) {
            st->rho[c] = 0.0;
            st->alpha[c] = 0.0;
            st->beta[c] = 0.0;
            st->bnorm[c] = 0.0;
            st->relres[c] = 0.0;
            st->iters[c] = 0;
            st->status[c] = SLA_SUCCESS;
            st->active[c] = c < nrhs ? 1 : 0;
        }
        st->all_done = nrhs > 0 ? 0 : 1;
        st->phase0 = 1;
        st->ticket = 0u;
        st->k = K;
        st->tol = tol;
        st->maxit = maxit;
        st->eps = eps;
        st->cond_handle = cond;
        st->has_cond = has_cond;
        st->profile = 0;
    }
}

// Timing mode: every RHS active, finalisation off, so each kernel can be launched alone
// any number of times on the workspace the last solve left.
__global__ void k_profile_mode(PcgState *st, int nrhs)
{
    for (int c = 0; c < KMAX; ++c)
        st->active[c] = c < nrhs ? 1 : 0;
    st->all_done = 0;
    st->has_cond = 0;
    st->profile = 1;
    st->ticket = 0u;
}

template <typename V, int K>
__global__ void k_copy_out(int64_t n, int nrhs, const V *x, V *X)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * nrhs; e += stride) {
        const int64_t i = e / nrhs;
        const int c = (int)(e - i * nrhs);
        X[e] = x[i * K + c];
    }
}

// ------------------------------------------------------------------ pattern gradient
// g_k = -sum_c lam[row(k)*nrhs + c] * x[col(k)*nrhs + c] over the tiles of A: the tile's
// row ends are staged in shared memory and each entry finds its row by binary search, so
// entries are read and g written with coalesced accesses, for any row-length mix.
constexpr int GRAD_T = 256;
constexpr int GRAD_D = 2048;

template <typename V>
__global__ void __launch_bounds__(GRAD_T)
k_pattern_grad(const MatView<V> m, int nrhs, const V *lam, const V *x, V *g)
{
    __shared__ int32_t s_rp[GRAD_D];
    for (int t = blockIdx.x; t < m.n_tiles; t += gridDim.x) {
        const int r0 = m.tile_row[t];
        const int r1 = m.tile_row[t + 1];
        const int nr = r1 - r0;
        const int64_t k0 = m.rp[r0];
        const int nk = (int)(m.rp[r1] - k0);
        const bool longrow = nr + nk > GRAD_D;
        if (!longrow)
            for (int r = threadIdx.x; r < nr; r += GRAD_T)
                s_rp[r] = (int32_t)(m.rp[r0 + 1 + r] - k0);
        __syncthreads();
        for (int e = threadIdx.x; e < nk; e += GRAD_T) {
            int row = 0;
            if (!longrow) {  // first row whose end exceeds e
                int lo = 0, hi = nr - 1;
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (s_rp[mid] > e)
                        hi = mid;
                    else
                        lo = mid + 1;
                }
                row = lo;
            }
            const int64_t i = r0 + row;
            const int64_t j = m.ci[k0 + e];
            double s = 0.0;
            for (int c = 0; c < nrhs; ++c)
                s = __fma_rn((double)lam[i * nrhs + c], (double)x[j * nrhs + c], s);
            g[k0 + e] = (V)(-s);
        }
        __syncthreads();
    }
}

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

// D^-1 of A in A's value type; a missing or non-positive diagonal sets *err.
template <typename V>
__global__ void k_jacobi_dinv(int64_t n, const int32_t *rp, const int32_t *ci, const V *val,
                              V *dinv, int *err)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        double d = 0.0;
        for (int64_t k = rp[i]; k < rp[i + 1]; ++k)
            if (ci[k] == i)
                d = (double)val[k];
        if (!(d > 0.0)) {
            atomicOr(err, 1);
            dinv[i] = (V)0;
        } else {
            dinv[i] = (V)(1.0 / d);
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

// ------------------------------------------------------------------ host helpers
static inline int vec_grid(const sla_csr *A) { return A->num_sms * 8; }

template <typename V>
static MatView<V> view(const sla_csr *A, const TilePart *tp)
{
    MatView<V> m;
    m.rp = A->rp;
    m.ci = A->ci;
    m.val = (const V *)A->val;
    m.tile_row = tp->d_tile_row;
    m.n_tiles = tp->n_tiles;
    m.n = A->n;
    return m;
}

template <int K, typename V, class Op>
static int tile_grid(const sla_csr *A, const TilePart *tp)
{
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_tile<K, V, Op>, TileCfg<K>::T, 0);
    per_sm = std::max(per_sm, 1);
    return std::max(1, std::min(tp->n_tiles, per_sm * A->num_sms));
}

template <typename V, int K>
static sla_status spmv_k(const sla_csr *A, int nc, const void *x, void *y, cudaStream_t s)
{
    const TilePart *tp;
    SLA_TRY(ensure_tiles(const_cast<sla_csr *>(A), TileCfg<K>::D, s, &tp));
    OpSpmv<V, K> op{(const V *)x, (V *)y, nc, nc};
    const int grid = tile_grid<K, V, OpSpmv<V, K>>(A, tp);
    if (tp->n_tiles > 0)
        k_tile<K, V, OpSpmv<V, K>><<<grid, TileCfg<K>::T, 0, s>>>(view<V>(A, tp), op, nullptr, nullptr);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

static int pad_k(int nrhs)
{
    int K = 1;
    while (K < nrhs)
        K <<= 1;
    return K;
}

template <typename V>
static sla_status spmv_v(const sla_csr *A, int nrhs, const void *x, void *y, cudaStream_t s)
{
    switch (pad_k(nrhs)) {
    case 1: return spmv_k<V, 1>(A, nrhs, x, y, s);
    case 2: return spmv_k<V, 2>(A, nrhs, x, y, s);
    case 4: return spmv_k<V, 4>(A, nrhs, x, y, s);
    case 8: return spmv_k<V, 8>(A, nrhs, x, y, s);
    case 16: return spmv_k<V, 16>(A, nrhs, x, y, s);
    default: return fail(SLA_ERR_INVALID_ARG, "nrhs must be in [1, 16]");
    }
}

sla_status launch_spmv(const sla_csr *A, int K, const void *x, void *y, cudaStream_t s)
{
    return A->dtype == SLA_F32 ? spmv_v<float>(A, K, x, y, s) : spmv_v<double>(A, K, x, y, s);
}

template <typename V>
static sla_status grad_v(const sla_csr *A, int nrhs, const void *lam, const void *x, void *g,
                         cudaStream_t s)
{
    const TilePart *tp;
    SLA_TRY(ensure_tiles(const_cast<sla_csr *>(A), GRAD_D, s, &tp));
    if (tp->n_tiles == 0)
        return SLA_SUCCESS;
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_pattern_grad<V>, GRAD_T, 0);
    const int grid = std::max(1, std::min(tp->n_tiles, std::max(per_sm, 1) * A->num_sms));
    k_pattern_grad<V><<<grid, GRAD_T, 0, s>>>(view<V>(A, tp), nrhs, (const V *)lam, (const V *)x,
                                              (V *)g);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

sla_status launch_pattern_grad(const sla_csr *A, int nrhs, const void *lam, const void *x, void *g,
                               cudaStream_t s)
{
    return A->dtype == SLA_F32 ? grad_v<float>(A, nrhs, lam, x, g, s)
                               : grad_v<double>(A, nrhs, lam, x, g, s);
}

sla_status launch_validate(const sla_csr *A, int *d_err, cudaStream_t s)
{
    if (A->n == 0)
        return SLA_SUCCESS;
    k_validate<<<vec_grid(A), 256, 0, s>>>(A->n, A->rp, A->ci, A->d_sys_off, A->batch, d_err);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

sla_status launch_jacobi_dinv(const sla_csr *A, void *dinv, int *d_err, cudaStream_t s)
{
    if (A->n == 0)
        return SLA_SUCCESS;
    if (A->dtype == SLA_F32)
        k_jacobi_dinv<float><<<vec_grid(A), 256, 0, s>>>(A->n, A->rp, A->ci, (const float *)A->val,
                                                         (float *)dinv, d_err);
    else
        k_jacobi_dinv<double><<<vec_grid(A), 256, 0, s>>>(A->n, A->rp, A->ci, (const double *)A->val,
                                                          (double *)dinv, d_err);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

sla_status refresh_transpose_values(const sla_csr *G, sla_csr *GT, const int32_t *perm,
                                    cudaStream_t s)
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

// ------------------------------------------------------------------ solve plans
// The kernels of one PCG iteration for a plan, with their grids and operands bound.
template <typename V, int K>
struct PlanKernels {
    int64_t n = 0;
    V *x, *ra, *rb, *pa, *pb, *q, *z, *y;
    const V *dinv = nullptr;
    PcgState *st;
    double *part;
    MatView<V> mA{}, mG{}, mGT{};
    int gA = 0, gG = 0, gGT = 0, gv = 0;

    sla_status bind(sla_csr *A, Plan *p, cudaStream_t s)
    {
        const sla_precond *M = p->M;
        n = A->n;
        const TilePart *tpA;
        SLA_TRY(ensure_tiles(A, TileCfg<K>::D, s, &tpA));
        x = (V *)p->x; ra = (V *)p->ra; rb = (V *)p->rb; pa = (V *)p->pa; pb = (V *)p->pb;
        q = (V *)p->q; z = (V *)p->z; y = (V *)p->y;
        st = p->st;
        part = p->partials;
        mA = view<V>(A, tpA);
        gA = tile_grid<K, V, OpQ<V, K>>(A, tpA);
        gv = vec_grid(A);
        if (p->kind == 1)
            dinv = (const V *)M->d_dinv;
        else if (p->kind == 0)
            dinv = (const V *)p->y;  // ones (y is unused without SPAI)
        if (p->kind == 2) {
            const TilePart *tpG, *tpGT;
            SLA_TRY(ensure_tiles(const_cast<sla_csr *>(M->G), TileCfg<K>::D, s, &tpG));
            SLA_TRY(ensure_tiles(M->GT, TileCfg<K>::D, s, &tpGT));
            mG = view<V>(M->G, tpG);
            mGT = view<V>(M->GT, tpGT);
            gG = tile_grid<K, V, OpZ<V, K>>(M->G, tpG);
            gGT = tile_grid<K, V, OpUS<V, K>>(M->GT, tpGT);
        }
        p->grid_tiles_A = gA;
        p->grid_tiles_G = gG;
        p->grid_tiles_GT = gGT;
        p->grid_vec = gv;
        return SLA_SUCCESS;
    }
    void Q(cudaStream_t s, const V *pold, V *pnew) const
    {
        OpQ<V, K> op{z, pold, pnew, q, st};
        k_tile<K, V, OpQ<V, K>><<<gA, TileCfg<K>::T, 0, s>>>(mA, op, part, st);
    }
    void UJ(cudaStream_t s, const V *pcur) const
    {
        k_update_jacobi<V, K><<<gv, VEC_T, 0, s>>>(n, x, ra, pcur, q, z, dinv, part, st);
    }
    void US(cudaStream_t s, const V *rold, V *rnew, const V *pcur) const
    {
        OpUS<V, K> op{rold, q, pcur, rnew, x, y, st};
        k_tile<K, V, OpUS<V, K>><<<gGT, TileCfg<K>::T, 0, s>>>(mGT, op, part, st);
    }
    void Z(cudaStream_t s, const V *rcur) const
    {
        OpZ<V, K> op{y, rcur, z, st};
        k_tile<K, V, OpZ<V, K>><<<gG, TileCfg<K>::T, 0, s>>>(mG, op, part, st);
    }
};

template <typename V, int K>
static sla_status capture_k(sla_csr *A, Plan *p)
{
    PlanKernels<V, K> kr;
    SLA_TRY(kr.bind(A, p, p->cs));
    SLA_CUDA_TRY(cudaStreamSynchronize(p->cs));
    V *ra = kr.ra, *rb = kr.rb, *pa = kr.pa, *pb = kr.pb;

    cudaGraph_t g = nullptr;
    SLA_CUDA_TRY(cudaGraphCreate(&g, 0));
    p->graph = g;
    cudaGraphConditionalHandle h;
    SLA_CUDA_TRY(cudaGraphConditionalHandleCreate(&h, g, 1, cudaGraphCondAssignDefault));
    p->cond = (unsigned long long)h;

    // prologue: the initial pass computes ||b||, z = M^-1 b and rho = b.z
    SLA_CUDA_TRY(cudaStreamBeginCaptureToGraph(p->cs, g, nullptr, nullptr, 0,
                                               cudaStreamCaptureModeThreadLocal));
    if (p->kind == 2) {
        kr.US(p->cs, ra, rb, pa);
        kr.Z(p->cs, rb);
    } else {
        kr.UJ(p->cs, pa);
    }
    cudaStreamCaptureStatus cst;
    const cudaGraphNode_t *deps = nullptr;
    size_t ndeps = 0;
    cudaGraph_t gcap = nullptr;
    SLA_CUDA_TRY(cudaStreamGetCaptureInfo(p->cs, &cst, nullptr, &gcap, &deps, &ndeps));
    cudaGraphNodeParams cp = {cudaGraphNodeTypeConditional};
    cp.conditional.handle = h;
    cp.conditional.type = cudaGraphCondTypeWhile;
    cp.conditional.size = 1;
    cudaGraphNode_t cnode;
    SLA_CUDA_TRY(cudaGraphAddNode(&cnode, gcap, deps, ndeps, &cp));
    SLA_CUDA_TRY(cudaStreamUpdateCaptureDependencies(p->cs, &cnode, 1, cudaStreamSetCaptureDependencies));
    cudaGraph_t body = cp.conditional.phGraph_out[0];
    // loop body: two iterations, so the double-buffered vectors return to their slots
    SLA_CUDA_TRY(cudaStreamBeginCaptureToGraph(p->cs2, body, nullptr, nullptr, 0,
                                               cudaStreamCaptureModeThreadLocal));
    if (p->kind == 2) {
        kr.Q(p->cs2, pa, pb);
        kr.US(p->cs2, rb, ra, pb);
        kr.Z(p->cs2, ra);
        kr.Q(p->cs2, pb, pa);
        kr.US(p->cs2, ra, rb, pa);
        kr.Z(p->cs2, rb);
    } else {
        kr.Q(p->cs2, pa, pb);
        kr.UJ(p->cs2, pb);
        kr.Q(p->cs2, pb, pa);
        kr.UJ(p->cs2, pa);
    }
    cudaError_t e1 = cudaGetLastError();
    cudaGraph_t body_out = nullptr;
    cudaError_t e2 = cudaStreamEndCapture(p->cs2, &body_out);
    cudaGraph_t g_out = nullptr;
    cudaError_t e3 = cudaStreamEndCapture(p->cs, &g_out);
    if (e1 != cudaSuccess)
        return cuda_fail(e1, "kernel launch during capture");
    if (e2 != cudaSuccess)
        return cuda_fail(e2, "end capture (loop body)");
    if (e3 != cudaSuccess)
        return cuda_fail(e3, "end capture (solve graph)");
    SLA_CUDA_TRY(cudaGraphInstantiate(&p->exec, g, 0));
    return SLA_SUCCESS;
}

// Mean device time of each kernel of one iteration, each launch bracketed by events in
// the order the loop runs them (so each sees the cache state of the real iteration).
template <typename V, int K>
static sla_status times_k(sla_csr *A, Plan *p, int nrhs, int reps, double *h_ms, cudaStream_t s)
{
    PlanKernels<V, K> kr;
    SLA_TRY(kr.bind(A, p, s));
    k_profile_mode<<<1, 1, 0, s>>>(p->st, nrhs);
    SLA_CUDA_TRY(cudaGetLastError());
    const int nk = p->kind == 2 ? 3 : 2;
    cudaEvent_t ev[4];
    for (int i = 0; i < 4; ++i)
        SLA_CUDA_TRY(cudaEventCreate(&ev[i]));
    double acc[3] = {0.0, 0.0, 0.0};
    sla_status st = SLA_SUCCESS;
    for (int r = 0; r < reps && st == SLA_SUCCESS; ++r) {
        cudaEventRecord(ev[0], s);
        kr.Q(s, kr.pa, kr.pb);
        cudaEventRecord(ev[1], s);
        if (p->kind == 2) {
            kr.US(s, kr.rb, kr.ra, kr.pb);
            cudaEventRecord(ev[2], s);
            kr.Z(s, kr.ra);
            cudaEventRecord(ev[3], s);
        } else {
            kr.UJ(s, kr.pb);
            cudaEventRecord(ev[2], s);
        }
        cudaError_t e = cudaEventSynchronize(ev[nk]);
        if (e != cudaSuccess) {
            st = cuda_fail(e, "kernel timing");
            break;
        }
        for (int i = 0; i < nk; ++i) {
            float ms = 0.f;
            cudaEventElapsedTime(&ms, ev[i], ev[i + 1]);
            acc[i] += ms;
        }
    }
    for (int i = 0; i < 4; ++i)
        cudaEventDestroy(ev[i]);
    for (int i = 0; i < 3; ++i)
        h_ms[i] = i < nk ? acc[i] / std::max(reps, 1) : 0.0;
    return st;
}

template <typename V>
static sla_status capture_v(sla_csr *A, Plan *p)
{
    switch (p->K) {
    case 1: return capture_k<V, 1>(A, p);
    case 2: return capture_k<V, 2>(A, p);
    case 4: return capture_k<V, 4>(A, p);
    case 8: return capture_k<V, 8>(A, p);
    case 16: return capture_k<V, 16>(A, p);
    default: return fail(SLA_ERR_INVALID_ARG, "unsupported right-hand-side count");
    }
}

sla_status capture_plan_graph(sla_csr *A, Plan *p)
{
    return A->dtype == SLA_F32 ? capture_v<float>(A, p) : capture_v<double>(A, p);
}

template <typename V>
static sla_status times_v(sla_csr *A, Plan *p, int nrhs, int reps, double *h_ms, cudaStream_t s)
{
    switch (p->K) {
    case 1: return times_k<V, 1>(A, p, nrhs, reps, h_ms, s);
    case 2: return times_k<V, 2>(A, p, nrhs, reps, h_ms, s);
    case 4: return times_k<V, 4>(A, p, nrhs, reps, h_ms, s);
    case 8: return times_k<V, 8>(A, p, nrhs, reps, h_ms, s);
    case 16: return times_k<V, 16>(A, p, nrhs, reps, h_ms, s);
    default: return fail(SLA_ERR_INVALID_ARG, "unsupported right-hand-side count");
    }
}

sla_status kernel_times(sla_csr *A, Plan *p, int nrhs, int reps, double *h_ms, cudaStream_t s)
{
    return A->dtype == SLA_F32 ? times_v<float>(A, p, nrhs, reps, h_ms, s)
                               : times_v<double>(A, p, nrhs, reps, h_ms, s);
}

template <typename V>
__global__ void k_fill(int64_t n, V *a, V v)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        a[i] = v;
}

template <typename V, int K>
static sla_status run_k(sla_csr *A, Plan *p, int nrhs, const void *B, void *X,
                        double tol, long long maxit, cudaStream_t s)
{
    const int64_t n = A->n;
    const int gv = vec_grid(A);
    V *y = (V *)p->y;
    if (p->kind == 0) {
        // without a preconditioner the Jacobi kernel runs with D^-1 = 1 (held in y)
        k_fill<V><<<gv, 256, 0, s>>>(n, y, (V)1);
        y = nullptr;
    }
    k_init<V, K><<<gv, 256, 0, s>>>(n, nrhs, (const V *)B, (V *)p->x, (V *)p->ra, (V *)p->pa,
                                    (V *)p->q, (V *)p->z, p->kind == 2 ? y : nullptr, p->st, tol,
                                    maxit, p->M ? p->M->eps : 0.0, p->cond, 1);
    SLA_CUDA_TRY(cudaGetLastError());
    SLA_CUDA_TRY(cudaGraphLaunch(p->exec, s));
    k_copy_out<V, K><<<gv, 256, 0, s>>>(n, nrhs, (const V *)p->x, (V *)X);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

template <typename V>
static sla_status run_v(sla_csr *A, Plan *p, int nrhs, const void *B, void *X, double tol,
                        long long maxit, cudaStream_t s)
{
    switch (p->K) {
    case 1: return run_k<V, 1>(A, p, nrhs, B, X, tol, maxit, s);
    case 2: return run_k<V, 2>(A, p, nrhs, B, X, tol, maxit, s);
    case 4: return run_k<V, 4>(A, p, nrhs, B, X, tol, maxit, s);
    case 8: return run_k<V, 8>(A, p, nrhs, B, X, tol, maxit, s);
    case 16: return run_k<V, 16>(A, p, nrhs, B, X, tol, maxit, s);
    default: return fail(SLA_ERR_INVALID_ARG, "unsupported right-hand-side count");
    }
}

sla_status run_plan(sla_csr *A, Plan *p, int nrhs, const void *B, void *X,
                    const sla_pcg_opts *opts, sla_pcg_info *info, const void *grad_x,
                    void *grad_out, cudaStream_t s)
{
    double tol = (opts && opts->rtol > 0) ? opts->rtol : (A->dtype == SLA_F32 ? 1e-6 : 1e-10);
    long long n_sys = A->batch > 1 ? A->max_sys_n : A->n;
    long long maxit = (opts && opts->maxit > 0) ? opts->maxit : 10 * std::max<long long>(n_sys, 1);
    sla_status st = A->dtype == SLA_F32 ? run_v<float>(A, p, nrhs, B, X, tol, maxit, s)
                                        : run_v<double>(A, p, nrhs, B, X, tol, maxit, s);
    if (st != SLA_SUCCESS)
        return st;
    if (grad_out)
        SLA_TRY(launch_pattern_grad(A, nrhs, X, grad_x, grad_out, s));
    SLA_CUDA_TRY(cudaMemcpyAsync(p->h_st, p->st, sizeof(PcgState), cudaMemcpyDeviceToHost, s));
    SLA_CUDA_TRY(cudaStreamSynchronize(s));
    sla_status worst = SLA_SUCCESS;
    for (int c = 0; c < nrhs; ++c) {
        if (info) {
            info[c].iters = p->h_st->iters[c];
            info[c].relres = p->h_st->relres[c];
            info[c].status = p->h_st->status[c];
            info[c].reserved = 0;
        }
        worst = std::max(worst, (sla_status)p->h_st->status[c]);
    }
    return worst;
}

}  // namespace sla
