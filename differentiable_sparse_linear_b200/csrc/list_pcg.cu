// PCG over a batch of independent small SPD systems with distinct patterns (the
// SparseTensorList batch of "torch-sla: Differentiable Sparse Linear Algebra with Adjoint
// Solvers and Sparse Tensor Parallelism for PyTorch", Methodology §1), forward and adjoint.
//
// One block owns one system for its whole solve: the system's vectors (x, r, p, q, D^-1,
// for the adjoint the forward x, and with SPAI z and y = G^T r) and its row offsets live in
// shared memory, so the only HBM traffic is the system's matrix (re-read from L2 after the
// first iteration), b, and the results.  Systems too large for shared memory keep the same vectors in a device
// workspace (nv values per row of the batch), with the same code and order of operations.
// Preconditioners: Jacobi, none, or SPAI z = G (G^T r) + eps r ([SPAI] "Learning Sparse
// Approximate Inverse Preconditioners for Conjugate Gradient Solvers on GPUs", Approach)
// with G block-diagonal on the list's systems (checked when the preconditioner is made).
// Dot products are block reductions in fp64 with a fixed order; each system has its own
// stopping test, iteration count and status.  There is no grid-wide dependency, so the
// whole batch is one launch and needs no graph.
#include <cuda_runtime.h>

#include <algorithm>

#include "sla_internal.cuh"

namespace sla {

constexpr int LIST_T = 512;

// Sum two values over the block; every thread receives both totals.
__device__ __forceinline__ void list_sum2(double &a, double &b, double *s_red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        a += __shfl_down_sync(0xffffffffu, a, off);
        b += __shfl_down_sync(0xffffffffu, b, off);
    }
    if (lane == 0) {
        s_red[2 * warp] = a;
        s_red[2 * warp + 1] = b;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double ta = 0.0, tb = 0.0;
        for (int w = 0; w < LIST_T / 32; ++w) {
            ta += s_red[2 * w];
            tb += s_red[2 * w + 1];
        }
        s_red[2 * (LIST_T / 32)] = ta;
        s_red[2 * (LIST_T / 32) + 1] = tb;
    }
    __syncthreads();
    a = s_red[2 * (LIST_T / 32)];
    b = s_red[2 * (LIST_T / 32) + 1];
    __syncthreads();
}

// q = A p on one system (rows [0, ns), local columns = global - o0), S lanes per row;
// `rpl` holds the system's row offsets (rpl[i] = first entry of local row i).  Each lane
// group takes LIST_RU rows at once, so every lane has that many independent loads in
// flight; a row's terms are still summed in entry order.  The trip count is the same for
// every lane of a warp (the shuffles need the whole warp).  Returns this thread's share of
// p.q (only the first lane of each row group contributes; 0 without DOT).
constexpr int LIST_RU = 4;

template <typename V, int S, bool DOT = true>
__device__ __forceinline__ double list_spmv(int ns, int64_t o0, const int32_t *rpl, const int32_t *ci,
                                            const V *val, const V *p, V *q)
{
    constexpr int NG = LIST_T / S;
    const int lane = threadIdx.x & (S - 1);
    const int grp = threadIdx.x / S;
    const int gw = grp & ~(32 / S - 1);            // first row group of this warp
    double part = 0.0;
    for (int t0 = 0; gw + t0 < ns; t0 += NG * LIST_RU) {
        uint32_t k[LIST_RU], k1[LIST_RU];          // entry offsets (< 2^31, so k + S cannot wrap)
        double acc[LIST_RU];
#pragma unroll
        for (int u = 0; u < LIST_RU; ++u) {
            const int i = grp + t0 + u * NG;
            k[u] = i < ns ? (uint32_t)rpl[i] + lane : 0u;
            k1[u] = i < ns ? (uint32_t)rpl[i + 1] : 0u;
            acc[u] = 0.0;
        }
        bool more = true;
        while (more) {
            V a[LIST_RU];
            int32_t c[LIST_RU];
#pragma unroll
            for (int u = 0; u < LIST_RU; ++u) {
                const bool in = k[u] < k1[u];
                a[u] = in ? val[k[u]] : (V)0;
                c[u] = in ? ci[k[u]] : -1;
            }
            more = false;
#pragma unroll
            for (int u = 0; u < LIST_RU; ++u) {
                if (c[u] >= 0)
                    acc[u] = __fma_rn((double)a[u], (double)p[c[u] - o0], acc[u]);
                k[u] += S;
                more |= k[u] < k1[u];
            }
        }
#pragma unroll
        for (int u = 0; u < LIST_RU; ++u)
#pragma unroll
            for (int off = S / 2; off > 0; off >>= 1)
                acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], off, S);
        if (lane == 0) {
#pragma unroll
            for (int u = 0; u < LIST_RU; ++u) {
                const int i = grp + t0 + u * NG;
                if (i < ns) {
                    const V qv = (V)acc[u];
                    q[i] = qv;
                    if (DOT)
                        part += (double)p[i] * (double)qv;
                }
            }
        }
    }
    return part;
}

// The SPAI factor of a list (block-diagonal G and its explicit transpose) for the kernel.
template <typename V>
struct ListSpai {
    const int32_t *g_rp, *g_ci;
    const V *g_val;
    const int32_t *gt_rp, *gt_ci;
    const V *gt_val;
    double eps;
};

// z = G (G^T r) + eps r on one system; returns this thread's share of r.z.  Ends with the
// block synchronised.
template <typename V, int S>
__device__ __forceinline__ double list_spai_apply(int ns, int64_t o0, const ListSpai<V> &m, const V *r, V *y,
                                                  V *z)
{
    list_spmv<V, S, false>(ns, o0, m.gt_rp + o0, m.gt_ci, m.gt_val, r, y);
    __syncthreads();
    list_spmv<V, S, false>(ns, o0, m.g_rp + o0, m.g_ci, m.g_val, y, z);
    __syncthreads();
    double rz = 0.0;
    for (int i = threadIdx.x; i < ns; i += LIST_T) {
        const V zi = (V)__fma_rn(m.eps, (double)r[i], (double)z[i]);
        z[i] = zi;
        rz += (double)r[i] * (double)zi;
    }
    return rz;
}

// Vectors a system keeps (per row): x, r, p, q, then D^-1 (Jacobi), z and y = G^T r (SPAI),
// the forward x (adjoint); without SPAI z = D^-1 r is formed where it is used, not stored.
// In shared memory the system's row offsets follow the vectors.
__host__ __device__ inline int list_nv(bool jacobi, bool spai, bool adjoint)
{
    return 4 + (jacobi ? 1 : 0) + (spai ? 2 : 0) + (adjoint ? 1 : 0);
}

template <typename V, int S>
__global__ void __launch_bounds__(LIST_T, 3)
k_list_pcg(const int32_t *rp, const int32_t *ci, const V *val, const int64_t *sys_off, int batch,
           const V *B, V *X, const V *dinv, const V *Xf, V *Gout, double tol, long long maxit_opt,
           sla_pcg_info *info, const ListSpai<V> spai, int use_spai, V *ws)
{
    extern __shared__ __align__(16) unsigned char s_raw[];
    __shared__ double s_red[2 * (LIST_T / 32) + 2];
    const int tid = threadIdx.x;
    const bool jac = dinv != nullptr;
    const int nv = list_nv(jac, use_spai, Xf != nullptr);
    for (int s = blockIdx.x; s < batch; s += gridDim.x) {
        const int64_t o0 = sys_off[s];
        const int ns = (int)(sys_off[s + 1] - o0);
        V *x = ws ? ws + (int64_t)nv * o0 : (V *)s_raw;
        V *r = x + ns;
        V *p = r + ns;
        V *q = p + ns;
        V *nxt = q + ns;
        V *dv = nullptr, *z = nullptr, *y = nullptr, *xf = nullptr;
        if (jac) {
            dv = nxt;
            nxt += ns;
        }
        if (use_spai) {
            z = nxt;
            y = nxt + ns;
            nxt += 2 * ns;
        }
        if (Xf) {
            xf = nxt;
            nxt += ns;
        }
        // the system's row offsets: staged in shared memory after the vectors
        const int32_t *rpl = rp + o0;
        if (!ws) {
            int32_t *s_rp = (int32_t *)(s_raw + (size_t)nv * ns * sizeof(V));
            for (int i = tid; i <= ns; i += LIST_T)
                s_rp[i] = rp[o0 + i];
            rpl = s_rp;
        }
        const long long maxit = maxit_opt > 0 ? maxit_opt : 10LL * (ns > 0 ? ns : 1);

        double bb = 0.0, rz = 0.0;
        for (int i = tid; i < ns; i += LIST_T) {
            const V bi = B[o0 + i];
            x[i] = (V)0;
            r[i] = bi;
            if (!use_spai) {
                const V di = jac ? dinv[o0 + i] : (V)1;
                const V zi = (V)((double)bi * (double)di);
                if (jac)
                    dv[i] = di;
                p[i] = zi;
                rz += (double)bi * (double)zi;
            }
            if (Xf)
                xf[i] = Xf[o0 + i];
            bb += (double)bi * (double)bi;
        }
        __syncthreads();
        if (use_spai) {
            rz = list_spai_apply<V, S>(ns, o0, spai, r, y, z);
            for (int i = tid; i < ns; i += LIST_T)
                p[i] = z[i];
        }
        list_sum2(bb, rz, s_red);
        const double bnorm = sqrt(bb);
        double rho = rz;
        long long it = 0;
        double relres = bnorm > 0.0 ? 1.0 : 0.0;
        int status = SLA_NOT_CONVERGED;
        if (!isfinite(bnorm))
            status = SLA_BREAKDOWN;
        else if (bnorm == 0.0)
            status = SLA_SUCCESS;
        else if (!(rho > 0.0) || !isfinite(rho))
            status = SLA_BREAKDOWN;
        else {
            while (it < maxit) {
                ++it;
                double pq = list_spmv<V, S>(ns, o0, rpl, ci, val, p, q), dummy = 0.0;
                list_sum2(pq, dummy, s_red);
                if (!(pq > 0.0) || !isfinite(pq)) {
                    status = SLA_BREAKDOWN;
                    break;
                }
                const double alpha = rho / pq;
                double rr = 0.0, rzn = 0.0;
                for (int i = tid; i < ns; i += LIST_T) {
                    x[i] = (V)__fma_rn(alpha, (double)p[i], (double)x[i]);
                    const V rn = (V)__fma_rn(-alpha, (double)q[i], (double)r[i]);
                    r[i] = rn;
                    rr += (double)rn * (double)rn;
                    if (!use_spai) {
                        const V zn = jac ? (V)((double)rn * (double)dv[i]) : rn;
                        rzn += (double)rn * (double)zn;
                    }
                }
                if (use_spai) {
                    // stopping test first (on r.r), then z = M^-1 r: the apply is skipped on
                    // the last iteration, as in the single-system solvers
                    double dummy = 0.0;
                    list_sum2(rr, dummy, s_red);
                    relres = sqrt(rr) / bnorm;
                    if (isfinite(relres) && relres > tol) {
                        rzn = list_spai_apply<V, S>(ns, o0, spai, r, y, z);
                        list_sum2(rzn, dummy, s_red);
                    }
                } else {
                    list_sum2(rr, rzn, s_red);
                }
                relres = sqrt(rr) / bnorm;
                if (!isfinite(relres)) {
                    status = SLA_BREAKDOWN;
                    break;
                }
                if (relres <= tol) {
                    status = SLA_SUCCESS;
                    break;
                }
                if (!(rzn > 0.0) || !isfinite(rzn)) {
                    status = SLA_BREAKDOWN;
                    break;
                }
                const double beta = rzn / rho;
                rho = rzn;
                if (use_spai) {
                    for (int i = tid; i < ns; i += LIST_T)
                        p[i] = (V)__fma_rn(beta, (double)p[i], (double)z[i]);
                } else {
                    for (int i = tid; i < ns; i += LIST_T) {
                        const V zi = jac ? (V)((double)r[i] * (double)dv[i]) : r[i];
                        p[i] = (V)__fma_rn(beta, (double)p[i], (double)zi);
                    }
                }
                __syncthreads();
            }
        }
        __syncthreads();
        for (int i = tid; i < ns; i += LIST_T)
            X[o0 + i] = x[i];
        if (Gout) {
            // dL/dA_ij = -lambda_i x_j on the system's pattern (lambda = this solve's x)
            const int lane = tid & (S - 1), grp = tid / S;
            for (int i = grp; i < ns; i += LIST_T / S) {
                const double li = (double)x[i];
                for (int64_t k = rpl[i] + lane; k < rpl[i + 1]; k += S)
                    Gout[k] = (V)(-li * (double)xf[ci[k] - o0]);
            }
        }
        if (tid == 0) {
            info[s].iters = it;
            info[s].relres = relres;
            info[s].status = status;
            info[s].engine = SLA_ENGINE_LIST;
        }
        __syncthreads();
    }
}

// Shared memory a system's vectors and row offsets take; above LIST_SMEM_MAX the vectors
// live in a workspace instead.
constexpr size_t LIST_SMEM_MAX = 200 * 1024;

static int list_nv_of(const sla_precond *M, bool adjoint)
{
    return list_nv(M && M->kind == 1, M && M->kind == 2, adjoint);
}

static size_t list_smem(const sla_csr *A, int nv)
{
    return (size_t)nv * (size_t)A->max_sys_n * (A->dtype == SLA_F32 ? 4 : 8) +
           ((size_t)A->max_sys_n + 1) * sizeof(int32_t);
}

template <typename V, int S>
static sla_status list_launch(const sla_csr *A, const V *dinv, const ListSpai<V> &spai, int use_spai, V *ws,
                              const void *B, void *X, const void *Xf, void *G, double tol, long long maxit,
                              sla_pcg_info *d_info, bool timed, cudaStream_t s)
{
    const size_t shm = ws ? 0 : list_smem(A, list_nv(dinv != nullptr, use_spai != 0, Xf != nullptr));
    auto kern = k_list_pcg<V, S>;
    SLA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm));
    int per_sm = 0;
    SLA_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, LIST_T, shm));
    if (per_sm < 1)
        return fail(SLA_ERR_UNSUPPORTED, "list solve: a system's vectors do not fit in shared memory");
    const int grid = std::min<int64_t>(A->batch, (int64_t)per_sm * A->num_sms);
    sla_csr *Am = const_cast<sla_csr *>(A);
    Am->list_ev_recorded = 0;
    if (timed) {
        for (cudaEvent_t &ev : Am->list_ev)
            if (!ev)
                SLA_CUDA_TRY(cudaEventCreate(&ev));
        SLA_CUDA_TRY(cudaEventRecord(Am->list_ev[0], s));
    }
    kern<<<grid, LIST_T, shm, s>>>(A->rp, A->ci, (const V *)A->val, A->d_sys_off, A->batch,
                                   (const V *)B, (V *)X, dinv, (const V *)Xf, (V *)G, tol, maxit,
                                   d_info, spai, use_spai, ws);
    SLA_CUDA_TRY(cudaGetLastError());
    if (timed) {
        SLA_CUDA_TRY(cudaEventRecord(Am->list_ev[1], s));
        Am->list_ev_recorded = 1;
    }
    return SLA_SUCCESS;
}

template <typename V>
static sla_status list_v(const sla_csr *A, const sla_precond *M, V *ws, const void *B, void *X, const void *Xf,
                         void *G, double tol, long long maxit, sla_pcg_info *d_info, bool timed, cudaStream_t s)
{
    const V *dinv = nullptr;
    ListSpai<V> sp{};
    int use_spai = 0;
    if (M && M->kind == 1) {
        dinv = (const V *)(sizeof(V) == 4 ? M->d_dinv : M->d_dinv64);
    } else if (M && M->kind == 2) {
        sp = ListSpai<V>{M->G->rp, M->G->ci, (const V *)M->G->val, M->GT->rp, M->GT->ci, (const V *)M->GT->val,
                         M->eps};
        use_spai = 1;
    }
    const double mean = A->n > 0 ? (double)A->nnz / (double)A->n : 0.0;
    if (mean <= 6.0)
        return list_launch<V, 4>(A, dinv, sp, use_spai, ws, B, X, Xf, G, tol, maxit, d_info, timed, s);
    if (mean <= 24.0)
        return list_launch<V, 8>(A, dinv, sp, use_spai, ws, B, X, Xf, G, tol, maxit, d_info, timed, s);
    if (mean <= 64.0)
        return list_launch<V, 16>(A, dinv, sp, use_spai, ws, B, X, Xf, G, tol, maxit, d_info, timed, s);
    return list_launch<V, 32>(A, dinv, sp, use_spai, ws, B, X, Xf, G, tol, maxit, d_info, timed, s);
}

static sla_status list_check_precond(const sla_precond *M)
{
    if (M && M->kind == 2 && (!M->G || !M->GT))
        return fail(SLA_ERR_INVALID_ARG, "the SPAI preconditioner's G was destroyed");
    return SLA_SUCCESS;
}

// Forward (Xf == nullptr) or adjoint (Xf = forward solution, B = dL/dx, X = dL/db,
// G = dL/dA or nullptr) over every system of a list handle.
sla_status run_list_solve(const sla_csr *A, const sla_precond *M, const void *B, void *X,
                          const void *Xf, void *G, const sla_pcg_opts *opts, sla_pcg_info *info,
                          cudaStream_t s)
{
    SLA_TRY(list_check_precond(M));
    const double tol = (opts && opts->rtol > 0) ? opts->rtol : (A->dtype == SLA_F32 ? 1e-6 : 1e-10);
    const long long maxit = (opts && opts->maxit > 0) ? opts->maxit : 0;
    sla_pcg_info *d_info = nullptr;
    SLA_CUDA_TRY(cudaMallocAsync((void **)&d_info, sizeof(sla_pcg_info) * (size_t)A->batch, s));
    // systems whose vectors do not fit in shared memory: a workspace of nv values per row
    const int nv = list_nv_of(M, Xf != nullptr);
    void *ws = nullptr;
    cudaError_t we = cudaSuccess;
    if (list_smem(A, nv) > LIST_SMEM_MAX && A->n > 0)
        we = cudaMallocAsync(&ws, (size_t)nv * (size_t)A->n * (A->dtype == SLA_F32 ? 4 : 8), s);
    sla_status st;
    if (we != cudaSuccess)
        st = fail(SLA_ERR_OOM, "list solve: workspace allocation");
    else if (A->dtype == SLA_F32)
        st = list_v<float>(A, M, (float *)ws, B, X, Xf, G, tol, maxit, d_info, true, s);
    else
        st = list_v<double>(A, M, (double *)ws, B, X, Xf, G, tol, maxit, d_info, true, s);
    if (ws)
        cudaFreeAsync(ws, s);
    if (st == SLA_SUCCESS) {
        cudaError_t e = cudaMemcpyAsync(info, d_info, sizeof(sla_pcg_info) * (size_t)A->batch,
                                        cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess)
            e = cudaStreamSynchronize(s);
        if (e != cudaSuccess)
            st = cuda_fail(e, "list solve result copy");
    }
    cudaFreeAsync(d_info, s);
    if (st != SLA_SUCCESS)
        return st;
    sla_status worst = SLA_SUCCESS;
    for (int i = 0; i < A->batch; ++i)
        worst = std::max(worst, (sla_status)info[i].status);
    return worst;
}

// *err = 1 if a row of M stores a column outside its system's range (block-diagonal check
// of a list's SPAI factor against the list's system offsets).
__global__ void k_check_blocks(int64_t n, const int32_t *rp, const int32_t *ci, const int64_t *sys_off,
                               int batch, int *err)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        int lo = 0, hi = batch - 1;                 // the system holding row i
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (sys_off[mid] <= i)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int64_t a = sys_off[lo], b = sys_off[lo + 1];
        for (int64_t k = rp[i]; k < rp[i + 1]; ++k)
            if (ci[k] < a || ci[k] >= b)
                atomicOr(err, 1);
    }
}

sla_status check_list_blocks(const sla_csr *A, const sla_csr *M, cudaStream_t s)
{
    if (M->n != A->n)
        return fail(SLA_ERR_INVALID_ARG, "the factor must have the list's size");
    if (A->n == 0)
        return SLA_SUCCESS;
    int *d_err = nullptr;
    SLA_CUDA_TRY(cudaMallocAsync((void **)&d_err, sizeof(int), s));
    cudaError_t e = cudaMemsetAsync(d_err, 0, sizeof(int), s);
    const int grid = (int)std::min<int64_t>((A->n + 255) / 256, (int64_t)A->num_sms * 8);
    if (e == cudaSuccess) {
        k_check_blocks<<<grid, 256, 0, s>>>(M->n, M->rp, M->ci, A->d_sys_off, A->batch, d_err);
        e = cudaGetLastError();
    }
    int h = 0;
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(&h, d_err, sizeof(int), cudaMemcpyDeviceToHost, s);
    cudaFreeAsync(d_err, s);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(s);
    if (e != cudaSuccess)
        return cuda_fail(e, "block-diagonal check of the SPAI factor");
    if (h)
        return fail(SLA_ERR_INVALID_ARG, "for a list handle, G must be block-diagonal on the list's systems");
    return SLA_SUCCESS;
}

}  // namespace sla

namespace sla {

// The list kernel with a caller-provided device array for the per-system results (no
// allocation here); the caller copies the results back and synchronises.
sla_status launch_list_kernel(const sla_csr *A, const sla_precond *M, const void *B, void *X,
                              const sla_pcg_opts *opts, sla_pcg_info *d_info, cudaStream_t s)
{
    SLA_TRY(list_check_precond(M));
    // this path allocates nothing: every system's vectors must fit in shared memory
    if (list_smem(A, list_nv_of(M, false)) > LIST_SMEM_MAX)
        return fail(SLA_ERR_UNSUPPORTED, "list solve without allocation: largest system exceeds the shared-memory size");
    const double tol = (opts && opts->rtol > 0) ? opts->rtol : (A->dtype == SLA_F32 ? 1e-6 : 1e-10);
    const long long maxit = (opts && opts->maxit > 0) ? opts->maxit : 0;
    if (A->dtype == SLA_F32)
        return list_v<float>(A, M, (float *)nullptr, B, X, nullptr, nullptr, tol, maxit, d_info, false, s);
    return list_v<double>(A, M, (double *)nullptr, B, X, nullptr, nullptr, tol, maxit, d_info, false, s);
}

}  // namespace sla

using namespace sla;

extern "C" sla_status sla_list_kernel_ms(const sla_csr *A, double *h_ms)
{
    if (!A || !h_ms)
        return fail(SLA_ERR_INVALID_ARG, "NULL argument");
    if (A->batch < 1 || A->sys_off.empty() || !A->list_ev_recorded)
        return fail(SLA_ERR_INVALID_ARG, "no list solve has run on this handle");
    SLA_CUDA_TRY(cudaEventSynchronize(A->list_ev[1]));
    float ms = 0.f;
    SLA_CUDA_TRY(cudaEventElapsedTime(&ms, A->list_ev[0], A->list_ev[1]));
    *h_ms = (double)ms;
    return SLA_SUCCESS;
}
