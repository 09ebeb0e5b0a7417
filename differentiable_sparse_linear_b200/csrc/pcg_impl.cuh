// Templates of the PCG solver kernels, shared by the per-precision translation units
// (pcg_ff.cu: fp32 values and vectors; pcg_dd.cu: fp64; pcg_fd.cu: fp32 values, fp64
// vectors).  See pcg_dispatch.cu for the method and the kernel schedule.
#pragma once

#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "sla_internal.cuh"
#include "pcg_ops.cuh"
#include "persist.cuh"
#include "row_engine.cuh"
#include "tile_engine.cuh"
#include "bsr.cuh"
#include "csb.cuh"

#include <type_traits>

namespace sla {

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
    __shared__ double s_sum[2 * K];
    __shared__ int s_flag;
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
    for (int64_t i = (int64_t)blockIdx.x * VEC_T + threadIdx.x; i < n; i += stride)
        jacobi_row<V, K>(i, x, r, p, q, z, dinv, s_a, s_on, part);
    UJFinal fin{st, K};
    auto sync = [] { __syncthreads(); };
    grid_reduce_finalize<VEC_T, 2 * K>(part, partials, st, fin, s_red, &s_flag, s_sum, (int)threadIdx.x, sync);
}

// E_p: p_new = z + beta p_old (all rows, K columns).
template <typename V, int K>
__global__ void __launch_bounds__(VEC_T)
k_ep(int64_t n, const V *z, const V *p_old, V *p_new, PcgState *st)
{
    __shared__ double s_b[K];
    if (*(volatile int *)&st->all_done)
        return;
    if (threadIdx.x < K)
        s_b[threadIdx.x] = st->beta[threadIdx.x];
    __syncthreads();
    using IO = RowIO<V, K>;
    const int64_t stride = (int64_t)gridDim.x * VEC_T;
    int64_t i0 = (int64_t)blockIdx.x * VEC_T + threadIdx.x;
    if constexpr (K == 1) {
        // one right-hand side: 16-byte loads and stores where the vectors allow them
        using L = typename std::conditional<sizeof(V) == 4, float4, double2>::type;
        constexpr int VW = 16 / sizeof(V);
        if ((((uintptr_t)z | (uintptr_t)p_old | (uintptr_t)p_new) & 15) == 0) {
            const int64_t n4 = n / VW;
            for (int64_t j = i0; j < n4; j += stride) {
                L zz = reinterpret_cast<const L *>(z)[j], pp = reinterpret_cast<const L *>(p_old)[j], pn;
                const V *zv = reinterpret_cast<const V *>(&zz), *pv = reinterpret_cast<const V *>(&pp);
                V *nv = reinterpret_cast<V *>(&pn);
#pragma unroll
                for (int e = 0; e < VW; ++e)
                    nv[e] = vfma<V>(s_b[0], pv[e], zv[e]);
                reinterpret_cast<L *>(p_new)[j] = pn;
            }
            i0 += n4 * VW;
        }
    }
    for (int64_t i = i0; i < n; i += stride) {
        V zz[K], pp[K], pn[K];
        IO::load(z + i * K, zz);
        IO::load(p_old + i * K, pp);
#pragma unroll
        for (int c = 0; c < K; ++c)
            pn[c] = vfma<V>(s_b[c], pp[c], zz[c]);
        IO::store(p_new + i * K, pn);
    }
}

struct ERFinal {
    PcgState *st;
    __device__ void finalize(const double *sums) const
    {
        finalize_residual(st, sums);
        signal_if_done(st);
    }
};

// E_r: r_new = r_old - alpha q and x += alpha p in the active columns; partial r_new.r_new,
// then the stopping test (the last block).
template <typename V, int K>
__global__ void __launch_bounds__(VEC_T)
k_er(int64_t n, const V *r_old, const V *q, const V *p, V *x, V *r_new, double *partials, PcgState *st)
{
    __shared__ double s_a[K];
    __shared__ double s_on[K];
    __shared__ double s_red[(VEC_T / 32) * K];
    __shared__ double s_sum[K];
    __shared__ int s_flag;
    if (*(volatile int *)&st->all_done)
        return;
    if (threadIdx.x < K) {
        s_a[threadIdx.x] = st->alpha[threadIdx.x];
        s_on[threadIdx.x] = st->active[threadIdx.x] ? 1.0 : 0.0;
    }
    __syncthreads();
    using IO = RowIO<V, K>;
    double part[K];
#pragma unroll
    for (int c = 0; c < K; ++c)
        part[c] = 0.0;
    const int64_t stride = (int64_t)gridDim.x * VEC_T;
    int64_t i0 = (int64_t)blockIdx.x * VEC_T + threadIdx.x;
    if constexpr (K == 1) {
        // one right-hand side: 16-byte loads and stores where the vectors allow them
        using L = typename std::conditional<sizeof(V) == 4, float4, double2>::type;
        constexpr int VW = 16 / sizeof(V);
        if ((((uintptr_t)r_old | (uintptr_t)q | (uintptr_t)p | (uintptr_t)x | (uintptr_t)r_new) & 15) == 0) {
            const int64_t n4 = n / VW;
            const bool on = s_on[0] != 0.0;
            for (int64_t j = i0; j < n4; j += stride) {
                L ro = reinterpret_cast<const L *>(r_old)[j], qq = reinterpret_cast<const L *>(q)[j];
                L pp = reinterpret_cast<const L *>(p)[j], xx = reinterpret_cast<const L *>(x)[j], rn;
                const V *rov = reinterpret_cast<const V *>(&ro), *qv = reinterpret_cast<const V *>(&qq);
                const V *pv = reinterpret_cast<const V *>(&pp);
                V *xv = reinterpret_cast<V *>(&xx), *rnv = reinterpret_cast<V *>(&rn);
#pragma unroll
                for (int e = 0; e < VW; ++e) {
                    if (on) {
                        rnv[e] = vfma<V>(-s_a[0], qv[e], rov[e]);
                        xv[e] = vfma<V>(s_a[0], pv[e], xv[e]);
                    } else {
                        rnv[e] = rov[e];
                    }
                    part[0] += (double)rnv[e] * (double)rnv[e];
                }
                reinterpret_cast<L *>(r_new)[j] = rn;
                reinterpret_cast<L *>(x)[j] = xx;
            }
            i0 += n4 * VW;
        }
    }
    for (int64_t i = i0; i < n; i += stride) {
        V ro[K], qq[K], pp[K], xx[K], rn[K];
        IO::load(r_old + i * K, ro);
        IO::load(q + i * K, qq);
        IO::load(p + i * K, pp);
        IO::load(x + i * K, xx);
#pragma unroll
        for (int c = 0; c < K; ++c) {
            if (s_on[c] != 0.0) {
                rn[c] = vfma<V>(-s_a[c], qq[c], ro[c]);
                xx[c] = vfma<V>(s_a[c], pp[c], xx[c]);
            } else {
                rn[c] = ro[c];
            }
            part[c] += (double)rn[c] * (double)rn[c];
        }
        IO::store(r_new + i * K, rn);
        IO::store(x + i * K, xx);
    }
    ERFinal fin{st};
    auto sync = [] { __syncthreads(); };
    grid_reduce_finalize<VEC_T, K>(part, partials, st, fin, s_red, &s_flag, s_sum, (int)threadIdx.x, sync);
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
        st->error = 0;
        st->persistent = 0;
        st->gbar = 0ull;
        for (int i = 0; i < 4; ++i) {
            st->phase_ns[i] = 0ull;
            st->phase_cnt[i] = 0;
        }
    }
}

// Timing mode: every RHS active, finalisation off, so each kernel can be launched alone
// any number of times on the workspace the last solve left.
static __global__ void k_profile_mode(PcgState *st, int nrhs)
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

template <typename V>
__global__ void k_fill(int64_t n, V *a, V v)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        a[i] = v;
}

// ------------------------------------------------------------------ pattern gradient
// g_k = -sum_c lam[row(k)*nrhs + c] * x[col(k)*nrhs + c] over the tiles of A: the tile's
// row ends are staged in shared memory and each entry finds its row by binary search, so
// entries are read and g written with coalesced accesses, for any row-length mix.
constexpr int GRAD_T = 256;
constexpr int GRAD_D = 2048;

template <typename VM, typename VV>
__global__ void __launch_bounds__(GRAD_T)
k_pattern_grad(const MatView<VM> m, int nrhs, const VV *lam, const VV *x, VM *g, double scale)
{
    __shared__ int32_t s_rp[GRAD_D];
    for (int t = blockIdx.x; t < m.n_tiles; t += gridDim.x) {
        const int r0 = m.desc[t].x;
        const int r1 = m.desc[t + 1].x;
        const int nr = r1 - r0;
        const int64_t k0 = (int64_t)(uint32_t)m.desc[t].y;
        const int nk = (int)((int64_t)(uint32_t)m.desc[t + 1].y - k0);
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
            g[k0 + e] = (VM)(scale * s);
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------ set-up kernels
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
    m.desc = tp ? tp->d_desc : nullptr;
    m.n_tiles = tp ? tp->n_tiles : 0;
    m.n = A->n;
    m.nnz = A->nnz;
    return m;
}

// Launch configuration of one fused SpMV operation: the short-row engine when every row
// holds at most 16 entries; otherwise the lane-group engine up to 4 right-hand sides and
// the load-balanced tile engine above.
constexpr int ROWS_MAXL = 16;

template <int K, typename VM, class Op>
struct TileLaunch {
    using LR = RowTmaLayout<K, VM, typename Op::VV, Op::NG>;
    static constexpr int RTHREADS = RowTmaCfg<K>::TC + 32;
    static constexpr size_t RSMEM = RowTmaCfg<K>::NST * LR::BYTES;
    // long-row matrices: rows grouped by length, a lane group per row, up to 4 right-hand
    // sides; above that, block-owned tiles (a lane's gathers would not fit its registers)
    static constexpr bool LANE_GROUPS = K <= 4;
    int grid = 0;
    int maxl = 0;                 // 0: tile engine; -1: lane groups; -2: BSR lane groups;
                                  // -3: column-sorted segments; else the short-row MAXL
    MatView<VM> m{};
    const WinDesc *win = nullptr; // operand windows (short-row engine, K <= 2)
    GroupView gv{};               // length-grouped rows (lane-group engine)
    CsbView<VM> cv{};             // column-sorted segments
    size_t csb_smem = 0;
    int bdim = 1;                 // BSR block size (maxl == -2)

    template <int MAXL>
    sla_status setup_rows(const sla_csr *A, cudaStream_t s)
    {
        const TilePart *tp;
        SLA_TRY(ensure_tiles(const_cast<sla_csr *>(A), RowTmaCfg<K>::D,
                             RowTmaCfg<K>::TC * RowTmaCfg<K>::RPT, s, &tp));
        m = view<VM>(A, tp);
        if (RowTmaCfg<K>::WMAX > 0) {
            SLA_TRY(ensure_windows(const_cast<sla_csr *>(A), tp, RowTmaCfg<K>::WMAX, s));
            win = tp->d_win;
        }
        auto kern = k_rows_tma<K, VM, MAXL, Op>;
        SLA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RSMEM));
        int per_sm = 0;
        SLA_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, RTHREADS, RSMEM));
        per_sm = std::max(per_sm, 1);
        grid = std::max(1, std::min(tp->n_tiles, per_sm * A->num_sms));
        maxl = MAXL;
        return SLA_SUCCESS;
    }

    template <int B>
    sla_status setup_bsr(const sla_csr *A, cudaStream_t s)
    {
        const GroupPart *gp;
        SLA_TRY(ensure_groups(const_cast<sla_csr *>(A), s, &gp));
        m = view<VM>(A, nullptr);
        gv.rows = gp->d_rows;
        for (int b = 0; b <= GBINS; ++b) {
            gv.task0[b] = gp->task0[b];
            gv.pos0[b] = gp->pos0[b];
        }
        gv.n_tasks = gp->n_tasks;
        int per_sm = 0;
        SLA_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_bsr_group<K, VM, B, Op>,
                                                                   BsrCfg<K, B, VM, Op>::T, 0));
        per_sm = std::max(per_sm, 1);
        const int per_block = BsrCfg<K, B, VM, Op>::T / 32;
        grid = std::max(1, std::min((gp->n_tasks + per_block - 1) / per_block, per_sm * A->num_sms));
        bdim = B;
        maxl = -2;
        return SLA_SUCCESS;
    }

    sla_status setup(const sla_csr *A, cudaStream_t s)
    {
        if (A->bdim > 1) {
            if constexpr (LANE_GROUPS) {
                switch (A->bdim) {
                case 2: return setup_bsr<2>(A, s);
                case 3: return setup_bsr<3>(A, s);
                case 4: return setup_bsr<4>(A, s);
                default: return fail(SLA_ERR_INVALID_ARG, "BSR block size must be 2, 3 or 4");
                }
            }
            return fail(SLA_ERR_INVALID_ARG, "a BSR matrix takes at most 4 right-hand sides");
        }
        if (A->max_row_len <= ROWS_MAXL) {
            if (A->max_row_len <= 4)
                return setup_rows<4>(A, s);
            if (A->max_row_len <= 6)
                return setup_rows<6>(A, s);
            if (A->max_row_len <= 8)
                return setup_rows<8>(A, s);
            return setup_rows<16>(A, s);
        }
        int per_sm = 0;
        // one right-hand side, one gathered vector: the column-sorted segments, for the
        // solver's operations (solves gather the values first) and for the caller-facing
        // product when the handle's values are declared static (otherwise that product reads
        // the CSR values, which may change between calls)
        if constexpr (K == 1 && Op::NG == 1) {
            if (A->batch == 1 && (!any_ld<Op>::value || (A->flags & SLA_STATIC_VALUES))) {
                const CsbPart *cp;
                SLA_TRY(ensure_csb(const_cast<sla_csr *>(A), s, &cp));
                cv.seg_row0 = cp->d_seg_row0;
                cv.seg_ch0 = cp->d_seg_ch0;
                cv.cbase = cp->d_cbase;
                cv.pk = cp->d_pk;
                cv.val = (const VM *)cp->d_val;
                cv.n_seg = cp->n_seg;
                cv.rmax = std::max(cp->rmax, 1);
                cv.seg_bound = cp->d_seg_bound;
                // exact fixed-point row sums for fp32 values and vectors
                cv.vmax = (sizeof(VM) == 4 && sizeof(typename Op::VV) == 4) ? cp->d_vmax : nullptr;
                cv.vmax_n = cp->vmax_n;
                cv.lb = cp->lb;
                // fp64 row sums, or three 32-bit fixed-point words per row
                csb_smem = (size_t)std::max(cp->rmax, 1) * (cv.vmax ? 4 * CSB_WORDS : sizeof(double));
                auto kern = k_csb<VM, Op>;
                SLA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)csb_smem));
                SLA_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, CsbCfg::T, csb_smem));
                per_sm = std::max(per_sm, 1);
                grid = std::max(1, std::min(cp->n_seg, per_sm * A->num_sms));
                m = view<VM>(A, nullptr);
                maxl = -3;
                return SLA_SUCCESS;
            }
        }
        if constexpr (LANE_GROUPS) {
            const GroupPart *gp;
            SLA_TRY(ensure_groups(const_cast<sla_csr *>(A), s, &gp));
            m = view<VM>(A, nullptr);
            gv.rows = gp->d_rows;
            for (int b = 0; b <= GBINS; ++b) {
                gv.task0[b] = gp->task0[b];
                gv.pos0[b] = gp->pos0[b];
            }
            gv.n_tasks = gp->n_tasks;
            SLA_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_rowgroup<K, VM, Op>,
                                                                       GroupCfg<K, Op>::T, 0));
            per_sm = std::max(per_sm, 1);
            const int per_block = GroupCfg<K, Op>::T / 32;
            grid = std::max(1, std::min((gp->n_tasks + per_block - 1) / per_block, per_sm * A->num_sms));
            maxl = -1;
            return SLA_SUCCESS;
        }
        const TilePart *tp;
        SLA_TRY(ensure_tiles(const_cast<sla_csr *>(A), Tile2Cfg<K>::D, Tile2Cfg<K>::RMAX, s, &tp));
        SLA_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_tile2<K, VM, Op>,
                                                                   Tile2Cfg<K>::T, 0));
        m = view<VM>(A, tp);
        per_sm = std::max(per_sm, 1);
        grid = std::max(1, std::min(tp->n_tiles, per_sm * A->num_sms));
        maxl = 0;
        return SLA_SUCCESS;
    }
    void launch(cudaStream_t s, const Op &op, double *part, PcgState *st, int *err) const
    {
        if (maxl == -3) {
            if constexpr (K == 1 && Op::NG == 1)
                if (cv.n_seg > 0) {
                    if (cv.vmax)    // max |v_j| of the gathered vector, for the fixed-point scale
                        k_vec_absmax<typename Op::VV><<<cv.vmax_n, CSB_VMAX_T, 0, s>>>(
                            m.n, op.gvec(0), const_cast<float *>(cv.vmax), st);
                    k_csb<VM, Op><<<grid, CsbCfg::T, csb_smem, s>>>(cv, op, part, st);
                }
            return;
        }
        if (maxl < 0 ? gv.n_tasks == 0 : m.n_tiles == 0)
            return;
        // windows are bulk-copied from the gathered vectors: they need 16-byte alignment
        bool aligned = true;
        for (int g = 0; g < Op::NG; ++g)
            aligned = aligned && (((uintptr_t)op.gvec(g) & 15) == 0);
        const WinDesc *w = aligned ? win : nullptr;
        switch (maxl) {
        case 4: k_rows_tma<K, VM, 4, Op><<<grid, RTHREADS, RSMEM, s>>>(m, w, op, part, st, err); break;
        case 6: k_rows_tma<K, VM, 6, Op><<<grid, RTHREADS, RSMEM, s>>>(m, w, op, part, st, err); break;
        case 8: k_rows_tma<K, VM, 8, Op><<<grid, RTHREADS, RSMEM, s>>>(m, w, op, part, st, err); break;
        case 16: k_rows_tma<K, VM, 16, Op><<<grid, RTHREADS, RSMEM, s>>>(m, w, op, part, st, err); break;
        case -1:
            if constexpr (LANE_GROUPS)
                k_rowgroup<K, VM, Op><<<grid, GroupCfg<K, Op>::T, 0, s>>>(m, gv, op, part, st);
            break;
        case -2:
            if constexpr (LANE_GROUPS) {
                if (bdim == 2)
                    k_bsr_group<K, VM, 2, Op><<<grid, BsrCfg<K, 2, VM, Op>::T, 0, s>>>(m, gv, op, part, st);
                else if (bdim == 3)
                    k_bsr_group<K, VM, 3, Op><<<grid, BsrCfg<K, 3, VM, Op>::T, 0, s>>>(m, gv, op, part, st);
                else if (bdim == 4)
                    k_bsr_group<K, VM, 4, Op><<<grid, BsrCfg<K, 4, VM, Op>::T, 0, s>>>(m, gv, op, part, st);
            }
            break;
        default:
            if constexpr (!LANE_GROUPS)
                k_tile2<K, VM, Op><<<grid, Tile2Cfg<K>::T, 0, s>>>(m, op, part, st);
            break;
        }
    }
};

template <typename V, int K, int MAXL>
static sla_status spmv_slices_k(const sla_csr *A, int nc, const void *x, void *y, cudaStream_t s)
{
    const SellPart *sp;
    SLA_TRY(ensure_sell(const_cast<sla_csr *>(A), s, &sp));
    auto kern = k_spmv_slices<V, K, MAXL>;
    int per_sm = 0;
    SLA_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, SPS_T, 0));
    const int64_t want = (sp->n_slices + 2 * (SPS_T / 32) - 1) / (2 * (SPS_T / 32));
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)std::max(per_sm, 1) * A->num_sms));
    kern<<<grid, SPS_T, 0, s>>>(A->n, sp->n_slices, sp->d_desc, sp->d_offs, A->rp, A->ci, (const V *)A->val,
                                (const V *)x, (V *)y, nc, nc);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

// Short rows, values declared static: the product over the sliced copy (values refreshed
// when stale), whole-row operand accesses where the layout and alignment allow them.
template <typename V, int K, int MAXL>
static sla_status spmv_sell_k(const sla_csr *A, int nc, const void *x, void *y, cudaStream_t s)
{
    const SellPart *sp;
    SLA_TRY(ensure_sell(const_cast<sla_csr *>(A), s, &sp));
    if (!A->sell_vals_current)
        SLA_TRY(launch_sell_values(A, sp, s));
    SellView<V> v;
    v.desc = sp->d_desc;
    v.offs = sp->d_offs;
    v.lens = sp->d_lens;
    v.idx16 = sp->rel16 ? (const int16_t *)sp->d_idx : nullptr;
    v.idx32 = sp->rel16 ? nullptr : (const int32_t *)sp->d_idx;
    v.val = (const V *)sp->d_val;
    v.n = A->n;
    v.n_slices = sp->n_slices;
    OpSpmv<V, K> op{(const V *)x, (V *)y, nc, nc};
    const uintptr_t wbytes = (uintptr_t)RowIO<V, K>::W;
    op.rows = nc == K && ((uintptr_t)x % wbytes) == 0 && ((uintptr_t)y % wbytes) == 0;
    auto kern = k_spmv_sell<V, K, MAXL>;
    int per_sm = 0;
    SLA_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, SPS_T, 0));
    const int64_t want = (sp->n_slices + 2 * (SPS_T / 32) - 1) / (2 * (SPS_T / 32));
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)std::max(per_sm, 1) * A->num_sms));
    kern<<<grid, SPS_T, 0, s>>>(v, op);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

template <typename V, int K>
static sla_status spmv_k(const sla_csr *A, int nc, const void *x, void *y, cudaStream_t s)
{
    // short rows: the sliced copy when the values are static, else the CSR-direct product
    // over the slice descriptors
    if (A->n > 0 && A->batch == 1 && A->bdim == 1 && A->max_row_len <= 16 && K <= 8) {
        if (A->flags & SLA_STATIC_VALUES) {
            if (A->max_row_len <= 8)
                return spmv_sell_k<V, K, 8>(A, nc, x, y, s);
            return spmv_sell_k<V, K, 16>(A, nc, x, y, s);
        }
        if (A->max_row_len <= 8)
            return spmv_slices_k<V, K, 8>(A, nc, x, y, s);
        return spmv_slices_k<V, K, 16>(A, nc, x, y, s);
    }
    using Op = OpSpmv<V, K>;
    Op op{(const V *)x, (V *)y, nc, nc};
    TileLaunch<K, V, Op> L;
    SLA_TRY(L.setup(A, s));
    if (L.maxl == -3 && !A->csb_vals_current)     // static values: the copy, refreshed on demand
        SLA_TRY(launch_csb_values(A, s));
    L.launch(s, op, nullptr, nullptr, A->d_err);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

template <typename VM, typename VV>
static sla_status grad_v(const sla_csr *A, int nrhs, const void *lam, const void *x, void *g,
                         double scale, cudaStream_t s)
{
    if (A->bdim > 1) {
        const int64_t nbr = pattern_rows(A);
        if (nbr == 0 || A->nnz == 0)
            return SLA_SUCCESS;
        const int grid = A->num_sms * 8;
        if (A->bdim == 2)
            k_bsr_grad<VM, VV, 2><<<grid, 256, 0, s>>>(nbr, A->rp, A->ci, nrhs, (const VV *)lam, (const VV *)x, (VM *)g, scale);
        else if (A->bdim == 3)
            k_bsr_grad<VM, VV, 3><<<grid, 256, 0, s>>>(nbr, A->rp, A->ci, nrhs, (const VV *)lam, (const VV *)x, (VM *)g, scale);
        else
            k_bsr_grad<VM, VV, 4><<<grid, 256, 0, s>>>(nbr, A->rp, A->ci, nrhs, (const VV *)lam, (const VV *)x, (VM *)g, scale);
        SLA_CUDA_TRY(cudaGetLastError());
        return SLA_SUCCESS;
    }
    const TilePart *tp;
    SLA_TRY(ensure_tiles(const_cast<sla_csr *>(A), GRAD_D, GRAD_D, s, &tp));
    if (tp->n_tiles == 0)
        return SLA_SUCCESS;
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_pattern_grad<VM, VV>, GRAD_T, 0);
    const int grid = std::max(1, std::min(tp->n_tiles, std::max(per_sm, 1) * A->num_sms));
    k_pattern_grad<VM, VV><<<grid, GRAD_T, 0, s>>>(view<VM>(A, tp), nrhs, (const VV *)lam,
                                                   (const VV *)x, (VM *)g, scale);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}


// ------------------------------------------------------------------ solve plans
// The kernels of one PCG iteration for a plan, with their grids and operands bound.
template <typename VM, typename VV, int K>
struct PlanKernels {
    TileLaunch<K, VM, OpQ<VV, K>> LQ;
    TileLaunch<K, VM, OpUS<VV, K>> LUS;
    TileLaunch<K, VM, OpZ<VV, K>> LZ;
    // matrices with long rows: operand vectors formed first (k_ep / k_er), one gather per entry
    TileLaunch<K, VM, OpQm<VV, K>> LQm;
    TileLaunch<K, VM, OpUSm<VV, K>> LUSm;
    bool formA = false, formGT = false;
    int64_t n = 0;
    VV *x, *ra, *rb, *pa, *pb, *q, *z, *y;
    const VV *dinv = nullptr;
    PcgState *st;
    double *part;
    int *err;
    int gv = 0;

    sla_status bind(sla_csr *A, Plan *p, cudaStream_t s)
    {
        const sla_precond *M = p->M;
        n = A->n;
        x = (VV *)p->x; ra = (VV *)p->ra; rb = (VV *)p->rb; pa = (VV *)p->pa; pb = (VV *)p->pb;
        q = (VV *)p->q; z = (VV *)p->z; y = (VV *)p->y;
        st = p->st;
        part = p->partials;
        err = &p->st->error;
        SLA_TRY(LQ.setup(A, s));
        formA = LQ.maxl <= 0;
        if (formA)
            SLA_TRY(LQm.setup(A, s));
        gv = vec_grid(A);
        if (p->kind == 1)
            dinv = (const VV *)(sizeof(VV) == 8 ? M->d_dinv64 : M->d_dinv);
        else if (p->kind == 0)
            dinv = (const VV *)p->y;  // ones (y is unused without SPAI)
        if (p->kind == 2) {
            SLA_TRY(LZ.setup(M->G, s));
            SLA_TRY(LUS.setup(M->GT, s));
            formGT = LUS.maxl <= 0;
            if (formGT)
                SLA_TRY(LUSm.setup(M->GT, s));
        }
        p->grid_tiles_A = LQ.grid;
        p->grid_tiles_G = LZ.grid;
        p->grid_tiles_GT = LUS.grid;
        p->grid_vec = gv;
        return SLA_SUCCESS;
    }
    void Q(cudaStream_t s, const VV *pold, VV *pnew) const
    {
        if (formA) {
            k_ep<VV, K><<<gv, VEC_T, 0, s>>>(n, z, pold, pnew, st);
            LQm.launch(s, OpQm<VV, K>{pnew, q, st}, part, st, err);
        } else {
            LQ.launch(s, OpQ<VV, K>{z, pold, pnew, q, st}, part, st, err);
        }
    }
    void UJ(cudaStream_t s, const VV *pcur) const
    {
        k_update_jacobi<VV, K><<<gv, VEC_T, 0, s>>>(n, x, ra, pcur, q, z, dinv, part, st);
    }
    void US(cudaStream_t s, const VV *rold, VV *rnew, const VV *pcur) const
    {
        if (formGT) {
            k_er<VV, K><<<gv, VEC_T, 0, s>>>(n, rold, q, pcur, x, rnew, part, st);
            LUSm.launch(s, OpUSm<VV, K>{rnew, y, st}, part, st, err);
        } else {
            LUS.launch(s, OpUS<VV, K>{rold, q, pcur, x, rnew, x, y, st}, part, st, err);
        }
    }
    void Z(cudaStream_t s, const VV *rcur) const
    {
        LZ.launch(s, OpZ<VV, K>{y, rcur, z, st}, part, st, err);
    }
};

template <typename VM, typename VV, int K>
static sla_status capture_k(sla_csr *A, Plan *p)
{
    PlanKernels<VM, VV, K> kr;
    SLA_TRY(kr.bind(A, p, p->cs));
    SLA_CUDA_TRY(cudaStreamSynchronize(p->cs));
    VV *ra = kr.ra, *rb = kr.rb, *pa = kr.pa, *pb = kr.pb;

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
template <typename VM, typename VV, int K>
static sla_status times_k(sla_csr *A, Plan *p, int nrhs, int reps, double *h_ms, cudaStream_t s)
{
    PlanKernels<VM, VV, K> kr;
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

// ------------------------------------------------------------------ persistent engine
// Row-length bound (the kernel's MAXL) the persistent engine uses for this plan, 0 when it
// does not apply: single systems whose matrices (A; with SPAI also G and G^T) have rows of
// at most 8 entries (16 with K <= 2), K <= 8, cooperative launch available.
// Instantiated combinations: those whose consumer code fits the register budget (fp64
// vectors: K <= 4 and rows of at most 8 entries).
template <typename VV, int K, int MAXL>
constexpr bool persist_compiled()
{
    return K <= 8 && (MAXL == 8 || K <= 2) && (sizeof(VV) == 4 || (K <= 4 && MAXL == 8));
}

template <typename VV, int K>
static int persist_maxl(const sla_csr *A, const Plan *p)
{
    if (K > 8 || A->batch > 1 || A->n == 0 || A->nnz == 0 || A->bdim > 1)
        return 0;
    int64_t L = A->max_row_len;
    if (p->kind == 2) {
        if (p->M->G->nnz == 0)
            return 0;
        L = std::max(L, std::max(p->M->G->max_row_len, p->M->GT->max_row_len));
    }
    int coop = 0;
    if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, A->device) != cudaSuccess || !coop)
        return 0;
    if (L <= 8)
        return persist_compiled<VV, K, 8>() ? 8 : 0;
    if (L <= 16)
        return persist_compiled<VV, K, 16>() ? 16 : 0;
    return 0;
}

template <typename VM, typename VV, int K, int MAXL>
static sla_status persist_launch(sla_csr *A, Plan *p, cudaStream_t s)
{
    using Pk = Persist<VM, VV, K, MAXL>;
    auto kern = k_pcg_persistent<VM, VV, K, MAXL>;
    PersistArgs<VM, VV> a{};
    // sliced ELL copies: built once per matrix; values gathered from the CSR arrays on every
    // solve, so values changed in place since the last solve are used
    auto sell = [&](const sla_csr *M_, SellView<VM> &v) -> sla_status {
        const SellPart *sp;
        SLA_TRY(ensure_sell(const_cast<sla_csr *>(M_), s, &sp));
        SLA_TRY(launch_sell_values(M_, sp, s));
        v.desc = sp->d_desc;
        v.offs = sp->d_offs;
        v.lens = sp->d_lens;
        v.idx16 = sp->rel16 ? (const int16_t *)sp->d_idx : nullptr;
        v.idx32 = sp->rel16 ? nullptr : (const int32_t *)sp->d_idx;
        v.val = (const VM *)sp->d_val;
        v.n = M_->n;
        v.n_slices = sp->n_slices;
        return SLA_SUCCESS;
    };
    a.spai = p->kind == 2 ? 1 : 0;
    SLA_TRY(sell(A, a.A));
    if (a.spai) {
        SLA_TRY(sell(p->M->G, a.G));
        SLA_TRY(sell(p->M->GT, a.GT));
    }
    a.x = (VV *)p->x; a.ra = (VV *)p->ra; a.rb = (VV *)p->rb; a.pa = (VV *)p->pa; a.pb = (VV *)p->pb;
    a.q = (VV *)p->q; a.z = (VV *)p->z; a.y = (VV *)p->y;
    if (p->kind == 1)
        a.dinv = (const VV *)(sizeof(VV) == 8 ? p->M->d_dinv64 : p->M->d_dinv);
    else if (p->kind == 0)
        a.dinv = (const VV *)p->y;   // ones (y is unused without SPAI)
    a.st = p->st;
    a.partials = p->partials;
    a.err = &p->st->error;
    if (p->persist_grid == 0) {
        int per_sm = 0;
        SLA_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Pk::TB, 0));
        if (per_sm < 1)
            return fail(SLA_ERR_UNSUPPORTED, "persistent solver kernel does not fit on an SM");
        // every block must be resident at once (cooperative launch); the partials buffer
        // holds 4 slots of 2K doubles per block.  At least one slice per warp: every block
        // arrives at every grid barrier, so idle blocks only add to the barrier's cost.
        const int cap = (int)(((size_t)A->num_sms * 32 * 2 * KMAX) / (4 * 2 * K));
        int64_t slices = a.A.n_slices;
        if (a.spai)
            slices = std::max(slices, std::max(a.G.n_slices, a.GT.n_slices));
        const int64_t units = (slices + Pk::TB / 32 - 1) / (Pk::TB / 32);
        p->persist_grid = (int)std::max<int64_t>(1, std::min<int64_t>(units, std::min(per_sm * A->num_sms, cap)));
    }
    void *args[] = {(void *)&a};
    SLA_CUDA_TRY(cudaLaunchCooperativeKernel((const void *)kern, dim3(p->persist_grid), dim3(Pk::TB), args, 0, s));
    return SLA_SUCCESS;
}

template <typename VM, typename VV, int K>
static sla_status run_k(sla_csr *A, Plan *p, int nrhs, const void *B, void *X, double tol,
                        long long maxit, int engine, cudaStream_t s)
{
    const int maxl = engine == SLA_ENGINE_GRAPH ? 0 : persist_maxl<VV, K>(A, p);
    if (engine == SLA_ENGINE_PERSISTENT && maxl == 0)
        return fail(SLA_ERR_INVALID_ARG, "the persistent engine does not apply to this system");
    const int64_t n = A->n;
    const int gv = vec_grid(A);
    VV *y = (VV *)p->y;
    if (p->kind == 0) {
        // without a preconditioner the Jacobi kernel runs with D^-1 = 1 (held in y)
        k_fill<VV><<<gv, 256, 0, s>>>(n, y, (VV)1);
        y = nullptr;
    }
    k_init<VV, K><<<gv, 256, 0, s>>>(n, nrhs, (const VV *)B, (VV *)p->x, (VV *)p->ra, (VV *)p->pa,
                                     (VV *)p->q, (VV *)p->z, p->kind == 2 ? y : nullptr, p->st, tol,
                                     maxit, p->M ? p->M->eps : 0.0, p->cond, 1);
    SLA_CUDA_TRY(cudaGetLastError());
    if (maxl == 8) {
        if constexpr (persist_compiled<VV, K, 8>())
            SLA_TRY((persist_launch<VM, VV, K, 8>(A, p, s)));
    } else if (maxl == 16) {
        if constexpr (persist_compiled<VV, K, 16>())
            SLA_TRY((persist_launch<VM, VV, K, 16>(A, p, s)));
    } else {
        // column-sorted copies of long-row matrices: values gathered from the CSR arrays
        // before every solve (they may have changed since the last one)
        SLA_TRY(launch_csb_values(A, s));
        if (p->kind == 2) {
            SLA_TRY(launch_csb_values(p->M->G, s));
            SLA_TRY(launch_csb_values(p->M->GT, s));
        }
        SLA_CUDA_TRY(cudaGraphLaunch(p->exec, s));
    }
    k_copy_out<VV, K><<<gv, 256, 0, s>>>(n, nrhs, (const VV *)p->x, (VV *)X);
    SLA_CUDA_TRY(cudaGetLastError());
    return SLA_SUCCESS;
}

}  // namespace sla
