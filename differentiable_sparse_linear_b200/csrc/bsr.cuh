// Block sparse row (BSR) kernels: the fused lane-group SpMV and the pattern gradient for
// matrices stored as b x b dense blocks (b = 2, 3, 4).
//
// Storage ("Efficient Sparse Matrix Algebra in Python for Mathematics", Key sparse formats
// and memory tradeoffs; Block sparse patterns and sharding strategies): block row I holds
// blocks k = row_ptr[I] .. row_ptr[I+1]-1 in block columns col[k]; block k keeps its b*b
// values row-major at val[k*b*b].  One column index serves b*b values, so the matrix
// stream is b*b*s_v + 4 bytes per block instead of b*b*(s_v + 4) in scalar CSR.
#pragma once

#include "tile_engine.cuh"

namespace sla {

// ------------------------------------------------------------------ lane-group BSR SpMV
// Block rows grouped by their number of blocks (GroupPart, two blocks per lane and pass):
// a group of G lanes owns a block row, each lane takes its blocks G apart (UB per pass,
// every value, column and operand load of a pass in flight), multiplies the b x b block
// into its b partial row sums, and the group sums its lanes with a fixed xor-shuffle
// tree; lane 0 of the group runs the row epilogue for the block row's b scalar rows.
template <int K, int B, typename VM, class Op>
struct BsrCfg {
    static constexpr int T = 256;
    static constexpr int UB = B * B * K <= 18 ? 2 : 1;      // blocks per lane per pass
    // fp64 values and runtime-strided operands (the standalone SpMV) need more registers
    static constexpr bool HEAVY = any_ld<Op>::value || sizeof(VM) == 8;
    static constexpr int MINB = (K == 1 && B <= 3) ? (HEAVY ? 4 : 6) : (B * B * K <= 8 && !HEAVY ? 4 : 2);
};

template <int K, typename VM, int B, class Op>
__global__ void __launch_bounds__(BsrCfg<K, B, VM, Op>::T, BsrCfg<K, B, VM, Op>::MINB)
k_bsr_group(const MatView<VM> m, const GroupView g, const Op op, double *partials, PcgState *st)
{
    constexpr int T = BsrCfg<K, B, VM, Op>::T;
    constexpr int NW = T / 32;
    constexpr int UB = BsrCfg<K, B, VM, Op>::UB;
    constexpr int BB = B * B;
    constexpr int NPK = Op::NP * K;
    constexpr int NR = NPK > K ? NPK : K;
    using VV = typename Op::VV;

    __shared__ double s_red[NW * NR];
    __shared__ double s_scal[Op::NS > 0 ? Op::NS : 1];
    __shared__ double s_sum[NR];
    __shared__ int s_flag;

    if (op.skip())
        return;
    const int tid = threadIdx.x, lane = tid & 31;
    if (tid == 0)
        op.stage(s_scal);
    __syncthreads();
    GlobalRows<Op, K> rv{op};
    double part[NPK > 0 ? NPK : 1];
#pragma unroll
    for (int i = 0; i < (NPK > 0 ? NPK : 1); ++i)
        part[i] = 0.0;

    const int nw = gridDim.x * NW;
    int t = blockIdx.x * NW + (tid >> 5);
    int bin = 0, pos = t < g.n_tasks ? group_locate(g, t, lane, bin) : -1;
    int4 cur = pos >= 0 ? __ldg(&g.rows[pos]) : make_int4(0, 0, 0, 0);
    for (; t < g.n_tasks; t += nw) {
        const int G = 32 >> bin;
        const bool live = pos >= 0;
        const int4 row = cur;                       // {block row, first block, end block}
        const int tn = t + nw;
        int bin_n = 0, pos_n = tn < g.n_tasks ? group_locate(g, tn, lane, bin_n) : -1;
        cur = pos_n >= 0 ? __ldg(&g.rows[pos_n]) : make_int4(0, 0, 0, 0);

        double acc[B][K];
#pragma unroll
        for (int r = 0; r < B; ++r)
#pragma unroll
            for (int c = 0; c < K; ++c)
                acc[r][c] = 0.0;
        const int gl = lane & (G - 1);
        if (live) {
            for (int k = row.y + gl; k < row.z; k += UB * G) {
                VM a[UB][BB];
                int32_t J[UB];
#pragma unroll
                for (int u = 0; u < UB; ++u) {
                    const int e = k + u * G;
                    J[u] = e < row.z ? m.ci[e] : -1;
#pragma unroll
                    for (int q = 0; q < BB; ++q)
                        a[u][q] = e < row.z ? m.val[(int64_t)e * BB + q] : (VM)0;
                }
#pragma unroll
                for (int u = 0; u < UB; ++u) {
                    if (J[u] >= 0) {
#pragma unroll
                        for (int cb = 0; cb < B; ++cb) {
                            VV o[K];
                            op.operand_row((int64_t)J[u] * B + cb, o, s_scal);
#pragma unroll
                            for (int r = 0; r < B; ++r)
#pragma unroll
                                for (int c = 0; c < K; ++c)
                                    acc[r][c] = fma((double)a[u][r * B + cb], (double)o[c], acc[r][c]);
                        }
                    }
                }
            }
        }
        for (int off = G >> 1; off > 0; off >>= 1)
#pragma unroll
            for (int r = 0; r < B; ++r)
#pragma unroll
                for (int c = 0; c < K; ++c)
                    acc[r][c] += __shfl_xor_sync(0xffffffffu, acc[r][c], off);
        if (live && gl == 0)
#pragma unroll
            for (int r = 0; r < B; ++r)
                op.emit((int64_t)row.x * B + r, acc[r], part, s_scal, rv);
        bin = bin_n;
        pos = pos_n;
    }

    if constexpr (NPK > 0) {
        auto sync = [] { __syncthreads(); };
        grid_reduce_finalize<T, NPK>(part, partials, st, op, s_red, &s_flag, s_sum, tid, sync);
    }
}

// ------------------------------------------------------------------ BSR pattern gradient
// g[k*b*b + r*b + c] = -sum_q lam[(I*b + r)*nrhs + q] * x[(col[k]*b + c)*nrhs + q] for
// block k of block row I: a warp per block row, its lanes over the row's b*b*blocks values
// in storage order (coalesced writes of g).
template <typename VM, typename VV, int B>
__global__ void __launch_bounds__(256)
k_bsr_grad(int64_t nbr, const int32_t *rp, const int32_t *ci, int nrhs, const VV *lam, const VV *x, VM *g,
           double scale)
{
    constexpr int BB = B * B;
    const int lane = threadIdx.x & 31;
    const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t I = w0; I < nbr; I += nw) {
        const int64_t k0 = rp[I], items = ((int64_t)rp[I + 1] - k0) * BB;
        for (int64_t t = lane; t < items; t += 32) {
            const int64_t k = k0 + t / BB;
            const int rc = (int)(t % BB), r = rc / B, c = rc % B;
            const int64_t i = I * B + r, j = (int64_t)ci[k] * B + c;
            double s = 0.0;
            for (int q = 0; q < nrhs; ++q)
                s = __fma_rn((double)lam[i * nrhs + q], (double)x[j * nrhs + q], s);
            g[k0 * BB + t] = (VM)(scale * s);
        }
    }
}

}  // namespace sla
