// Short-row CSR SpMV engine: one thread per row, for matrices whose rows hold at most
// MAXL stored entries (stencils and their triangular factors).
//
// A thread loads its row's column indices and values with predicated, fully unrolled loads
// (all in flight at once), gathers the operand values, accumulates (fp32 when values and
// vectors are fp32 -- at most MAXL terms per row -- fp64 otherwise) and runs the
// same fused row epilogue as the tile engine, reading its own-row vector values straight
// from global memory (consecutive threads own consecutive rows, so those loads and the
// epilogue's stores are coalesced).  There is no shared-memory staging and no barrier in
// the row loop, which keeps the instruction count per stored entry small; rows are
// assigned grid-stride, so the dot-product partials are fixed-order sums and the result
// is deterministic for a given device.
#pragma once

#include <type_traits>

#include "tile_engine.cuh"

namespace sla {

constexpr int ROW_T = 256;

// Own-row vector values read from global memory (same interface as RowVecs).
template <typename VV, int K, int NV>
struct GlobalRowVecs {
    const VV *base[NV > 0 ? NV : 1];
    __device__ __forceinline__ VV get(int v, int64_t i, int c) const { return base[v][i * K + c]; }
};

template <int K, typename VM, int MAXL, class Op>
__global__ void __launch_bounds__(ROW_T)
k_rows(const MatView<VM> m, const Op op, double *partials, PcgState *st)
{
    using VV = typename Op::VV;
    // row sums in fp32 when matrix and vectors are fp32 (at most MAXL terms), fp64 otherwise
    using Acc = typename std::conditional<sizeof(VM) == 4 && sizeof(VV) == 4, float, double>::type;
    constexpr int NV = Op::NV;
    constexpr int NPK = Op::NP * K;
    constexpr int NR = NPK > 0 ? NPK : 1;
    __shared__ double s_scal[Op::NS > 0 ? Op::NS : 1];
    __shared__ double s_red[(ROW_T / 32) * NR];
    __shared__ double s_sum[NR];
    __shared__ int s_flag;

    if (op.skip())
        return;
    const int tid = threadIdx.x;
    if (tid == 0)
        op.stage(s_scal);
    __syncthreads();
    GlobalRowVecs<VV, K, NV> rv;
#pragma unroll
    for (int v = 0; v < NV; ++v)
        rv.base[v] = op.row_vec(v);

    double part[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i)
        part[i] = 0.0;
    const int64_t stride = (int64_t)gridDim.x * ROW_T;
    for (int64_t i = (int64_t)blockIdx.x * ROW_T + tid; i < m.n; i += stride) {
        const int k0 = m.rp[i];
        const int len = m.rp[i + 1] - k0;
        int cj[MAXL];
        VM av[MAXL];
#pragma unroll
        for (int u = 0; u < MAXL; ++u) {
            cj[u] = u < len ? __ldg(&m.ci[k0 + u]) : 0;
            av[u] = u < len ? __ldg(&m.val[k0 + u]) : (VM)0;
        }
        VV ov[MAXL][K];
#pragma unroll
        for (int u = 0; u < MAXL; ++u) {
#pragma unroll
            for (int c = 0; c < K; ++c)
                ov[u][c] = u < len ? op.operand(cj[u], c, s_scal) : (VV)0;
        }
        double acc[K];
#pragma unroll
        for (int c = 0; c < K; ++c) {
            Acc a = (Acc)0;
#pragma unroll
            for (int u = 0; u < MAXL; ++u)
                a = fma((Acc)av[u], (Acc)ov[u][c], a);
            acc[c] = (double)a;
        }
        op.emit(i, acc, part, s_scal, rv);
    }

    if constexpr (NPK > 0) {
        auto sync = [] { __syncthreads(); };
        grid_reduce_finalize<ROW_T, NPK>(part, partials, st, op, s_red, &s_flag, s_sum, tid, sync);
    }
}

}  // namespace sla
