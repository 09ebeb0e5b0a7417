// Load-balanced CSR SpMV engine with fused row epilogues and fused dot products.
//
// Work unit: a "tile" = a run of whole rows holding at most D items (rows + stored
// entries), built once per matrix on the host; a row longer than that is a tile of its own
// and is reduced by the whole block.  Rows never straddle tiles, so every row is finished
// inside one block and its epilogue (vector updates, dot-product partials) runs there.
//
// Inside a tile:
//   1. stage the tile's row ends into shared memory and form every product
//      A_k * operand(col_k) in fp64 with coalesced loads of col/val (one (entry, rhs) pair
//      per thread step, so K right-hand sides read K contiguous operand values);
//   2. split the tile's items evenly over the threads along the merge path of (row ends,
//      entries) -- the merge-based SpMV decomposition -- and let each thread sum its run;
//   3. a row that spans several threads is finished by the thread holding its end, which
//      adds the partial sums the earlier threads left in shared memory, in a fixed order.
// Blocks are persistent (grid = resident blocks) and walk the tiles round-robin, so each
// block's dot-product partial is a fixed-order sum; the last block to finish reduces the
// per-block partials in block order and runs the operation's scalar finalisation.  The
// result is deterministic for a given device.
#pragma once

#include "sla_internal.cuh"

namespace sla {

template <int K>
struct TileCfg;
template <> struct TileCfg<1> { static constexpr int T = 256, D = 2048; };
template <> struct TileCfg<2> { static constexpr int T = 256, D = 1024; };
template <> struct TileCfg<4> { static constexpr int T = 256, D = 512; };
template <> struct TileCfg<8> { static constexpr int T = 128, D = 512; };
template <> struct TileCfg<16> { static constexpr int T = 64, D = 256; };

// Sum N values over the block.  On return thread i (< N) holds the total of value i in
// v[0]; the order of additions is fixed.
template <int T, int N>
__device__ __forceinline__ void block_sum(double (&v)[N], double *s_red)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int i = 0; i < N; ++i) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            v[i] += __shfl_down_sync(0xffffffffu, v[i], off);
    }
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < N; ++i)
            s_red[warp * N + i] = v[i];
    }
    __syncthreads();
    double t = 0.0;
    if (tid < N) {
#pragma unroll
        for (int w = 0; w < T / 32; ++w)
            t += s_red[w * N + tid];
    }
    __syncthreads();
    v[0] = t;
}

// Write this block's partials, and in the last block to finish, reduce all blocks'
// partials (block order) and call op.finalize(sums) on thread 0.
template <int T, int N, class Op>
__device__ __forceinline__ void grid_reduce_finalize(double (&part)[N], double *partials,
                                                     PcgState *st, const Op &op, double *s_red)
{
    __shared__ int s_last;
    __shared__ double s_sum[N];
    block_sum<T, N>(part, s_red);
    if (threadIdx.x < N)
        partials[(size_t)blockIdx.x * N + threadIdx.x] = part[0];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned int t = atomicAdd(&st->ticket, 1u);
        s_last = (t == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last)
        return;
    __threadfence();
    double v[N];
#pragma unroll
    for (int i = 0; i < N; ++i)
        v[i] = 0.0;
    for (int c = threadIdx.x; c < (int)gridDim.x; c += T) {
#pragma unroll
        for (int i = 0; i < N; ++i)
            v[i] += __ldcg(&partials[(size_t)c * N + i]);
    }
    block_sum<T, N>(v, s_red);
    if (threadIdx.x < N)
        s_sum[threadIdx.x] = v[0];
    __syncthreads();
    if (threadIdx.x == 0) {
        op.finalize(s_sum);
        st->ticket = 0u;
    }
}

// Op concept:
//   static constexpr int NP;                       dot products per rhs (0: none)
//   static constexpr int NS;                       scalars staged in shared memory
//   bool skip() const;                             whole kernel is a no-op (solve finished)
//   void stage(double *s) const;                   thread 0 fills s[0..NS)
//   double operand(int64_t j, int c, const double *s) const;
//   void emit(int64_t i, const double (&acc)[K], double (&part)[NP*K or 1], const double *s) const;
//   void finalize(const double *sums) const;       sums[p*K + c]
template <int K, typename V, class Op>
__global__ void __launch_bounds__(TileCfg<K>::T)
k_tile(const MatView<V> m, const Op op, double *partials, PcgState *st)
{
    constexpr int T = TileCfg<K>::T;
    constexpr int D = TileCfg<K>::D;
    constexpr int IPT = D / T;
    constexpr int NPK = Op::NP * K;
    constexpr int NR = NPK > K ? NPK : K;
    __shared__ int32_t s_rp[D];
    __shared__ double s_prod[D * K];
    __shared__ int32_t s_crow[T];
    __shared__ double s_cval[T * K];
    __shared__ double s_red[(T / 32) * NR];
    __shared__ double s_scal[Op::NS > 0 ? Op::NS : 1];

    if (op.skip())
        return;
    const int tid = threadIdx.x;
    if (tid == 0)
        op.stage(s_scal);
    __syncthreads();

    double part[NPK > 0 ? NPK : 1];
#pragma unroll
    for (int i = 0; i < (NPK > 0 ? NPK : 1); ++i)
        part[i] = 0.0;

    for (int t = blockIdx.x; t < m.n_tiles; t += gridDim.x) {
        const int r0 = m.tile_row[t];
        const int r1 = m.tile_row[t + 1];
        const int nr = r1 - r0;
        const int64_t k0 = m.rp[r0];
        const int nk = (int)(m.rp[r1] - k0);

        if (nr + nk > D) {
            // one long row: block-strided products, fixed-tree block sum
            double acc[K];
#pragma unroll
            for (int c = 0; c < K; ++c)
                acc[c] = 0.0;
            for (int e = tid; e < nk; e += T) {
                const int64_t j = m.ci[k0 + e];
                const double a = (double)m.val[k0 + e];
#pragma unroll
                for (int c = 0; c < K; ++c)
                    acc[c] = fma(a, op.operand(j, c, s_scal), acc[c]);
            }
#pragma unroll
            for (int c = 0; c < K; ++c) {
                double one[1] = {acc[c]};
                block_sum<T, 1>(one, s_red);
                if (tid == 0)
                    s_cval[c] = one[0];
            }
            __syncthreads();
            if (tid == 0) {
                double tot[K];
#pragma unroll
                for (int c = 0; c < K; ++c)
                    tot[c] = s_cval[c];
                op.emit(r0, tot, part, s_scal);
            }
            __syncthreads();
            continue;
        }

        for (int r = tid; r < nr; r += T)
            s_rp[r] = (int32_t)(m.rp[r0 + 1 + r] - k0);
        for (int f = tid; f < nk * K; f += T) {
            const int e = f / K;
            const int c = f - e * K;
            const int64_t j = m.ci[k0 + e];
            s_prod[f] = (double)m.val[k0 + e] * op.operand(j, c, s_scal);
        }
        __syncthreads();

        const int items = nr + nk;
        const int d0 = min(tid * IPT, items);
        const int d1 = min(d0 + IPT, items);
        // merge-path split: largest x (rows finished) with row_end[x-1] <= d0 - x
        int lo = max(0, d0 - nk), hi = min(d0, nr);
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_rp[mid - 1] <= d0 - mid)
                lo = mid;
            else
                hi = mid - 1;
        }
        int r = lo, k = d0 - lo;
        double acc[K], facc[K];
#pragma unroll
        for (int c = 0; c < K; ++c) {
            acc[c] = 0.0;
            facc[c] = 0.0;
        }
        int frow = -1;
        for (int d = d0; d < d1; ++d) {
            if (k < s_rp[r]) {
#pragma unroll
                for (int c = 0; c < K; ++c)
                    acc[c] += s_prod[k * K + c];
                ++k;
            } else {
                if (frow < 0) {
                    frow = r;
#pragma unroll
                    for (int c = 0; c < K; ++c)
                        facc[c] = acc[c];
                } else {
                    op.emit(r0 + r, acc, part, s_scal);
                }
#pragma unroll
                for (int c = 0; c < K; ++c)
                    acc[c] = 0.0;
                ++r;
            }
        }
        s_crow[tid] = (r < nr) ? r : -1;
#pragma unroll
        for (int c = 0; c < K; ++c)
            s_cval[tid * K + c] = acc[c];
        __syncthreads();
        if (frow >= 0) {
            for (int u = tid - 1; u >= 0 && s_crow[u] == frow; --u) {
#pragma unroll
                for (int c = 0; c < K; ++c)
                    facc[c] += s_cval[u * K + c];
            }
            op.emit(r0 + frow, facc, part, s_scal);
        }
        __syncthreads();
    }

    if constexpr (NPK > 0)
        grid_reduce_finalize<T, NPK>(part, partials, st, op, s_red);
}

}  // namespace sla
