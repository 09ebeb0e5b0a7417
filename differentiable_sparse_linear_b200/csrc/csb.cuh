// Column-sorted row segments: the SpMV engine for matrices whose rows gather their operands
// from scattered columns (a random graph's neighbours, the power-law system).
//
// In CSR order every stored entry gathers one operand from a random column, so each entry
// costs its own L2 request; measured on B200, a random 4-byte gather stream tops out near
// 270 G gathers/s, a third of what the matrix stream alone would allow.  Here the rows are
// cut into segments of at most CSB_RMAX consecutive rows, and each segment's entries are
// stored in COLUMN order: the 32 lanes of a warp then gather from a few hundred neighbouring
// columns instead of 32 random ones, so one L2 request serves several entries.  The row sums
// are accumulated in shared memory (one slot per row of the segment, fp64, atomic adds), and
// the fused row epilogue of the operation runs once the segment's entries are done.
//
// Storage (CsbPart): per segment its first row and first chunk; entries in chunks of 32
// (one warp load), per chunk the smallest column `base`, per entry a 32-bit word
// (column - base) << 16 | local row, padding marked by local row 0xFFFF, and the entry's
// value, gathered from the caller's CSR values by `perm` at the start of every solve (the
// values may change between solves; the pattern may not).  8 bytes per entry plus 4 per 32
// entries, as CSR's value + column index.
//
// The sums are fp64 in any order (the atomic adds' order varies from launch to launch), so
// a row sum may differ from one launch to the next by the last bits of an fp64 value, which
// the rounding to fp32 vectors almost always absorbs.
#pragma once

#include <cuda_runtime.h>

#include "sla_internal.cuh"
#include "pcg_ops.cuh"
#include "tile_engine.cuh"

namespace sla {

constexpr int CSB_RMAX = 16384;                // rows per segment (fp64 sums in shared memory)
constexpr uint32_t CSB_PAD = 0xFFFFu;

template <typename VM>
struct CsbView {
    const int32_t *seg_row0;                   // n_seg + 1
    const int32_t *seg_ch0;                    // n_seg + 1
    const int32_t *cbase;                      // per chunk
    const uint32_t *pk;                        // per entry slot
    const VM *val;                             // per entry slot
    int n_seg;
    int rmax;                                  // rows of the largest segment
};

// 4 chunks per warp per round with the next round prefetched measured the same as 2, 6, or
// 8 without the prefetch (q = A p on the 4M system: 0.773 / 0.773 / 0.786 / 0.783 ms).
struct CsbCfg {
    static constexpr int T = 1024;             // threads per block (one block per SM)
    static constexpr int U = 4;                // chunks per warp per round
};

// One round's matrix data of a warp: U chunks (or padding past the segment's end).
template <typename VM, int U>
struct CsbRound {
    int base[U];
    uint32_t w[U];
    VM a[U];
    __device__ __forceinline__ void load(const CsbView<VM> &c, int ch, int ch1, int lane)
    {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int cc = ch + u * (CsbCfg::T / 32);
            if (cc < ch1) {
                base[u] = __ldg(&c.cbase[cc]);
                w[u] = __ldg(&c.pk[(int64_t)cc * 32 + lane]);
                a[u] = __ldg(&c.val[(int64_t)cc * 32 + lane]);
            } else {
                base[u] = 0;
                w[u] = CSB_PAD;
                a[u] = (VM)0;
            }
        }
    }
};

// y rows of one segment summed in shared memory, then the operation's row epilogue.
// Single right-hand side; operations that gather one vector (NG == 1).  Each warp walks
// the segment's chunks U at a time and loads the next round's matrix data while the
// current round's gathers and sums are in flight.
template <typename VM, class Op>
__global__ void __launch_bounds__(CsbCfg::T, 1)
k_csb(const CsbView<VM> c, const Op op, double *partials, PcgState *st)
{
    constexpr int T = CsbCfg::T;
    constexpr int U = CsbCfg::U;
    constexpr int NW = T / 32;
    constexpr int NPK = Op::NP;
    constexpr int NR = NPK > 1 ? NPK : 1;
    using VV = typename Op::VV;
    static_assert(Op::NG == 1, "the column-sorted engine gathers one vector");

    extern __shared__ __align__(16) double s_y[];
    __shared__ double s_red[NW * NR];
    __shared__ double s_scal[Op::NS > 0 ? Op::NS : 1];
    __shared__ double s_sum[NR];
    __shared__ int s_flag;

    if (op.skip())
        return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0)
        op.stage(s_scal);
    __syncthreads();
    GlobalRows<Op, 1> rv{op};
    double part[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i)
        part[i] = 0.0;

    for (int s = blockIdx.x; s < c.n_seg; s += gridDim.x) {
        const int r0 = c.seg_row0[s];
        const int R = c.seg_row0[s + 1] - r0;
        const int ch1 = c.seg_ch0[s + 1];
        int ch = c.seg_ch0[s] + warp;
        CsbRound<VM, U> cur;
        cur.load(c, ch, ch1, lane);
        for (int i = tid; i < R; i += T)
            s_y[i] = 0.0;
        __syncthreads();
        for (; ch < ch1; ch += U * NW) {
            CsbRound<VM, U> nxt;
            nxt.load(c, ch + U * NW, ch1, lane);
            VV g[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                g[u] = (cur.w[u] & 0xFFFFu) != CSB_PAD
                           ? op.operand((int64_t)cur.base[u] + (cur.w[u] >> 16), 0, s_scal) : (VV)0;
#pragma unroll
            for (int u = 0; u < U; ++u)
                if ((cur.w[u] & 0xFFFFu) != CSB_PAD)
                    atomicAdd(&s_y[cur.w[u] & 0xFFFFu], (double)cur.a[u] * (double)g[u]);
            cur = nxt;
        }
        __syncthreads();
        for (int i = tid; i < R; i += T) {
            const double acc[1] = {s_y[i]};
            op.emit((int64_t)(r0 + i), acc, part, s_scal, rv);
        }
        __syncthreads();
    }

    if constexpr (NPK > 0) {
        auto sync = [] { __syncthreads(); };
        grid_reduce_finalize<T, NPK>(part, partials, st, op, s_red, &s_flag, s_sum, tid, sync);
    }
}

// Values of the sorted copy from the caller's CSR values (0 in the padding).
template <typename VM>
__global__ void k_csb_values(int64_t slots, const int32_t *perm, const VM *src, VM *dst)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < slots; e += stride) {
        const int32_t k = perm[e];
        dst[e] = k >= 0 ? src[k] : (VM)0;
    }
}

}  // namespace sla
