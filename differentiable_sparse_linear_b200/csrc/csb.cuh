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
#include "row_engine.cuh"

namespace sla {

constexpr int CSB_RMAX = 16384;                // rows per segment (fp64 sums in shared memory)
#ifndef SLA_CSB_TMA
#define SLA_CSB_TMA 0
#endif
#ifndef SLA_CSB_PAIR
#define SLA_CSB_PAIR 0
#endif
constexpr bool CSB_TMA = SLA_CSB_TMA != 0;     // matrix stream by bulk copies (k_csb_tma)
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

// A segment's row sums in shared memory (8 bytes per row).  fp32 values with fp32 vectors:
// a pair of fp32 sums per row -- hi takes each product rounded to fp32 with an atomic add
// that returns the old value, and lo takes that addition's exact rounding error (recovered
// from the old value and the addend by the two-sum identity) plus the product's own fp32
// rounding error -- so the row sum hi + lo carries about 48 bits, where a plain fp32 sum in
// arbitrary order would move the solver's iteration counts.  Otherwise fp64 atomic adds.
constexpr bool CSB_PAIR = SLA_CSB_PAIR != 0;
template <typename VM, typename VV>
struct CsbSums {
    static constexpr bool PAIR = CSB_PAIR && sizeof(VM) == 4 && sizeof(VV) == 4;
    double *d;
    float *hi, *lo;
    __device__ __forceinline__ CsbSums(void *base, int rmax)
        : d((double *)base), hi((float *)base), lo((float *)base + rmax) {}
    __device__ __forceinline__ void zero(int i)
    {
        if constexpr (PAIR) {
            hi[i] = 0.f;
            lo[i] = 0.f;
        } else {
            d[i] = 0.0;
        }
    }
    __device__ __forceinline__ void add(int r, double p)
    {
        if constexpr (PAIR) {
            const float ph = __double2float_rn(p);
            const float pl = __double2float_rn(p - (double)ph);
            const float old = atomicAdd(&hi[r], ph);
            const float sm = __fadd_rn(old, ph);
            const float bb = __fsub_rn(sm, old);
            const float err = __fadd_rn(__fsub_rn(old, __fsub_rn(sm, bb)), __fsub_rn(ph, bb));
            atomicAdd(&lo[r], __fadd_rn(err, pl));
        } else {
            atomicAdd(&d[r], p);
        }
    }
    __device__ __forceinline__ double get(int i) const
    {
        if constexpr (PAIR)
            return (double)hi[i] + (double)lo[i];
        else
            return d[i];
    }
};

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
    CsbSums<VM, VV> sums(s_y, c.rmax);
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
            sums.zero(i);
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
                    sums.add((int)(cur.w[u] & 0xFFFFu), (double)cur.a[u] * (double)g[u]);
            cur = nxt;
        }
        __syncthreads();
        for (int i = tid; i < R; i += T) {
            const double acc[1] = {sums.get(i)};
            op.emit((int64_t)(r0 + i), acc, part, s_scal, rv);
        }
        __syncthreads();
    }

    if constexpr (NPK > 0) {
        auto sync = [] { __syncthreads(); };
        grid_reduce_finalize<T, NPK>(part, partials, st, op, s_red, &s_flag, s_sum, tid, sync);
    }
}

// The same product with the matrix stream fed by bulk copies: one producer warp copies each
// stage's chunks (their column words and values, SC chunks = one per consumer warp) into a
// shared-memory ring NST stages ahead; the consumer warps take their chunk of U stages at a
// time, release the stages as soon as the data is in registers, then gather and sum.  The
// stream's latency is then covered by the ring instead of by the warps' own loads.  Every
// wait is bounded in time (a wait that runs out sets *err and the abort flag; the kernel
// then runs to its end without further copies, its results flagged invalid by the host).
struct CsbTmaCfg {
    static constexpr int NCW = 31;             // consumer warps (+1 producer: 1024 threads)
    static constexpr int TC = NCW * 32;        // consumer threads
    static constexpr int T = TC + 32;          // + the producer warp
    static constexpr int SC = NCW;             // chunks per stage
    static constexpr int U = 4;                // stages per consumer round
};
template <typename VM>
struct CsbTmaLayout {
    static constexpr int NST = sizeof(VM) == 4 ? 8 : 6;
    static constexpr size_t PK = (size_t)CsbTmaCfg::SC * 32 * 4;
    static constexpr size_t VAL = (size_t)CsbTmaCfg::SC * 32 * sizeof(VM);
    static constexpr size_t STAGE = PK + VAL;
    static constexpr size_t RING = NST * STAGE;
};

template <typename VM, class Op>
__global__ void __launch_bounds__(CsbTmaCfg::T, 1)
k_csb_tma(const CsbView<VM> c, const Op op, double *partials, PcgState *st, int *err)
{
    using Cfg = CsbTmaCfg;
    using L = CsbTmaLayout<VM>;
    constexpr int NST = L::NST;
    constexpr int U = Cfg::U;
    constexpr int NPK = Op::NP;
    constexpr int NR = NPK > 1 ? NPK : 1;
    using VV = typename Op::VV;
    static_assert(Op::NG == 1, "the column-sorted engine gathers one vector");

    extern __shared__ __align__(128) unsigned char smem[];
    CsbSums<VM, VV> sums(smem + L::RING, c.rmax);
    __shared__ __align__(8) uint64_t full_bar[NST];
    __shared__ __align__(8) uint64_t empty_bar[NST];
    __shared__ int s_abort;
    __shared__ double s_red[Cfg::NCW * NR];
    __shared__ double s_scal[Op::NS > 0 ? Op::NS : 1];
    __shared__ double s_sum[NR];
    __shared__ int s_flag;

    if (op.skip())
        return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], Cfg::NCW);
        }
        fence_mbar_init();
        s_abort = 0;
        op.stage(s_scal);
    }
    __syncthreads();
    volatile int *abort = &s_abort;

    // ---------------------------------------------------------------- producer
    if (warp == Cfg::NCW) {
        if (lane != 0)
            return;
        RingPos rp;
        int issued[NST];
#pragma unroll
        for (int i = 0; i < NST; ++i)
            issued[i] = -1;
        for (int s = blockIdx.x; s < c.n_seg && !*abort; s += gridDim.x) {
            const int c1 = c.seg_ch0[s + 1];
            for (int g0 = c.seg_ch0[s]; g0 < c1 && !*abort; g0 += Cfg::SC) {
                const int nch = min(Cfg::SC, c1 - g0);
                mbar_wait_bounded(&empty_bar[rp.stage], rp.phase ^ 1u, err, abort);
                if (*abort)
                    break;
                unsigned char *sb = smem + (size_t)rp.stage * L::STAGE;
                const uint32_t pkb = (uint32_t)nch * 32u * 4u, vb = (uint32_t)nch * 32u * (uint32_t)sizeof(VM);
                mbar_arrive_expect_tx(&full_bar[rp.stage], pkb + vb);
                bulk_g2s(sb, c.pk + (int64_t)g0 * 32, pkb, &full_bar[rp.stage]);
                bulk_g2s(sb + L::PK, c.val + (int64_t)g0 * 32, vb, &full_bar[rp.stage]);
                issued[rp.stage] = (int)rp.phase;
                rp.next<NST>();
            }
        }
        // no copy may still be writing this block's shared memory when it exits
        for (int i = 0; i < NST; ++i)
            if (issued[i] >= 0)
                mbar_wait_bounded(&full_bar[i], (uint32_t)issued[i], err);
        return;
    }

    // ---------------------------------------------------------------- consumers
    auto csync = [] { consumer_sync(Cfg::TC); };
    GlobalRows<Op, 1> rv{op};
    double part[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i)
        part[i] = 0.0;
    RingPos rp;
    for (int s = blockIdx.x; s < c.n_seg; s += gridDim.x) {
        const int r0 = c.seg_row0[s];
        const int R = c.seg_row0[s + 1] - r0;
        const int c0 = c.seg_ch0[s], c1 = c.seg_ch0[s + 1];
        const int ngroups = (c1 - c0 + Cfg::SC - 1) / Cfg::SC;
        for (int i = tid; i < R; i += Cfg::TC)
            sums.zero(i);
        csync();
        for (int gb = 0; gb < ngroups; gb += U) {
            int base[U];
            uint32_t w[U];
            VM a[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {               // chunk bases first: independent of the ring
                const int cc = c0 + (gb + u) * Cfg::SC + warp;
                base[u] = (gb + u < ngroups && cc < c1) ? __ldg(&c.cbase[cc]) : 0;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                w[u] = CSB_PAD;
                a[u] = (VM)0;
                if (gb + u < ngroups) {
                    mbar_wait_bounded(&full_bar[rp.stage], rp.phase, err, abort);
                    const int cc = c0 + (gb + u) * Cfg::SC + warp;
                    const unsigned char *sb = smem + (size_t)rp.stage * L::STAGE;
                    if (cc < c1 && !*abort) {
                        w[u] = ((const uint32_t *)sb)[warp * 32 + lane];
                        a[u] = ((const VM *)(sb + L::PK))[warp * 32 + lane];
                    }
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&empty_bar[rp.stage]);
                    rp.next<NST>();
                }
            }
            VV g[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                g[u] = (w[u] & 0xFFFFu) != CSB_PAD ? op.operand((int64_t)base[u] + (w[u] >> 16), 0, s_scal) : (VV)0;
#pragma unroll
            for (int u = 0; u < U; ++u)
                if ((w[u] & 0xFFFFu) != CSB_PAD)
                    sums.add((int)(w[u] & 0xFFFFu), (double)a[u] * (double)g[u]);
        }
        csync();
        for (int i = tid; i < R; i += Cfg::TC) {
            const double acc[1] = {sums.get(i)};
            op.emit((int64_t)(r0 + i), acc, part, s_scal, rv);
        }
        csync();
    }

    if constexpr (NPK > 0)
        grid_reduce_finalize<Cfg::TC, NPK>(part, partials, st, op, s_red, &s_flag, s_sum, tid, csync);
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
