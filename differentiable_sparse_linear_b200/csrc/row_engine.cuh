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

namespace sla {

// ------------------------------------------------------------------ TMA-fed short-row engine
// Same per-row work as k_rows, but the contiguous arrays of a tile of rows (row pointers,
// column indices, values) are streamed into shared memory by a producer warp with
// cp.async.bulk, NST tiles ahead, so a consumer thread's dependent chain shrinks to the
// operand gather.  Tiles hold at most RMAX rows (RPT per consumer thread) and at most D
// items (rows + entries); rows have at most MAXL entries, so there are no long rows.
// Consumers release a stage by arriving on its "empty" mbarrier (one arrival per thread),
// so no block-wide barrier is needed in the steady state.
//
// Operand windows (WIN): for a banded matrix the columns a tile touches lie in a few
// contiguous row ranges of the gathered vectors (for a 2D grid: the rows one grid line
// above, the tile's own rows, one grid line below).  Those ranges, precomputed per tile on
// the host (at most WSEG segments, 4-row aligned, at most WMAX rows in all), are bulk-copied
// into the stage with the matrix arrays, and the consumers read their operands from shared
// memory.  The gather latency is then hidden by the pipeline like the matrix stream's.  A
// tile whose columns do not fit keeps global gathers.
template <int K>
struct RowTmaCfg;
template <> struct RowTmaCfg<1> { static constexpr int TC = 256, RPT = 2, D = 2048, NST = 2, WMAX = 2048; };
template <> struct RowTmaCfg<2> { static constexpr int TC = 256, RPT = 2, D = 2048, NST = 2, WMAX = 1024; };
template <> struct RowTmaCfg<4> { static constexpr int TC = 256, RPT = 1, D = 2048, NST = 2, WMAX = 0; };
template <> struct RowTmaCfg<8> { static constexpr int TC = 256, RPT = 1, D = 2048, NST = 2, WMAX = 0; };
template <> struct RowTmaCfg<16> { static constexpr int TC = 128, RPT = 1, D = 1024, NST = 2, WMAX = 0; };

template <int K, typename VM, typename VV, int NG>
struct RowTmaLayout {
    static constexpr int D = RowTmaCfg<K>::D;
    static constexpr int RMAX = RowTmaCfg<K>::TC * RowTmaCfg<K>::RPT;
    static constexpr int WMAX = RowTmaCfg<K>::WMAX;
    static constexpr int PAD = 8;
    static constexpr size_t align16(size_t b) { return (b + 15) & ~(size_t)15; }
    static constexpr size_t HDR = 128;
    static constexpr size_t COL_OFF = HDR;
    static constexpr size_t VAL_OFF = COL_OFF + align16((D + PAD) * 4);
    static constexpr size_t RP_OFF = VAL_OFF + align16((D + PAD) * sizeof(VM));
    static constexpr size_t WIN_OFF = RP_OFF + align16((RMAX + 1 + PAD) * 4);
    static constexpr size_t WIN_STRIDE = align16((size_t)WMAX * K * sizeof(VV));
    static constexpr size_t BYTES = align16(WIN_OFF + (WMAX > 0 ? NG : 0) * WIN_STRIDE);
};

// Own-row vector values loaded into registers before the row's gathers.
template <typename VV, int K, int NV>
struct RowVals {
    VV v[NV > 0 ? NV : 1][K];
    __device__ __forceinline__ VV get(int vi, int64_t, int c) const { return v[vi][c]; }
};

template <int K, typename VM, int MAXL, class Op>
__global__ void __launch_bounds__(RowTmaCfg<K>::TC + 32)
k_rows_tma(const MatView<VM> m, const WinDesc *win, const Op op, double *partials, PcgState *st,
           int *err)
{
    using VV = typename Op::VV;
    using Acc = typename std::conditional<sizeof(VM) == 4 && sizeof(VV) == 4, float, double>::type;
    constexpr int TC = RowTmaCfg<K>::TC;
    constexpr int RPT = RowTmaCfg<K>::RPT;
    constexpr int NST = RowTmaCfg<K>::NST;
    constexpr int WMAX = RowTmaCfg<K>::WMAX;
    constexpr int NV = Op::NV;
    constexpr int NG = Op::NG;
    constexpr int NPK = Op::NP * K;
    constexpr int NR = NPK > 0 ? NPK : 1;
    using L = RowTmaLayout<K, VM, VV, NG>;

    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ uint64_t full_bar[NST], empty_bar[NST];
    __shared__ double s_red[(TC / 32) * NR];
    __shared__ double s_scal[Op::NS > 0 ? Op::NS : 1];
    __shared__ double s_sum[NR];
    __shared__ int s_flag;

    if (op.skip())
        return;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], TC);
        }
        fence_mbar_init();
        op.stage(s_scal);
    }
    __syncthreads();
    const int gs = op.gstride();

    // ---------------------------------------------------------------- producer
    if (threadIdx.x >= TC) {
        if (threadIdx.x != TC)
            return;
        int stage = 0;
        uint32_t phase = 0;
        for (int t = blockIdx.x; t < m.n_tiles; t += gridDim.x) {
            const int2 d0 = m.desc[t], d1 = m.desc[t + 1];
            WinDesc wd;
            if (WMAX > 0 && win)
                wd = win[t];
            else
                wd.nseg = 0;
            const int r0 = d0.x, r1 = d1.x;
            const int64_t kb = (int64_t)(uint32_t)d0.y, ke = (int64_t)(uint32_t)d1.y;
            mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, err);
            unsigned char *sb = smem + (size_t)stage * L::BYTES;
            const Span<4> sc(kb, ke, m.nnz);
            const Span<sizeof(VM)> sv(kb, ke, m.nnz);
            const Span<4> sr(r0, (int64_t)r1 + 1, m.n + 1);
            int32_t *hdr = (int32_t *)sb;
            hdr[0] = r0;
            hdr[1] = r1;
            hdr[2] = (int32_t)kb;
            hdr[3] = (int32_t)ke;
            hdr[4] = (int32_t)(kb - sc.ab);          // smem index of entry kb in col[]
            hdr[5] = (int32_t)(kb - sv.ab);          // ... in val[]
            hdr[6] = (int32_t)(r0 - sr.ab);          // smem index of row_ptr[r0]
            hdr[7] = (sc.tail < ke || sv.tail < ke || sr.tail < (int64_t)r1 + 1) ? 1 : 0;
            uint32_t tx = sc.bytes() + sv.bytes() + sr.bytes();
            if (WMAX > 0) {
                *(WinDesc *)(sb + 32) = wd;
                for (int s2 = 0; s2 < wd.nseg; ++s2)
                    tx += (uint32_t)NG * (uint32_t)wd.l[s2] * (uint32_t)gs * (uint32_t)sizeof(VV);
            }
            mbar_arrive_expect_tx(&full_bar[stage], tx);
            span_issue(sc, sb + L::COL_OFF, m.ci, &full_bar[stage]);
            span_issue(sv, sb + L::VAL_OFF, m.val, &full_bar[stage]);
            span_issue(sr, sb + L::RP_OFF, m.rp, &full_bar[stage]);
            if (WMAX > 0) {
                int cum = 0;
                for (int s2 = 0; s2 < wd.nseg; ++s2) {
                    const uint32_t bytes = (uint32_t)wd.l[s2] * (uint32_t)gs * (uint32_t)sizeof(VV);
#pragma unroll
                    for (int g = 0; g < NG; ++g)
                        bulk_g2s(sb + L::WIN_OFF + g * L::WIN_STRIDE + (size_t)cum * gs * sizeof(VV),
                                 op.gvec(g) + (int64_t)wd.a[s2] * gs, bytes, &full_bar[stage]);
                    cum += wd.l[s2];
                }
            }
            if (++stage == NST) {
                stage = 0;
                phase ^= 1u;
            }
        }
        for (int s = 0; s < NST; ++s) {
            mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, err);
            if (++stage == NST) {
                stage = 0;
                phase ^= 1u;
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int tid = threadIdx.x;
    double part[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i)
        part[i] = 0.0;
    int stage = 0;
    uint32_t phase = 0;
    for (int t = blockIdx.x; t < m.n_tiles; t += gridDim.x) {
        mbar_wait_bounded(&full_bar[stage], phase, err);
        unsigned char *sb = smem + (size_t)stage * L::BYTES;
        const int32_t *hdr = (const int32_t *)sb;
        const int r0 = hdr[0], r1 = hdr[1];
        const int nr = r1 - r0;
        int32_t *s_col = (int32_t *)(sb + L::COL_OFF);
        VM *s_val = (VM *)(sb + L::VAL_OFF);
        int32_t *s_rp = (int32_t *)(sb + L::RP_OFF);
        if (hdr[7]) {
            // the end of an array: load what the bulk copies could not move
            const int64_t kb = (int64_t)(uint32_t)hdr[2], ke = (int64_t)(uint32_t)hdr[3];
            const Span<4> sc(kb, ke, m.nnz);
            const Span<sizeof(VM)> sv(kb, ke, m.nnz);
            const Span<4> sr(r0, (int64_t)r1 + 1, m.n + 1);
            span_tail(sc, ke, s_col, m.ci, tid, TC);
            span_tail(sv, ke, s_val, m.val, tid, TC);
            span_tail(sr, (int64_t)r1 + 1, s_rp, m.rp, tid, TC);
            consumer_sync(TC);
        }
        const int32_t kb32 = hdr[2];
        const int32_t *cc = s_col + hdr[4];
        const VM *vv = s_val + hdr[5];
        const int32_t *rpp = s_rp + hdr[6];
        // window of this tile (nseg == 0: operands come from global memory)
        int nseg = 0, wa[WSEG], wl[WSEG], wc[WSEG];
        if (WMAX > 0) {
            const WinDesc *wd = (const WinDesc *)(sb + 32);
            nseg = wd->nseg;
            int cum = 0;
#pragma unroll
            for (int s2 = 0; s2 < WSEG; ++s2) {
                wa[s2] = wd->a[s2];
                wl[s2] = s2 < nseg ? wd->l[s2] : 0;
                wc[s2] = cum;
                cum += wl[s2];
            }
        }
        const VV *swin = (const VV *)(sb + L::WIN_OFF);
        auto wrow = [&](int j) -> int {   // window row of vector row j, -1 if outside
            int pos = -1;
#pragma unroll
            for (int s2 = 0; s2 < WSEG; ++s2)
                if ((unsigned)(j - wa[s2]) < (unsigned)wl[s2])
                    pos = wc[s2] + (j - wa[s2]);
            return pos;
        };

        RowVals<VV, K, NV> rvals[RPT];
        if (WMAX > 0 && nseg > 0) {
            // windowed tile: operands and own-row values of gathered vectors come from shared
            // memory, so the row sums are formed while reading; only the other own-row
            // vectors are loaded from global memory (issued first).
            const VV *wv[NG];
#pragma unroll
            for (int g = 0; g < NG; ++g)
                wv[g] = swin + (size_t)g * (L::WIN_STRIDE / sizeof(VV));
#pragma unroll
            for (int q = 0; q < RPT; ++q) {
                const int r = tid + q * TC;
#pragma unroll
                for (int v = 0; v < NV; ++v)
                    if (Op::rv_src(v) < 0)
#pragma unroll
                        for (int c = 0; c < K; ++c)
                            rvals[q].v[v][c] = r < nr ? op.row_vec(v)[((int64_t)r0 + r) * K + c] : (VV)0;
            }
            double acc[RPT][K];
#pragma unroll
            for (int q = 0; q < RPT; ++q) {
                const int r = tid + q * TC;
                const bool live = r < nr;
                const int o = live ? rpp[r] - kb32 : 0;
                const int n_ = live ? rpp[r + 1] - kb32 - o : 0;
                const int rw = live ? wrow(r0 + r) : 0;
#pragma unroll
                for (int v = 0; v < NV; ++v)
                    if (Op::rv_src(v) >= 0)
#pragma unroll
                        for (int c = 0; c < K; ++c)
                            rvals[q].v[v][c] = !live ? (VV)0
                                               : rw >= 0 ? wv[Op::rv_src(v)][(size_t)rw * gs + c]
                                                         : op.row_vec(v)[((int64_t)r0 + r) * K + c];
                Acc a[K];
#pragma unroll
                for (int c = 0; c < K; ++c)
                    a[c] = (Acc)0;
#pragma unroll
                for (int u = 0; u < MAXL; ++u) {
                    if (u < n_) {
                        const int j = cc[o + u];
                        const int w = wrow(j);       // always inside: the window was built from these columns
                        const Acc av = (Acc)vv[o + u];
#pragma unroll
                        for (int c = 0; c < K; ++c) {
                            VV gv[NG];
#pragma unroll
                            for (int g = 0; g < NG; ++g)
                                gv[g] = w >= 0 ? wv[g][(size_t)w * gs + c] : op.gvec(g)[(int64_t)j * gs + c];
                            a[c] = fma(av, (Acc)op.combine(gv, c, s_scal), a[c]);
                        }
                    }
                }
#pragma unroll
                for (int c = 0; c < K; ++c)
                    acc[q][c] = (double)a[c];
            }
            // the stage's shared memory is no longer read: hand it back to the producer
            fence_proxy_async_smem();
            mbar_arrive(&empty_bar[stage]);
            if (++stage == NST) {
                stage = 0;
                phase ^= 1u;
            }
#pragma unroll
            for (int q = 0; q < RPT; ++q) {
                const int r = tid + q * TC;
                if (r < nr)
                    op.emit((int64_t)r0 + r, acc[q], part, s_scal, rvals[q]);
            }
            continue;
        }

        // global gathers: every load of this thread in flight at once
        int len[RPT], off[RPT];
        int cj[RPT][MAXL];
        VM av[RPT][MAXL];
#pragma unroll
        for (int q = 0; q < RPT; ++q) {
            const int r = tid + q * TC;
            const bool live = r < nr;
            off[q] = live ? rpp[r] - kb32 : 0;
            len[q] = live ? rpp[r + 1] - kb32 - off[q] : 0;
#pragma unroll
            for (int v = 0; v < NV; ++v)
#pragma unroll
                for (int c = 0; c < K; ++c)
                    rvals[q].v[v][c] = live ? op.row_vec(v)[((int64_t)r0 + r) * K + c] : (VV)0;
#pragma unroll
            for (int u = 0; u < MAXL; ++u) {
                cj[q][u] = u < len[q] ? cc[off[q] + u] : 0;
                av[q][u] = u < len[q] ? vv[off[q] + u] : (VM)0;
            }
        }
        // the stage's shared memory is no longer read: hand it back to the producer
        fence_proxy_async_smem();
        mbar_arrive(&empty_bar[stage]);
        if (++stage == NST) {
            stage = 0;
            phase ^= 1u;
        }
        VV ov[RPT][MAXL][K];
#pragma unroll
        for (int q = 0; q < RPT; ++q)
#pragma unroll
            for (int u = 0; u < MAXL; ++u)
#pragma unroll
                for (int c = 0; c < K; ++c)
                    ov[q][u][c] = u < len[q] ? op.operand(cj[q][u], c, s_scal) : (VV)0;
#pragma unroll
        for (int q = 0; q < RPT; ++q) {
            const int r = tid + q * TC;
            if (r < nr) {
                double acc[K];
#pragma unroll
                for (int c = 0; c < K; ++c) {
                    Acc a = (Acc)0;
#pragma unroll
                    for (int u = 0; u < MAXL; ++u)
                        a = fma((Acc)av[q][u], (Acc)ov[q][u][c], a);
                    acc[c] = (double)a;
                }
                op.emit((int64_t)r0 + r, acc, part, s_scal, rvals[q]);
            }
        }
    }

    if constexpr (NPK > 0) {
        auto sync = [] { consumer_sync(TC); };
        grid_reduce_finalize<TC, NPK>(part, partials, st, op, s_red, &s_flag, s_sum, tid, sync);
    }
}

}  // namespace sla
