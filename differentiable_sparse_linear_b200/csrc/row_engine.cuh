// Short-row CSR SpMV engine, fed by a TMA bulk-copy pipeline (sm_100a), for matrices whose
// rows hold at most MAXL stored entries (stencils and their triangular factors).
//
// One consumer thread per row (RPT rows per thread per tile).  A tile is a run of whole
// rows holding at most RMAX rows and D items (rows + entries).  The contiguous arrays of a
// tile (row pointers, column indices, values) are streamed into shared memory by a producer
// thread with cp.async.bulk, NST tiles ahead, so a consumer's dependent chain shrinks to the
// operand gather.  Consumers release a stage by arriving on its "empty" mbarrier (one
// arrival per thread), so there is no block-wide barrier in the steady state.  Row sums are
// fp32 when values and vectors are fp32 (at most MAXL terms per row), fp64 otherwise; the
// same fused row epilogue as the tile engine runs on the row's result.
//
// Operand windows: for a banded matrix the columns a tile touches lie in a few contiguous
// row ranges of the gathered vectors (for a 2D grid: the rows one grid line above, the
// tile's own rows, one grid line below).  Those ranges, precomputed per tile on the host
// (at most WSEG segments, 4-row aligned, at most WMAX rows in all), are bulk-copied into the
// stage with the matrix arrays, and the consumers read their operands from shared memory,
// so the gather latency is hidden by the pipeline like the matrix stream's.  A tile whose
// columns do not fit keeps global gathers.
//
// The per-tile producer and consumer steps are device functions (RowTma::issue and
// RowTma::consume) shared by the one-operation kernel below and by the persistent solver
// kernel, which runs the pipeline across the phases of a whole PCG solve.  A "gate" object
// tells the producer when the gathered vectors of a tile's phase are final: window copies
// wait for it, the matrix copies (constant data) do not.
#pragma once

#include <climits>
#include <type_traits>

#include "tile_engine.cuh"

namespace sla {

// TC consumer threads, RPT rows per thread per tile, D items per tile, NST stages, WMAX
// window rows per tile (0: no windows).
template <int K>
struct RowTmaCfg;
template <> struct RowTmaCfg<1> { static constexpr int TC = 256, RPT = 2, D = 3072, NST = 2, WMAX = 2048; };
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

// Position in the stage ring (stage index and mbarrier parity).
struct RingPos {
    int stage = 0;
    uint32_t phase = 0;
    template <int NST>
    __device__ __forceinline__ void next()
    {
        if (++stage == NST) {
            stage = 0;
            phase ^= 1u;
        }
    }
};

// Gate of a single-operation kernel: the gathered vectors are final before it starts.
struct OpenGate {
    __device__ __forceinline__ bool ready() const { return true; }
    __device__ __forceinline__ bool wait() { return true; }
};

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// Order this thread's earlier generic-proxy accesses of global memory with its later
// async-proxy (bulk copy) accesses, and the other way round.
__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

template <int K, typename VM, int MAXL, class Op>
struct RowTma {
    using VV = typename Op::VV;
    using Acc = typename std::conditional<sizeof(VM) == 4 && sizeof(VV) == 4, float, double>::type;
    static constexpr int TC = RowTmaCfg<K>::TC;
    static constexpr int RPT = RowTmaCfg<K>::RPT;
    static constexpr int NST = RowTmaCfg<K>::NST;
    static constexpr int WMAX = RowTmaCfg<K>::WMAX;
    static constexpr int NV = Op::NV;
    static constexpr int NG = Op::NG;
    using L = RowTmaLayout<K, VM, VV, NG>;

    // Producer: write the header of the tile with descriptors (d0, d1) and window wd into
    // the stage buffer sb and issue its copies, completing on `full`.  The matrix copies go
    // out at once; window copies only once gate.wait() says the gathered vectors are final.
    // Returns false when the gate reports a stop: the stage then completes with the matrix
    // copies alone (nothing will read it).
    template <class Gate>
    static __device__ __forceinline__ bool issue(const MatView<VM> &m, const Op &op, const int2 d0,
                                                 const int2 d1, const WinDesc &wd, unsigned char *sb,
                                                 uint64_t *full, Gate &gate)
    {
        const int gs = op.gstride();
        const int r0 = d0.x, r1 = d1.x;
        const int64_t kb = (int64_t)(uint32_t)d0.y, ke = (int64_t)(uint32_t)d1.y;
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
        const uint32_t tx_m = sc.bytes() + sv.bytes() + sr.bytes();
        uint32_t tx_w = 0;
        if (WMAX > 0) {
            *(WinDesc *)(sb + 32) = wd;
            for (int s2 = 0; s2 < wd.nseg; ++s2)
                tx_w += (uint32_t)NG * (uint32_t)wd.l[s2] * (uint32_t)gs * (uint32_t)sizeof(VV);
        }
        const bool split = tx_w > 0 && !gate.ready();
        if (split)
            mbar_expect_tx(full, tx_m);
        else
            mbar_arrive_expect_tx(full, tx_m + tx_w);
        span_issue(sc, sb + L::COL_OFF, m.ci, full);
        span_issue(sv, sb + L::VAL_OFF, m.val, full);
        span_issue(sr, sb + L::RP_OFF, m.rp, full);
        if (tx_w == 0)
            return true;
        if (split) {
            if (!gate.wait()) {
                mbar_arrive(full);
                return false;
            }
            mbar_arrive_expect_tx(full, tx_w);
        }
        int cum = 0;
        for (int s2 = 0; s2 < wd.nseg; ++s2) {
            const uint32_t bytes = (uint32_t)wd.l[s2] * (uint32_t)gs * (uint32_t)sizeof(VV);
#pragma unroll
            for (int g = 0; g < NG; ++g)
                bulk_g2s(sb + L::WIN_OFF + g * L::WIN_STRIDE + (size_t)cum * gs * sizeof(VV),
                         op.gvec(g) + (int64_t)wd.a[s2] * gs, bytes, full);
            cum += wd.l[s2];
        }
        return true;
    }

    // Consumer: wait for the tile in stage buffer sb, run its rows (products, row sums,
    // fused epilogue, dot-product partials into part) and release the stage.
    template <int NR>
    static __device__ __forceinline__ void consume(const MatView<VM> &m, const Op &op, unsigned char *sb,
                                                   uint64_t *full, uint64_t *empty, uint32_t parity,
                                                   double (&part)[NR], const double *s_scal, int tid,
                                                   int *err, volatile int *abort = nullptr)
    {
        const int gs = op.gstride();
        mbar_wait_bounded(full, parity, err, abort);
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
        // window of this tile (nseg == 0: operands come from global memory).  Vector row j
        // sits at window row j + wo[s] for the segment s that holds it: s = number of
        // segment starts after the first that are <= j (segments are sorted and disjoint).
        int nseg = 0, wb1 = INT_MAX, wb2 = INT_MAX, wb3 = INT_MAX, wo0 = 0, wo1 = 0, wo2 = 0, wo3 = 0;
        if (WMAX > 0) {
            const WinDesc *wd = (const WinDesc *)(sb + 32);
            nseg = wd->nseg;
            if (nseg > 0) {
                int cum = 0, a[WSEG], o[WSEG];
#pragma unroll
                for (int s2 = 0; s2 < WSEG; ++s2) {
                    a[s2] = s2 < nseg ? wd->a[s2] : INT_MAX;
                    o[s2] = s2 < nseg ? cum - wd->a[s2] : 0;
                    cum += s2 < nseg ? wd->l[s2] : 0;
                }
                wb1 = a[1];
                wb2 = a[2];
                wb3 = a[3];
                wo0 = o[0];
                wo1 = o[1];
                wo2 = o[2];
                wo3 = o[3];
            }
        }
        const VV *swin = (const VV *)(sb + L::WIN_OFF);
        auto wrow = [&](int j) -> int {   // window row of vector row j (clamped into the window)
            const int o = j >= wb3 ? wo3 : j >= wb2 ? wo2 : j >= wb1 ? wo1 : wo0;
            return min(max(j + o, 0), (WMAX > 0 ? WMAX : 1) - 1);
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
                    if (Op::rv_src(v) < 0) {
                        if (r < nr) {
                            op.load_rv(v, (int64_t)r0 + r, rvals[q].v[v]);
                        } else {
#pragma unroll
                            for (int c = 0; c < K; ++c)
                                rvals[q].v[v][c] = (VV)0;
                        }
                    }
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
                            rvals[q].v[v][c] = live ? wv[Op::rv_src(v)][(size_t)rw * gs + c] : (VV)0;
                Acc a[K];
#pragma unroll
                for (int c = 0; c < K; ++c)
                    a[c] = (Acc)0;
#pragma unroll
                for (int u = 0; u < MAXL; ++u) {
                    if (u < n_) {
                        // the window was built from exactly these columns and rows
                        const int w = wrow(cc[o + u]);
                        const Acc av = (Acc)vv[o + u];
#pragma unroll
                        for (int c = 0; c < K; ++c) {
                            VV gv[NG];
#pragma unroll
                            for (int g = 0; g < NG; ++g)
                                gv[g] = wv[g][(size_t)w * gs + c];
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
            mbar_arrive(empty);
#pragma unroll
            for (int q = 0; q < RPT; ++q) {
                const int r = tid + q * TC;
                if (r < nr)
                    op.emit((int64_t)r0 + r, acc[q], part, s_scal, rvals[q]);
            }
            return;
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
            for (int v = 0; v < NV; ++v) {
                if (live) {
                    op.load_rv(v, (int64_t)r0 + r, rvals[q].v[v]);
                } else {
#pragma unroll
                    for (int c = 0; c < K; ++c)
                        rvals[q].v[v][c] = (VV)0;
                }
            }
#pragma unroll
            for (int u = 0; u < MAXL; ++u) {
                cj[q][u] = u < len[q] ? cc[off[q] + u] : 0;
                av[q][u] = u < len[q] ? vv[off[q] + u] : (VM)0;
            }
        }
        // the stage's shared memory is no longer read: hand it back to the producer
        fence_proxy_async_smem();
        mbar_arrive(empty);
        VV ov[RPT][MAXL][K];
#pragma unroll
        for (int q = 0; q < RPT; ++q)
#pragma unroll
            for (int u = 0; u < MAXL; ++u) {
                if (u < len[q]) {
                    op.operand_row(cj[q][u], ov[q][u], s_scal);
                } else {
#pragma unroll
                    for (int c = 0; c < K; ++c)
                        ov[q][u][c] = (VV)0;
                }
            }
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
};

// One fused operation (SpMV with its row epilogue and dot products) in one launch:
// producer thread TC walks the block's tiles round-robin over the grid; the last block to
// finish reduces the per-block partials in block order and runs op.finalize.
template <int K, typename VM, int MAXL, class Op>
__global__ void __launch_bounds__(RowTmaCfg<K>::TC + 32)
k_rows_tma(const MatView<VM> m, const WinDesc *win, const Op op, double *partials, PcgState *st,
           int *err)
{
    using E = RowTma<K, VM, MAXL, Op>;
    constexpr int TC = E::TC;
    constexpr int NST = E::NST;
    constexpr int NPK = Op::NP * K;
    constexpr int NR = NPK > 0 ? NPK : 1;
    constexpr size_t PITCH = E::L::BYTES;

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

    // ---------------------------------------------------------------- producer
    if (threadIdx.x >= TC) {
        if (threadIdx.x != TC)
            return;
        OpenGate gate;
        RingPos rp;
        // descriptors are loaded one tile ahead, so their latency overlaps the stage wait
        int2 n0 = make_int2(0, 0), n1 = make_int2(0, 0);
        WinDesc nw;
        nw.nseg = 0;
        int issued_phase[NST];             // phase parity of each stage's last issued copies
#pragma unroll
        for (int s = 0; s < NST; ++s)
            issued_phase[s] = -1;
        if (blockIdx.x < m.n_tiles) {
            n0 = m.desc[blockIdx.x];
            n1 = m.desc[blockIdx.x + 1];
            if (E::WMAX > 0 && win)
                nw = win[blockIdx.x];
        }
        for (int t = blockIdx.x; t < m.n_tiles; t += gridDim.x) {
            const int2 d0 = n0, d1 = n1;
            const WinDesc wd = nw;
            const int tn = t + gridDim.x;
            if (tn < m.n_tiles) {
                n0 = m.desc[tn];
                n1 = m.desc[tn + 1];
                if (E::WMAX > 0 && win)
                    nw = win[tn];
            }
            mbar_wait_bounded(&empty_bar[rp.stage], rp.phase ^ 1u, err);
            E::issue(m, op, d0, d1, wd, smem + (size_t)rp.stage * PITCH, &full_bar[rp.stage], gate);
            issued_phase[rp.stage] = (int)rp.phase;
            rp.next<NST>();
        }
        // every copy has landed and been read before the block exits: the consumers release
        // each stage after its copies landed; if a consumer's wait ran out instead, the
        // stage's last copies may still be in flight, so wait (bounded) for their completion
        // too -- no bulk copy may still write this block's shared memory after it exits
        for (int s = 0; s < NST; ++s) {
            mbar_wait_bounded(&empty_bar[rp.stage], rp.phase ^ 1u, err);
            rp.next<NST>();
        }
        for (int s = 0; s < NST; ++s)
            if (issued_phase[s] >= 0)
                mbar_wait_bounded(&full_bar[s], (uint32_t)issued_phase[s], err);
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int tid = threadIdx.x;
    double part[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i)
        part[i] = 0.0;
    RingPos rp;
    for (int t = blockIdx.x; t < m.n_tiles; t += gridDim.x) {
        E::consume(m, op, smem + (size_t)rp.stage * PITCH, &full_bar[rp.stage], &empty_bar[rp.stage],
                   rp.phase, part, s_scal, tid, err);
        rp.next<NST>();
    }

    if constexpr (NPK > 0) {
        auto sync = [] { consumer_sync(TC); };
        grid_reduce_finalize<TC, NPK>(part, partials, st, op, s_red, &s_flag, s_sum, tid, sync);
    }
}

}  // namespace sla
