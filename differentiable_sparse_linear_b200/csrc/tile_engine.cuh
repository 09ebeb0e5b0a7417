// Load-balanced CSR SpMV engine with fused row epilogues and fused dot products, fed by a
// TMA bulk-copy pipeline (sm_100a).
//
// Work unit: a "tile" = a run of whole rows holding at most D items (rows + stored entries)
// and at most RMAX rows, built once per matrix on the host.  A row with D or more entries is
// a tile of its own ("long row") and is streamed in chunks of D entries.  Rows never
// straddle tiles, so every row is finished inside one block, where its epilogue (vector
// updates, dot-product partials) runs.
//
// Block = 1 producer warp + consumer warps.  The producer walks the block's tiles
// (round-robin over the grid) and, for each chunk, issues cp.async.bulk copies of the
// chunk's column indices, values and row pointers, and of the own-row slices of the vectors
// the epilogue needs, into one of NST shared-memory stages; a "full" mbarrier per stage
// counts the bytes in.  Consumers wait on it, then
//   1. form every product A_k * operand(col_k) in fp64 (the operand is a gathered vector
//      value; K right-hand sides read K contiguous values), all loads independent;
//   2. split the tile's items evenly over the threads along the merge path of (row ends,
//      entries) -- the merge-based SpMV decomposition -- and sum each thread's run;
//   3. finish a row spanning several threads in the thread holding its end, which adds the
//      partial sums the earlier threads left in shared memory, in a fixed order;
// and release the stage through an "empty" mbarrier.  Unaligned edges of each copy (the
// bulk engine moves 16-byte-aligned spans) are loaded by the consumers with plain loads.
// Every mbarrier wait is bounded in time; a wait that runs out sets an error word and the
// block carries on to a normal exit (results are then flagged invalid by the host).
//
// The block's dot-product partial is a fixed-order sum; the last block to finish reduces
// the per-block partials in block order and runs the operation's scalar finalisation, so
// results are deterministic for a given device.
#pragma once

#include "sla_internal.cuh"

namespace sla {

// ------------------------------------------------------------------ configuration
template <int K>
struct TileCfg;
// TC: consumer threads; D: items (rows + entries) per tile and entries per long-row chunk;
// RMAX: rows per tile; NST: pipeline stages.
template <> struct TileCfg<1> { static constexpr int TC = 256, D = 1024, RMAX = 512, NST = 2; };
template <> struct TileCfg<2> { static constexpr int TC = 256, D = 512, RMAX = 256, NST = 2; };
template <> struct TileCfg<4> { static constexpr int TC = 256, D = 512, RMAX = 256, NST = 2; };
template <> struct TileCfg<8> { static constexpr int TC = 128, D = 256, RMAX = 128, NST = 2; };
template <> struct TileCfg<16> { static constexpr int TC = 128, D = 128, RMAX = 64, NST = 2; };

constexpr unsigned long long WAIT_LIMIT_NS = 4000000000ull;   // 4 s per mbarrier wait

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// try_wait that lets the hardware suspend the thread until the phase completes (or the
// hinted time passes), so waiting warps leave the issue slots to the working ones.
constexpr uint32_t SUSPEND_HINT_NS = 100000;
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(SUSPEND_HINT_NS)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Wait for the phase with the given parity; give up after WAIT_LIMIT_NS and flag it.  Also
// give up at once when *abort (a block-wide flag, may be null) is set; a wait that runs
// out sets it, so one stalled wait does not leave the block's later waits running out too.
// The clock is read only every 16th round.
__device__ __forceinline__ void mbar_wait_bounded(uint64_t *bar, uint32_t parity, int *err,
                                                  volatile int *abort = nullptr)
{
    if (mbar_try_wait(bar, parity))
        return;
    const unsigned long long t0 = global_ns();
    for (unsigned i = 1;; ++i) {
        if (mbar_try_wait_sleep(bar, parity))
            return;
        if ((i & 15u) == 0) {
            if (abort && *abort)
                return;
            if (global_ns() - t0 > WAIT_LIMIT_NS) {
                atomicOr(err, 2);
                if (abort)
                    *abort = 1;
                return;
            }
        }
    }
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void consumer_sync(int nthreads)
{
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// ------------------------------------------------------------------ reductions
// Sum N values over the NT threads of a (sub)block that synchronises with `sync`.
// On return thread i (< N) holds the total of value i in v[0]; the order is fixed.
template <int NT, int N, class Sync>
__device__ __forceinline__ void block_sum(double (&v)[N], double *s_red, int tid, Sync sync)
{
    const int lane = tid & 31, warp = tid >> 5;
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
    sync();
    double t = 0.0;
    if (tid < N) {
#pragma unroll
        for (int w = 0; w < NT / 32; ++w)
            t += s_red[w * N + tid];
    }
    sync();
    v[0] = t;
}

// Write this block's partials; the last block to finish reduces all blocks' partials
// (block order) and calls op.finalize(sums) on thread 0.
template <int NT, int N, class Op, class Sync>
__device__ __forceinline__ void grid_reduce_finalize(double (&part)[N], double *partials,
                                                     PcgState *st, const Op &op, double *s_red,
                                                     int *s_flag, double *s_sum, int tid, Sync sync)
{
    block_sum<NT, N>(part, s_red, tid, sync);
    if (tid < N)
        partials[(size_t)blockIdx.x * N + tid] = part[0];
    __threadfence();
    sync();
    if (tid == 0) {
        unsigned int t = atomicAdd(&st->ticket, 1u);
        *s_flag = (t == gridDim.x - 1);
    }
    sync();
    if (!*s_flag)
        return;
    __threadfence();
    double v[N];
#pragma unroll
    for (int i = 0; i < N; ++i)
        v[i] = 0.0;
    for (int c = tid; c < (int)gridDim.x; c += NT) {
#pragma unroll
        for (int i = 0; i < N; ++i)
            v[i] += __ldcg(&partials[(size_t)c * N + i]);
    }
    block_sum<NT, N>(v, s_red, tid, sync);
    if (tid < N)
        s_sum[tid] = v[0];
    sync();
    if (tid == 0) {
        op.finalize(s_sum);
        st->ticket = 0u;
    }
}

// ------------------------------------------------------------------ staged rows
// Own-row vector values of the current tile, staged in shared memory.
template <typename VV, int K, int NV>
struct RowVecs {
    const VV *base[NV > 0 ? NV : 1];
    int64_t r0;
    __device__ __forceinline__ VV get(int v, int64_t i, int c) const { return base[v][(i - r0) * K + c]; }
};

// One stage of the pipeline: header + arrays (capacities padded for the alignment shift
// of each bulk copy: up to 2 * (16 / S - 1) extra elements).
template <int K, typename VM, typename VV, int NV>
struct StageLayout {
    static constexpr int D = TileCfg<K>::D;
    static constexpr int RMAX = TileCfg<K>::RMAX;
    static constexpr int PAD = 8;
    static constexpr size_t align16(size_t b) { return (b + 15) & ~(size_t)15; }
    static constexpr size_t HDR = 32;
    static constexpr size_t COL_OFF = HDR;
    static constexpr size_t VAL_OFF = COL_OFF + align16((D + PAD) * 4);
    static constexpr size_t RP_OFF = VAL_OFF + align16((D + PAD) * sizeof(VM));
    static constexpr size_t RV_OFF = RP_OFF + align16((RMAX + 1 + PAD) * 4);
    static constexpr size_t RV_STRIDE = align16((RMAX * K + PAD) * sizeof(VV));
    static constexpr size_t BYTES = align16(RV_OFF + (NV > 0 ? NV : 0) * RV_STRIDE);
};

// Of the element range [b, e) of an array of `len` elements of S bytes, the bulk engine
// moves the 16-byte-aligned span [ab, ce) that lies inside the array; the rest, [tail, e),
// is loaded with plain loads.  Element g lives at shared index g - ab.
template <int S>
struct Span {
    int64_t ab, ce, tail;
    __device__ __forceinline__ Span(int64_t b, int64_t e, int64_t len)
    {
        constexpr int64_t A = 16 / S;
        ab = b & ~(A - 1);
        const int64_t up = (e + A - 1) & ~(A - 1);
        const int64_t safe = len & ~(A - 1);
        ce = up < safe ? up : safe;
        if (e <= b || ce <= ab) {
            ce = ab;
            tail = b;
        } else {
            tail = ce < e ? ce : e;
        }
    }
    __device__ __forceinline__ uint32_t bytes() const { return (uint32_t)((ce - ab) * S); }
};

template <int S>
__device__ __forceinline__ void span_issue(const Span<S> &sp, void *smem, const void *gbase, uint64_t *bar)
{
    if (sp.ce > sp.ab)
        bulk_g2s(smem, (const char *)gbase + sp.ab * S, sp.bytes(), bar);
}

template <int S, typename E>
__device__ __forceinline__ void span_tail(const Span<S> &sp, int64_t e, E *smem, const E *gbase, int tid, int nt)
{
    for (int64_t g = sp.tail + tid; g < e; g += nt)
        smem[g - sp.ab] = gbase[g];
}

constexpr int HDR_LONG = 1, HDR_LAST = 2;

// ------------------------------------------------------------------ the kernel
// Op concept:
//   using VV;                                      vector element type
//   static constexpr int NP, NS, NV;               dots per rhs, staged scalars, staged row vectors
//   const VV *row_vec(int v) const;                base of staged own-row vector v (K-interleaved)
//   bool skip() const;  void stage(double *s) const;
//   VV operand(int64_t j, int c, const double *s) const;              gathered value
//   template <int N> void emit(int64_t i, const double (&acc)[K], double (&part)[N],
//                              const double *s, const RowVecs<VV,K,NV> &rv) const;
//   void finalize(const double *sums) const;       sums[p*K + c]
template <int K, typename VM, class Op>
__global__ void __launch_bounds__(TileCfg<K>::TC + 32)
k_tile(const MatView<VM> m, const Op op, double *partials, PcgState *st, int *err)
{
    using VV = typename Op::VV;
    constexpr int TC = TileCfg<K>::TC;
    constexpr int D = TileCfg<K>::D;
    constexpr int NST = TileCfg<K>::NST;
    constexpr int IPT = D / TC;
    constexpr int NV = Op::NV;
    constexpr int NPK = Op::NP * K;
    constexpr int NR = NPK > K ? NPK : K;
    using L = StageLayout<K, VM, VV, NV>;

    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ uint64_t full_bar[NST], empty_bar[NST];
    __shared__ double s_prod[D * K];
    __shared__ int32_t s_crow[TC];
    __shared__ double s_cval[TC * K];
    __shared__ double s_red[(TC / 32) * NR];
    __shared__ double s_scal[Op::NS > 0 ? Op::NS : 1];
    __shared__ double s_sum[NR];
    __shared__ int s_flag;

    if (op.skip())
        return;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        fence_mbar_init();
        op.stage(s_scal);
    }
    __syncthreads();

    // ---------------------------------------------------------------- producer warp
    if (threadIdx.x >= TC) {
        if (threadIdx.x != TC)
            return;
        int stage = 0;
        uint32_t phase = 0;
        for (int t = blockIdx.x; t < m.n_tiles; t += gridDim.x) {
            const int2 d0 = m.desc[t], d1 = m.desc[t + 1];
            const int r0 = d0.x, r1 = d1.x;
            const int64_t k0 = (int64_t)(uint32_t)d0.y, k1 = (int64_t)(uint32_t)d1.y;
            const bool longrow = (int64_t)(r1 - r0) + (k1 - k0) > D;
            const int nch = longrow ? (int)((k1 - k0 + D - 1) / D) : 1;
            for (int ch = 0; ch < nch; ++ch) {
                mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, err);
                unsigned char *sb = smem + (size_t)stage * L::BYTES;
                const int64_t kb = longrow ? k0 + (int64_t)ch * D : k0;
                const int64_t ke = longrow ? (kb + D < k1 ? kb + D : k1) : k1;
                int32_t *hdr = (int32_t *)sb;
                hdr[0] = r0;
                hdr[1] = r1;
                hdr[2] = (int32_t)kb;
                hdr[3] = (int32_t)ke;
                hdr[4] = (longrow ? HDR_LONG : 0) | (ch == nch - 1 ? HDR_LAST : 0);
                const Span<4> sc(kb, ke, m.nnz);
                const Span<sizeof(VM)> sv(kb, ke, m.nnz);
                const Span<4> sr(r0, longrow ? r0 : (int64_t)r1 + 1, m.n + 1);
                uint32_t tx = sc.bytes() + sv.bytes() + sr.bytes();
#pragma unroll
                for (int v = 0; v < NV; ++v)
                    tx += Span<sizeof(VV)>((int64_t)r0 * K, (int64_t)r1 * K, m.n * K).bytes();
                // the arrive registers the byte count, then the copies credit it
                mbar_arrive_expect_tx(&full_bar[stage], tx);
                span_issue(sc, sb + L::COL_OFF, m.ci, &full_bar[stage]);
                span_issue(sv, sb + L::VAL_OFF, m.val, &full_bar[stage]);
                span_issue(sr, sb + L::RP_OFF, m.rp, &full_bar[stage]);
#pragma unroll
                for (int v = 0; v < NV; ++v)
                    span_issue(Span<sizeof(VV)>((int64_t)r0 * K, (int64_t)r1 * K, m.n * K),
                               sb + L::RV_OFF + v * L::RV_STRIDE, op.row_vec(v), &full_bar[stage]);
                if (++stage == NST) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // drain: every fill issued must be consumed (and so have landed) before exit
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
    auto sync = [] { consumer_sync(TC); };
    double part[NPK > 0 ? NPK : 1];
#pragma unroll
    for (int i = 0; i < (NPK > 0 ? NPK : 1); ++i)
        part[i] = 0.0;
    double lacc[K];
#pragma unroll
    for (int c = 0; c < K; ++c)
        lacc[c] = 0.0;

    int stage = 0;
    uint32_t phase = 0;
    for (int t = blockIdx.x; t < m.n_tiles; t += gridDim.x) {
        int flags = 0;
        do {
            mbar_wait_bounded(&full_bar[stage], phase, err);
            unsigned char *sb = smem + (size_t)stage * L::BYTES;
            const int32_t *hdr = (const int32_t *)sb;
            const int r0 = hdr[0], r1 = hdr[1];
            const int64_t kb = (int64_t)(uint32_t)hdr[2], ke = (int64_t)(uint32_t)hdr[3];
            flags = hdr[4];
            const bool is_long = flags & HDR_LONG;
            const int nr = r1 - r0;
            const int nk = (int)(ke - kb);
            int32_t *s_col = (int32_t *)(sb + L::COL_OFF);
            VM *s_val = (VM *)(sb + L::VAL_OFF);
            int32_t *s_rp = (int32_t *)(sb + L::RP_OFF);
            const Span<4> sc(kb, ke, m.nnz);
            const Span<sizeof(VM)> sv(kb, ke, m.nnz);
            const Span<4> sr(r0, is_long ? r0 : (int64_t)r1 + 1, m.n + 1);
            // the edges the bulk copies could not move
            span_tail(sc, ke, s_col, m.ci, tid, TC);
            span_tail(sv, ke, s_val, m.val, tid, TC);
            if (!is_long)
                span_tail(sr, (int64_t)r1 + 1, s_rp, m.rp, tid, TC);
            RowVecs<VV, K, NV> rv;
            rv.r0 = r0;
#pragma unroll
            for (int v = 0; v < NV; ++v) {
                const Span<sizeof(VV)> sx((int64_t)r0 * K, (int64_t)r1 * K, m.n * K);
                VV *s_v = (VV *)(sb + L::RV_OFF + v * L::RV_STRIDE);
                span_tail(sx, (int64_t)r1 * K, s_v, op.row_vec(v), tid, TC);
                rv.base[v] = s_v + ((int64_t)r0 * K - sx.ab);
            }
            sync();
            const int32_t *cc = s_col + (kb - sc.ab);
            const VM *vv = s_val + (kb - sv.ab);

            if (is_long) {
                // chunk of one long row: thread-strided partial sums, kept across chunks;
                // all of this thread's operand loads are issued before the first use
                constexpr int GL = (D + TC - 1) / TC;
                double ov[GL][K];
#pragma unroll
                for (int u = 0; u < GL; ++u) {
                    const int e = tid + u * TC;
#pragma unroll
                    for (int c = 0; c < K; ++c)
                        ov[u][c] = e < nk ? (double)op.operand(cc[e], c, s_scal) : 0.0;
                }
#pragma unroll
                for (int u = 0; u < GL; ++u) {
                    const int e = tid + u * TC;
                    if (e < nk) {
                        const double a = (double)vv[e];
#pragma unroll
                        for (int c = 0; c < K; ++c)
                            lacc[c] = fma(a, ov[u][c], lacc[c]);
                    }
                }
                if (flags & HDR_LAST) {
#pragma unroll
                    for (int c = 0; c < K; ++c) {
                        double one[1] = {lacc[c]};
                        block_sum<TC, 1>(one, s_red, tid, sync);
                        if (tid == 0)
                            s_cval[c] = one[0];
                        lacc[c] = 0.0;
                    }
                    sync();
                    if (tid == 0) {
                        double tot[K];
#pragma unroll
                        for (int c = 0; c < K; ++c)
                            tot[c] = s_cval[c];
                        op.emit(r0, tot, part, s_scal, rv);
                    }
                }
            } else {
                // row ends relative to the tile's first entry: rend(x) = end of row x
                const int32_t *rpp = s_rp + (r0 - sr.ab);
                const int32_t kb32 = (int32_t)kb;
                // 1. products: every operand load of this thread in flight at once
                constexpr int GU = (D * K + TC - 1) / TC;
                double ov[GU];
#pragma unroll
                for (int u = 0; u < GU; ++u) {
                    const int f = tid + u * TC;
                    const int e = f / K;
                    ov[u] = f < nk * K ? (double)op.operand(cc[e], f - e * K, s_scal) : 0.0;
                }
#pragma unroll
                for (int u = 0; u < GU; ++u) {
                    const int f = tid + u * TC;
                    if (f < nk * K)
                        s_prod[f] = (double)vv[f / K] * ov[u];
                }
                sync();
                // 2. merge-path split: largest x (rows finished) with rend(x-1) <= d0 - x
                const int items = nr + nk;
                const int d0 = min(tid * IPT, items);
                const int d1 = min(d0 + IPT, items);
                int lo = max(0, d0 - nk), hi = min(d0, nr);
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (rpp[mid] - kb32 <= d0 - mid)
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
                    if (k < rpp[r + 1] - kb32) {
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
                            op.emit(r0 + r, acc, part, s_scal, rv);
                        }
#pragma unroll
                        for (int c = 0; c < K; ++c)
                            acc[c] = 0.0;
                        ++r;
                    }
                }
                // 3. rows spanning threads
                s_crow[tid] = (r < nr) ? r : -1;
#pragma unroll
                for (int c = 0; c < K; ++c)
                    s_cval[tid * K + c] = acc[c];
                sync();
                if (frow >= 0) {
                    for (int u = tid - 1; u >= 0 && s_crow[u] == frow; --u) {
#pragma unroll
                        for (int c = 0; c < K; ++c)
                            facc[c] += s_cval[u * K + c];
                    }
                    op.emit(r0 + frow, facc, part, s_scal, rv);
                }
            }
            // release the stage: order this block's generic accesses before the next fill
            fence_proxy_async_smem();
            sync();
            if (tid == 0)
                mbar_arrive(&empty_bar[stage]);
            if (++stage == NST) {
                stage = 0;
                phase ^= 1u;
            }
        } while (!(flags & HDR_LAST));
    }

    if constexpr (NPK > 0)
        grid_reduce_finalize<TC, NPK>(part, partials, st, op, s_red, &s_flag, s_sum, tid, sync);
}

}  // namespace sla
