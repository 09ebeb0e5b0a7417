// Shared pieces of the SpMV engines (sm_100a) and the load-balanced CSR SpMV for matrices
// with long rows.
//
// * PTX helpers for the TMA-fed row engine: mbarriers (every wait bounded in time; a wait
//   that runs out sets an error word and the block carries on to a normal exit, results
//   are then flagged invalid by the host), bulk copies, 16-byte-aligned spans of an array
//   range with plain-load tails, named consumer barriers.
// * Block reductions and the last-block grid reduction: each block writes its fixed-order
//   partial, the last block to finish reduces the partials in block order and runs the
//   operation's scalar finalisation, so results are deterministic for a given device.
// * k_tile2, the load-balanced SpMV with fused row epilogues.  Work unit: a "tile" = a run
//   of whole rows holding at most D items (rows + stored entries) and at most RMAX rows,
//   built once per matrix on the host; a row with D or more entries is a tile of its own
//   ("long row") streamed in chunks of D entries.  Rows never straddle tiles, so every row
//   is finished inside one block.  Per tile every thread loads its strided share of the
//   entries (coalesced) and gathers each operand as soon as its column is in a register,
//   so all of a thread's matrix loads and then all of its gathers are in flight; the
//   products go to shared memory; the tile's items are split evenly over the threads along
//   the merge path of (row ends, entries) -- the merge-based SpMV decomposition -- and
//   each thread sums its run; a row spanning threads is finished by the thread holding its
//   end, which adds the partial sums the earlier threads left, in a fixed order.  Several
//   blocks per SM hide the latency.  Used above 4 right-hand sides.
// * k_rowgroup, the SpMV with fused row epilogues for long-row matrices up to 4 right-hand
//   sides: rows binned by length (GroupPart), a lane group sized to the row owns it and
//   reduces with a fixed shuffle tree.  No shared-memory staging and no block barrier: a
//   stored entry costs its two loads, its gather and one FMA, where the tile kernel also
//   spends a merge-path split and a carry walk on it.
#pragma once

#include <type_traits>

#include "sla_internal.cuh"

namespace sla {

// ------------------------------------------------------------------ configuration
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

// ------------------------------------------------------------------ the load-and-gather tile kernel
// Fixed-size tiles of entries with a merge-path split over their rows and the fused
// epilogues, without a producer warp: every
// thread loads entries tid, tid + T, ... of the tile (coalesced) and gathers each operand
// as soon as its column is in a register, so a thread has all of its matrix loads and then
// all of its gathers in flight; the products go to shared memory for the merge-path sums.
// Own-row vectors are read from global memory by the thread that emits the row.  Several
// blocks per SM hide the latency that the TMA pipeline hid.
template <int K>
struct Tile2Cfg {
    static constexpr int T = 256;                       // threads
    // 1024-item tiles, 8 blocks per SM (K = 1): one block's merge and carry work overlaps the
    // others' gathers (power-law 4M system: 222 -> 288 iterations/s against 2048-item tiles
    // at 5 blocks per SM)
    static constexpr int D = K <= 2 ? 1024 / K : 512 / (K / 2 > 1 ? K / 2 : 1);
    static constexpr int MINB = K == 1 ? 8 : K == 2 ? 4 : 1;   // register budget without spills
    static constexpr int RMAX = D;                      // rows per tile at most
};

// Own-row values read from global memory on use.
template <class Op, int K>
struct GlobalRows {
    Op op;
    __device__ __forceinline__ typename Op::VV get(int v, int64_t i, int c) const
    {
        return op.row_vec(v)[i * K + c];
    }
};

template <int K, typename VM, class Op>
__global__ void __launch_bounds__(Tile2Cfg<K>::T, Tile2Cfg<K>::MINB)
k_tile2(const MatView<VM> m, const Op op, double *partials, PcgState *st)
{
    constexpr int T = Tile2Cfg<K>::T;
    constexpr int D = Tile2Cfg<K>::D;
    constexpr int RMAX = Tile2Cfg<K>::RMAX;
    constexpr int IPT = (2 * D + T - 1) / T;            // items (rows + entries) per thread at most
    constexpr int EPT = (D + T - 1) / T;                // entries per thread
    constexpr int NPK = Op::NP * K;
    constexpr int NR = NPK > K ? NPK : K;
    using VV = typename Op::VV;

    __shared__ double s_prod[D * K];
    __shared__ int32_t s_rp[RMAX + 1];
    __shared__ int32_t s_crow[T];
    __shared__ double s_cval[T * K];
    __shared__ double s_red[(T / 32) * NR];
    __shared__ double s_scal[Op::NS > 0 ? Op::NS : 1];
    __shared__ double s_sum[NR];
    __shared__ int s_flag;

    if (op.skip())
        return;
    const int tid = threadIdx.x;
    if (tid == 0)
        op.stage(s_scal);
    __syncthreads();
    auto sync = [] { __syncthreads(); };
    GlobalRows<Op, K> rv{op};
    double part[NPK > 0 ? NPK : 1];
#pragma unroll
    for (int i = 0; i < (NPK > 0 ? NPK : 1); ++i)
        part[i] = 0.0;

    for (int t = blockIdx.x; t < m.n_tiles; t += gridDim.x) {
        const int2 d0 = m.desc[t], d1 = m.desc[t + 1];
        const int r0 = d0.x, r1 = d1.x;
        const int64_t k0 = (int64_t)(uint32_t)d0.y, k1 = (int64_t)(uint32_t)d1.y;
        const int nr = r1 - r0;
        if ((int64_t)nr + (k1 - k0) > D) {
            // one long row, in chunks of D entries: thread-strided partial sums
            double lacc[K];
#pragma unroll
            for (int c = 0; c < K; ++c)
                lacc[c] = 0.0;
            for (int64_t kb = k0; kb < k1; kb += D) {
                const int nk = (int)min((int64_t)D, k1 - kb);
                double prod[EPT][K];
#pragma unroll
                for (int u = 0; u < EPT; ++u) {
                    const int e = tid + u * T;
                    VV o[K];
                    double a = 0.0;
                    if (e < nk) {
                        a = (double)m.val[kb + e];
                        op.operand_row(m.ci[kb + e], o, s_scal);
                    }
#pragma unroll
                    for (int c = 0; c < K; ++c)
                        prod[u][c] = e < nk ? a * (double)o[c] : 0.0;
                }
#pragma unroll
                for (int u = 0; u < EPT; ++u)
#pragma unroll
                    for (int c = 0; c < K; ++c)
                        lacc[c] += prod[u][c];
            }
#pragma unroll
            for (int c = 0; c < K; ++c) {
                double one[1] = {lacc[c]};
                block_sum<T, 1>(one, s_red, tid, sync);
                if (tid == 0)
                    s_cval[c] = one[0];
            }
            sync();
            if (tid == 0) {
                double tot[K];
#pragma unroll
                for (int c = 0; c < K; ++c)
                    tot[c] = s_cval[c];
                op.emit(r0, tot, part, s_scal, rv);
            }
            sync();
            continue;
        }
        const int nk = (int)(k1 - k0);
        // 1. products (matrix loads, then gathers, all in flight) and row ends
#pragma unroll
        for (int u = 0; u < EPT; ++u) {
            const int e = tid + u * T;
            if (e < nk) {
                const double a = (double)m.val[k0 + e];
                VV o[K];
                op.operand_row(m.ci[k0 + e], o, s_scal);
#pragma unroll
                for (int c = 0; c < K; ++c)
                    s_prod[e * K + c] = a * (double)o[c];
            }
        }
        for (int x = tid; x <= nr; x += T)
            s_rp[x] = (int32_t)((int64_t)m.rp[r0 + x] - k0);
        sync();
        // 2. merge-path split: largest x (rows finished) with rend(x-1) <= d0 - x
        const int items = nr + nk;
        const int ipt = (items + T - 1) / T;
        const int d0i = min(tid * ipt, items);
        const int d1i = min(d0i + ipt, items);
        int lo = max(0, d0i - nk), hi = min(d0i, nr);
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_rp[mid] <= d0i - mid)
                lo = mid;
            else
                hi = mid - 1;
        }
        int r = lo, k = d0i - lo;
        double acc[K], facc[K];
#pragma unroll
        for (int c = 0; c < K; ++c) {
            acc[c] = 0.0;
            facc[c] = 0.0;
        }
        int frow = -1;
        for (int d = d0i; d < d1i; ++d) {
            if (k < s_rp[r + 1]) {
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
        // 3. rows spanning threads: the thread holding a row's end adds the partial sums
        //    the earlier threads left, in a fixed order
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
        sync();
        (void)IPT;
    }

    if constexpr (NPK > 0)
        grid_reduce_finalize<T, NPK>(part, partials, st, op, s_red, &s_flag, s_sum, tid, sync);
}

// ------------------------------------------------------------------ lane-group kernel
// Rows grouped by length (GroupPart): a group of G lanes owns a row, each lane takes the
// row's entries G apart (4 per pass, all of a pass's loads in flight) and the group sums
// its lanes with a fixed xor-shuffle tree.  A warp takes one task (32 / G rows of one bin)
// at a time, the tasks round-robin over the grid's warps; the next task's row list entries
// are loaded while the current one runs.
struct GroupView {
    const int4 *rows;
    int task0[GBINS + 1];
    int pos0[GBINS + 1];
    int n_tasks;
};

// Ops that read caller vectors with a runtime leading dimension (the standalone SpMV) mark
// themselves ANY_LD: their 64-bit operand addressing needs more registers.
template <class Op, class = void>
struct any_ld : std::false_type {};
template <class Op>
struct any_ld<Op, std::void_t<decltype(Op::ANY_LD)>> : std::bool_constant<Op::ANY_LD> {};

template <int K, class Op>
struct GroupCfg {
    static constexpr int T = 256;
    static constexpr int U = 4;                          // entries per lane per pass
    static constexpr int MINB = K == 1 ? (any_ld<Op>::value ? 6 : 8) : K == 2 ? 5 : 4;
};

template <int U, int K, typename VM, class Op>
__device__ __forceinline__ void group_row_sum(const MatView<VM> &m, const Op &op, int k, int k1, int G,
                                              const double *s_scal, double (&acc)[K])
{
    using VV = typename Op::VV;
    for (; k < k1; k += U * G) {
        VM a[U];
        int32_t j[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = k + u * G;
            a[u] = e < k1 ? m.val[e] : (VM)0;
            j[u] = e < k1 ? m.ci[e] : -1;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (j[u] >= 0) {
                VV o[K];
                op.operand_row(j[u], o, s_scal);
#pragma unroll
                for (int c = 0; c < K; ++c)
                    acc[c] = fma((double)a[u], (double)o[c], acc[c]);
            }
        }
    }
}

// This lane's row position in task t (-1: none) and the task's bin.  Static indices only,
// so the bin table stays in the parameter bank.
__device__ __forceinline__ int group_locate(const GroupView &g, int t, int lane, int &bin)
{
    int b = 0, t0 = g.task0[0], p0 = g.pos0[0], p1 = g.pos0[1];
#pragma unroll
    for (int i = 1; i < GBINS; ++i)
        if (t >= g.task0[i]) {
            b = i;
            t0 = g.task0[i];
            p0 = g.pos0[i];
            p1 = g.pos0[i + 1];
        }
    bin = b;
    const int pos = p0 + ((t - t0) << b) + (lane >> (GBINS - 1 - b));
    return pos < p1 ? pos : -1;
}

template <int K, typename VM, class Op>
__global__ void __launch_bounds__(GroupCfg<K, Op>::T, GroupCfg<K, Op>::MINB)
k_rowgroup(const MatView<VM> m, const GroupView g, const Op op, double *partials, PcgState *st)
{
    constexpr int T = GroupCfg<K, Op>::T;
    constexpr int NW = T / 32;
    constexpr int NPK = Op::NP * K;
    constexpr int NR = NPK > K ? NPK : K;

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

    auto locate = [&](int t, int &bin) { return group_locate(g, t, lane, bin); };
    const int nw = gridDim.x * NW;
    int t = blockIdx.x * NW + (tid >> 5);
    int bin = 0, pos = t < g.n_tasks ? locate(t, bin) : -1;
    int4 cur = pos >= 0 ? __ldg(&g.rows[pos]) : make_int4(0, 0, 0, 0);
    for (; t < g.n_tasks; t += nw) {
        const int G = 32 >> bin;
        const bool live = pos >= 0;
        const int4 row = cur;
        // the next task's entries, in flight during this one
        const int tn = t + nw;
        int bin_n = 0, pos_n = tn < g.n_tasks ? locate(tn, bin_n) : -1;
        cur = pos_n >= 0 ? __ldg(&g.rows[pos_n]) : make_int4(0, 0, 0, 0);

        double acc[K];
#pragma unroll
        for (int c = 0; c < K; ++c)
            acc[c] = 0.0;
        const int gl = lane & (G - 1);
        if (live)
            group_row_sum<GroupCfg<K, Op>::U, K>(m, op, row.y + gl, row.z, G, s_scal, acc);
        for (int off = G >> 1; off > 0; off >>= 1)
#pragma unroll
            for (int c = 0; c < K; ++c)
                acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], off);
        if (live && gl == 0)
            op.emit(row.x, acc, part, s_scal, rv);
        bin = bin_n;
        pos = pos_n;
    }

    if constexpr (NPK > 0) {
        auto sync = [] { __syncthreads(); };
        grid_reduce_finalize<T, NPK>(part, partials, st, op, s_red, &s_flag, s_sum, tid, sync);
    }
}

}  // namespace sla
