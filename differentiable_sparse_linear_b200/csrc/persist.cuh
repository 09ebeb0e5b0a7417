// Persistent PCG solver kernel for short-row systems: the whole solve (initial pass and
// every iteration) in ONE cooperative launch, one or a few blocks per SM.
//
// The kernels of the graph-driven solve (Q, U_S, Z with SPAI; Q, U_J with Jacobi or no
// preconditioner) become phases of one kernel.  Between two phases every block
// publishes its dot-product partial (fixed-order block sum) and arrives on a grid barrier
// (one 64-bit counter that only grows, so it needs no reset between phases); after it,
// every block sums all blocks' partials in block order -- the same operations in the same
// order in every block, so every block derives bit-identical scalars (alpha, the stopping
// test, beta) without a last-block ticket or a round trip through global state.  Block 0
// writes the final state back for the host.
//
// The producer thread of each block runs the stage ring across phases: the matrix arrays
// of the next phase's tiles are constant, so it streams them while the consumers still work
// on the current phase (at most one phase ahead); the operand windows, which hold vectors
// the current phase writes, are copied only after the consumers report that the grid
// barrier has passed (a sequence number in shared memory, the "gate").  Vector writes are
// ordered before other blocks' bulk copies by a generic-to-async proxy fence, a block
// barrier and a release/acquire pair on the grid counter.
//
// Every wait is bounded in time (mbarriers, the grid barrier, the gate): a wait that runs
// out sets the solve's error word and a block-wide abort flag, after which the block stops
// at the next phase end; the producer waits for its copies in flight before it exits.
#pragma once

#include "pcg_ops.cuh"
#include "row_engine.cuh"

namespace sla {

enum PhaseKind { PH_Q = 0, PH_US = 1, PH_Z = 2, PH_UJ = 3 };

template <typename VM, typename VV>
struct PersistArgs {
    MatView<VM> A, G, GT;             // G and GT: SPAI only
    const WinDesc *winA, *winG, *winGT;   // operand windows (null: global gathers)
    VV *x, *ra, *rb, *pa, *pb, *q, *z, *y;
    const VV *dinv;                   // Jacobi (or ones without a preconditioner)
    PcgState *st;
    double *partials;                 // 2 slots of [grid][2K]
    int spai;                         // 1: Q, U_S, Z phases; 0: Q, U_J phases
    int *err;
};

__device__ __forceinline__ unsigned long long ld_acquire_gpu(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Bounded wait until *go >= target; false on a stop, an abort or a time-out.
__device__ __forceinline__ bool wait_go(volatile int *go, volatile int *stop, volatile int *abort,
                                        int target, int *err)
{
    if (*go >= target)
        return true;
    const unsigned long long t0 = global_ns();
    for (unsigned i = 1;; ++i) {
        if (*go >= target)
            break;
        if (*stop || *abort)
            return false;
        __nanosleep(64);
        if ((i & 15u) == 0 && global_ns() - t0 > WAIT_LIMIT_NS) {
            atomicOr(err, 4);
            *abort = 1;
            return false;
        }
    }
    __threadfence_block();
    return !*stop;
}

// Gate of one phase for the producer: window copies wait until the consumers have passed
// the grid barrier that ends the previous phase.
struct SeqGate {
    volatile int *go, *stop, *abort;
    int *err;
    int seq;
    bool open;
    __device__ __forceinline__ bool ready() const { return open; }
    __device__ __forceinline__ bool wait()
    {
        if (open)
            return true;
        if (!wait_go(go, stop, abort, seq, err))
            return false;
        fence_proxy_async_global();
        open = true;
        return true;
    }
};

// Bounded wait for a free stage; false when the consumers have stopped.
__device__ __forceinline__ bool wait_empty(uint64_t *bar, uint32_t parity, volatile int *stop,
                                           volatile int *abort, int *err)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = global_ns();
    for (unsigned i = 1;; ++i) {
        // a short suspension: the stop flag is polled between rounds
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity), "r"(2000u)
            : "memory");
        if (ok)
            return true;
        if (*stop || *abort)
            return false;
        if ((i & 15u) == 0 && global_ns() - t0 > WAIT_LIMIT_NS) {
            atomicOr(err, 2);
            *abort = 1;
            return false;
        }
    }
}

template <typename VM, typename VV, int K, int MAXL>
struct Persist {
    static constexpr int TC = RowTmaCfg<K>::TC;
    static constexpr int NST = RowTmaCfg<K>::NST;
    static constexpr int NR = 2 * K;
    // blocks per SM the register budget is cut for: two where the consumer code is small
    // enough to fit without spills (fp32, one right-hand side, rows of at most 8 entries)
    static constexpr int MINB = (K == 1 && MAXL == 8 && sizeof(VM) == 4 && sizeof(VV) == 4) ? 2 : 1;
    using LMax = RowTmaLayout<K, VM, VV, 2>;
    static constexpr size_t PITCH = LMax::BYTES;     // stage pitch: the widest operation's
    static constexpr size_t SMEM = NST * PITCH;
    using OQ = OpQ<VV, K>;
    using OUS = OpUS<VV, K>;
    using OZ = OpZ<VV, K>;

    // Operations of one iteration; `odd` selects the double-buffered slots (the initial
    // pass uses the odd slots of U_S and Z, and of U_J).
    static __device__ __forceinline__ OQ opQ(const PersistArgs<VM, VV> &a, bool odd, PcgState *s)
    {
        return OQ{a.z, odd ? a.pb : a.pa, odd ? a.pa : a.pb, a.q, s};
    }
    static __device__ __forceinline__ OUS opUS(const PersistArgs<VM, VV> &a, bool odd, PcgState *s)
    {
        VV *rold = odd ? a.ra : a.rb, *rnew = odd ? a.rb : a.ra;
        const VV *p = odd ? a.pa : a.pb;
        return OUS{rold, a.q, p, a.x, rnew, a.x, a.y, s};
    }
    static __device__ __forceinline__ OZ opZ(const PersistArgs<VM, VV> &a, bool odd, PcgState *s)
    {
        return OZ{a.y, odd ? a.rb : a.ra, a.z, s};
    }
};

// Producer side of one matrix phase (sequence number seq): at most one phase ahead of the
// consumers; windows behind the gate.  Returns false once the consumers stop.
template <int K, typename VM, int MAXL, class Op>
__device__ __forceinline__ bool produce_phase(const MatView<VM> &m, const WinDesc *win, const Op &op,
                                              unsigned char *smem, size_t pitch, uint64_t *full,
                                              uint64_t *empty, RingPos &rp, int *last, int seq,
                                              volatile int *go, volatile int *stop, volatile int *abort,
                                              int *err)
{
    using E = RowTma<K, VM, MAXL, Op>;
    constexpr int NST = E::NST;
    if (!wait_go(go, stop, abort, seq - 1, err))
        return false;
    SeqGate gate{go, stop, abort, err, seq, false};
    int2 n0 = make_int2(0, 0), n1 = make_int2(0, 0);
    WinDesc nw;
    nw.nseg = 0;
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
        if (!wait_empty(&empty[rp.stage], rp.phase ^ 1u, stop, abort, err))
            return false;
        const bool ok = E::issue(m, op, d0, d1, wd, smem + (size_t)rp.stage * pitch, &full[rp.stage], gate);
        last[rp.stage] = (int)rp.phase;       // parity of the stage's latest copies
        rp.next<NST>();
        if (!ok)
            return false;
    }
    return true;
}

// Consumer side of one matrix phase.
template <int K, typename VM, int MAXL, class Op, int NR>
__device__ __forceinline__ void consume_phase(const MatView<VM> &m, const Op &op, unsigned char *smem,
                                              size_t pitch, uint64_t *full, uint64_t *empty, RingPos &rp,
                                              double (&part)[NR], const double *s_scal, int tid, int *err,
                                              volatile int *abort)
{
    using E = RowTma<K, VM, MAXL, Op>;
    for (int t = blockIdx.x; t < m.n_tiles; t += gridDim.x) {
        E::consume(m, op, smem + (size_t)rp.stage * pitch, &full[rp.stage], &empty[rp.stage], rp.phase,
                   part, s_scal, tid, err, abort);
        rp.next<E::NST>();
    }
}

template <typename VM, typename VV, int K, int MAXL>
__global__ void __launch_bounds__(RowTmaCfg<K>::TC + 32, (Persist<VM, VV, K, MAXL>::MINB))
k_pcg_persistent(const PersistArgs<VM, VV> a)
{
    using P = Persist<VM, VV, K, MAXL>;
    constexpr int TC = P::TC;
    constexpr int NST = P::NST;
    constexpr int NR = P::NR;
    constexpr size_t PITCH = P::PITCH;

    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ uint64_t full_bar[NST], empty_bar[NST];
    __shared__ double s_red[(TC / 32) * NR];
    __shared__ double s_scal[2 * K + 1];
    __shared__ double s_sum[NR];
    __shared__ PcgState s_st;
    __shared__ int s_go, s_stop, s_abort, s_quit;

    const int tid = threadIdx.x;
    if (tid == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], TC);
        }
        fence_mbar_init();
        s_st = *a.st;
        s_st.has_cond = 0;
        s_st.profile = 0;
        s_go = 1;            // phase 1 reads only what the set-up kernels wrote
        s_stop = 0;
        s_abort = 0;
        s_quit = s_st.all_done;
    }
    __syncthreads();
    volatile int *go = &s_go, *stop = &s_stop, *abort = &s_abort;

    // ---------------------------------------------------------------- producer
    if (tid >= TC) {
        if (tid != TC)
            return;
        if (s_quit)
            return;
        RingPos rp;
        int last[NST];
        for (int s = 0; s < NST; ++s)
            last[s] = -1;
        int seq = 1;
        bool run = true;
        if (a.spai) {
            run = produce_phase<K, VM, MAXL>(a.GT, a.winGT, P::opUS(a, true, &s_st), smem, PITCH, full_bar,
                                             empty_bar, rp, last, seq++, go, stop, abort, a.err) &&
                  produce_phase<K, VM, MAXL>(a.G, a.winG, P::opZ(a, true, &s_st), smem, PITCH, full_bar,
                                             empty_bar, rp, last, seq++, go, stop, abort, a.err);
        } else {
            ++seq;           // U_J: no tiles
        }
        for (int it = 0; run; ++it) {
            const bool odd = it & 1;
            run = produce_phase<K, VM, MAXL>(a.A, a.winA, P::opQ(a, odd, &s_st), smem, PITCH, full_bar,
                                             empty_bar, rp, last, seq++, go, stop, abort, a.err);
            if (!run)
                break;
            if (a.spai) {
                run = produce_phase<K, VM, MAXL>(a.GT, a.winGT, P::opUS(a, odd, &s_st), smem, PITCH,
                                                 full_bar, empty_bar, rp, last, seq++, go, stop, abort,
                                                 a.err) &&
                      produce_phase<K, VM, MAXL>(a.G, a.winG, P::opZ(a, odd, &s_st), smem, PITCH, full_bar,
                                                 empty_bar, rp, last, seq++, go, stop, abort, a.err);
            } else {
                ++seq;
            }
        }
        // the copies of every stage have landed before the block exits
        for (int s = 0; s < NST; ++s)
            if (last[s] >= 0)
                mbar_wait_bounded(&full_bar[s], (uint32_t)last[s], a.err);
        return;
    }

    // ---------------------------------------------------------------- consumers
    if (s_quit) {
        if (blockIdx.x == 0 && tid == 0)
            a.st->persistent = 1;
        return;
    }
    auto sync = [] { consumer_sync(TC); };
    RingPos rp;
    int seq = 1;
    unsigned long long t_phase = 0;
    if (blockIdx.x == 0 && tid == 0)
        t_phase = global_ns();

    // End of a phase: block sum, publish, grid barrier, all blocks' partials in block order
    // into s_sum.  Thread 0 then finalises the scalars on the block's copy of the state.
    auto phase_end = [&](double (&part)[NR], int n, int kind) {
        double *slot = a.partials + (size_t)(seq & 1) * gridDim.x * NR;
        block_sum<TC, NR>(part, s_red, tid, sync);
        if (tid < n)
            slot[(size_t)blockIdx.x * NR + tid] = part[0];
        fence_proxy_async_global();
        __threadfence();
        sync();
        if (tid == 0) {
            unsigned long long *bar = &a.st->gbar;
            const unsigned long long target = (unsigned long long)seq * gridDim.x;
            atomicAdd(bar, 1ull);
            if (ld_acquire_gpu(bar) < target) {
                const unsigned long long t0 = global_ns();
                for (unsigned i = 1; ld_acquire_gpu(bar) < target; ++i) {
                    if ((i & 15u) == 0) {
                        if (*abort)
                            break;
                        if (global_ns() - t0 > WAIT_LIMIT_NS) {
                            atomicOr(a.err, 4);
                            *abort = 1;
                            break;
                        }
                    }
                }
            }
            __threadfence();
            *go = seq + 1;                 // the producer may copy the next phase's windows
            if (blockIdx.x == 0) {
                const unsigned long long t1 = global_ns();
                s_st.phase_ns[kind] += t1 - t_phase;
                s_st.phase_cnt[kind] += 1;
                t_phase = t1;
            }
        }
        sync();
        double v[NR];
#pragma unroll
        for (int i = 0; i < NR; ++i)
            v[i] = 0.0;
        for (int b = tid; b < (int)gridDim.x; b += TC) {
#pragma unroll
            for (int i = 0; i < NR; ++i)
                if (i < n)
                    v[i] += __ldcg(&slot[(size_t)b * NR + i]);
        }
        block_sum<TC, NR>(v, s_red, tid, sync);
        if (tid < n)
            s_sum[tid] = v[0];
        sync();
        ++seq;
    };
    // After thread 0 finalised: stop when every column is done or a wait ran out.
    auto decide = [&]() -> bool {
        if (tid == 0) {
            int q = s_st.all_done || *abort || *(volatile int *)a.err;
            s_quit = q;
            if (q) {
                __threadfence_block();
                *stop = 1;
            }
        }
        sync();
        return s_quit != 0;
    };

    double part[NR];
    auto zero = [&]() {
#pragma unroll
        for (int i = 0; i < NR; ++i)
            part[i] = 0.0;
    };

    // U_J over this block's rows (grid-stride): x += alpha p, r -= alpha q, z = D^-1 r;
    // partials r.r (0..K-1) and r.z (K..2K-1).
    auto run_uj = [&](const VV *p) -> bool {
        if (tid == 0) {
            for (int c = 0; c < K; ++c) {
                s_scal[c] = s_st.alpha[c];
                s_scal[K + c] = s_st.active[c] ? 1.0 : 0.0;
            }
        }
        sync();
        zero();
        const int64_t n = a.A.n;
        const int64_t stride = (int64_t)gridDim.x * TC;
        for (int64_t i = (int64_t)blockIdx.x * TC + tid; i < n; i += stride)
            jacobi_row<VV, K>(i, a.x, a.ra, p, a.q, a.z, a.dinv, s_scal, s_scal + K, part);
        phase_end(part, 2 * K, PH_UJ);
        if (tid == 0) {
            finalize_residual(&s_st, s_sum);
            finalize_beta(&s_st, s_sum + K);
        }
        return decide();
    };
    auto run_q = [&](bool odd) -> bool {
        const auto op = P::opQ(a, odd, &s_st);
        if (tid == 0)
            op.stage(s_scal);
        sync();
        zero();
        consume_phase<K, VM, MAXL>(a.A, op, smem, PITCH, full_bar, empty_bar, rp, part, s_scal, tid, a.err,
                                   abort);
        phase_end(part, K, PH_Q);
        if (tid == 0)
            finalize_alpha(&s_st, s_sum);
        return decide();
    };
    auto run_us = [&](bool odd) -> bool {
        const auto op = P::opUS(a, odd, &s_st);
        if (tid == 0)
            op.stage(s_scal);
        sync();
        zero();
        consume_phase<K, VM, MAXL>(a.GT, op, smem, PITCH, full_bar, empty_bar, rp, part, s_scal, tid,
                                   a.err, abort);
        phase_end(part, K, PH_US);
        if (tid == 0) {
            finalize_residual(&s_st, s_sum);
            signal_if_done(&s_st);
        }
        return decide();
    };
    auto run_z = [&](bool odd) -> bool {
        const auto op = P::opZ(a, odd, &s_st);
        if (tid == 0)
            op.stage(s_scal);
        sync();
        zero();
        consume_phase<K, VM, MAXL>(a.G, op, smem, PITCH, full_bar, empty_bar, rp, part, s_scal, tid, a.err,
                                   abort);
        phase_end(part, K, PH_Z);
        if (tid == 0)
            finalize_beta(&s_st, s_sum);
        return decide();
    };

    bool quit;
    if (a.spai)
        quit = run_us(true) || run_z(true);
    else
        quit = run_uj(a.pa);
    for (int it = 0; !quit; ++it) {
        const bool odd = it & 1;
        if (run_q(odd))
            break;
        if (a.spai)
            quit = run_us(odd) || run_z(odd);
        else
            quit = run_uj(odd ? a.pa : a.pb);
    }

    if (blockIdx.x == 0 && tid == 0) {
        PcgState *g = a.st;
        for (int c = 0; c < KMAX; ++c) {
            g->rho[c] = s_st.rho[c];
            g->alpha[c] = s_st.alpha[c];
            g->beta[c] = s_st.beta[c];
            g->bnorm[c] = s_st.bnorm[c];
            g->relres[c] = s_st.relres[c];
            g->iters[c] = s_st.iters[c];
            g->status[c] = s_st.status[c];
            g->active[c] = s_st.active[c];
        }
        g->all_done = s_st.all_done;
        g->phase0 = s_st.phase0;
        for (int i = 0; i < 4; ++i) {
            g->phase_ns[i] = s_st.phase_ns[i];
            g->phase_cnt[i] = s_st.phase_cnt[i];
        }
        g->persistent = 1;
    }
}

}  // namespace sla
