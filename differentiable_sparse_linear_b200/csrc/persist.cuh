// Persistent PCG solver kernel for short-row systems: the whole solve (initial pass and
// every iteration) in ONE cooperative launch, with all blocks resident.
//
// The kernels of the graph-driven solve (Q, U_S, Z with SPAI; Q, U_J with Jacobi or no
// preconditioner) become phases of one kernel.  The matrices are read in their sliced ELL
// copies (sell.cuh) with coalesced loads; operands are gathered through L1/L2.  Between two
// phases every block publishes its dot-product partial (fixed-order block sum) and arrives
// on a grid barrier (one 64-bit counter that only grows, so it needs no reset between
// phases); after it every block sums all blocks' partials in block order -- the same
// operations in the same order in every block, so every block derives bit-identical scalars
// (alpha, the stopping test, beta) without a last-block ticket or a round trip through
// global state.  Block 0 writes the final state back for the host.
//
// Memory ordering across the barrier: block barrier, then thread 0 arrives with a release
// reduction on the counter and spins on it with acquire loads, then releases its block with
// another block barrier (causality is transitive through the block barriers).
//
// The grid barrier's wait is bounded in time: a wait that runs out sets the solve's error
// word and a block-wide abort flag, and the block stops at that phase end.
#pragma once

#include "pcg_ops.cuh"
#include "sell.cuh"
#include "tile_engine.cuh"

namespace sla {

enum PhaseKind { PH_Q = 0, PH_US = 1, PH_Z = 2, PH_UJ = 3 };

template <typename VM, typename VV>
struct PersistArgs {
    SellView<VM> A, G, GT;            // G and GT: SPAI only
    VV *x, *ra, *rb, *pa, *pb, *q, *z, *y;
    const VV *dinv;                   // Jacobi (or ones without a preconditioner)
    PcgState *st;
    double *partials;                 // 4 slots of [grid][2K]
    int spai;                         // 1: Q, U_S, Z phases; 0: Q, U_J phases
    int *err;
};

__device__ __forceinline__ unsigned long long ld_acquire_gpu(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

template <typename VM, typename VV, int K, int MAXL>
struct Persist {
    // threads per block: one 1024-thread block per SM for one right-hand side (half the grid
    // barrier's arrivals of two 512-thread blocks: 35.7 against 37.7 us per SPAI iteration on
    // the 1024^2 problem), 512 for more (their lanes need more than 64 registers)
    static constexpr int TB = K == 1 ? 1024 : 512;
    static constexpr int NR = 2 * K;
    // blocks per SM the register budget is cut for
    static constexpr int MINB = 1;
    // slices per warp round (their loads in flight together): two where that fits the registers
    static constexpr int RS = (K == 1 || (K == 2 && sizeof(VV) == 4)) ? 2 : 1;
    // wide rows (K >= 4 right-hand sides): p_new is formed in a phase of its own, so Q
    // gathers one K-row per stored entry instead of two (the extra grid barrier costs far
    // less than the gathers it saves)
    static constexpr bool FORM_P = K >= 4;
    using OQ = OpQ<VV, K>;
    using OQM = OpQm<VV, K>;
    using OUS = OpUS<VV, K>;
    using OZ = OpZ<VV, K>;

    // Operations of one iteration; `odd` selects the double-buffered slots (the initial
    // pass uses the odd slots of U_S and Z, and of U_J).
    static __device__ __forceinline__ OQ opQ(const PersistArgs<VM, VV> &a, bool odd, PcgState *s)
    {
        return OQ{a.z, odd ? a.pb : a.pa, odd ? a.pa : a.pb, a.q, s};
    }
    static __device__ __forceinline__ OQM opQm(const PersistArgs<VM, VV> &a, bool odd, PcgState *s)
    {
        return OQM{odd ? a.pa : a.pb, a.q, s};
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

template <typename VM, typename VV, int K, int MAXL>
__global__ void __launch_bounds__(Persist<VM, VV, K, MAXL>::TB, (Persist<VM, VV, K, MAXL>::MINB))
k_pcg_persistent(const PersistArgs<VM, VV> a)
{
    using P = Persist<VM, VV, K, MAXL>;
    constexpr int TB = P::TB;
    constexpr int NR = P::NR;

    __shared__ double s_red[(TB / 32) * NR];
    __shared__ double s_scal[2 * K + 1];
    __shared__ double s_eps[1];
    __shared__ double s_sum[2 * NR];
    __shared__ PcgState s_st;
    __shared__ int s_abort, s_quit;

    const int tid = threadIdx.x;
    if (tid == 0) {
        s_st = *a.st;
        s_st.has_cond = 0;
        s_st.profile = 0;
        s_abort = 0;
        s_quit = s_st.all_done;
    }
    __syncthreads();
    if (s_quit) {
        if (blockIdx.x == 0 && tid == 0)
            a.st->persistent = 1;
        return;
    }
    volatile int *abort = &s_abort;
    const int lane = tid & 31, warp = tid >> 5;
    int seq = 1;
    unsigned long long t_phase = 0;
    if (blockIdx.x == 0 && tid == 0)
        t_phase = global_ns();
    // scalars of the operations, staged by thread 0 at the end of the phase before:
    // s_scal = {alpha, active} for U_S / U_J, {beta} for Q; Z's eps is constant
    auto stage_update = [&]() {
        for (int c = 0; c < K; ++c) {
            s_scal[c] = s_st.alpha[c];
            s_scal[K + c] = s_st.active[c] ? 1.0 : 0.0;
        }
    };
    auto stage_q = [&]() {
        for (int c = 0; c < K; ++c)
            s_scal[c] = s_st.beta[c];
    };
    if (tid == 0) {
        s_eps[0] = s_st.eps;
        stage_update();
    }
    __syncthreads();

    // End of a phase, first half: warp sums, then thread 0 adds the warps' sums in a fixed
    // order, publishes the block's partial in this phase's slot (4 slots in turn: a slot is
    // written again only after a barrier every reader of it has passed) and passes the
    // grid barrier; the block waits for it.  Returns the slot.
    auto publish = [&](double (&part)[NR], int n, int kind) -> double * {
        double *slot = a.partials + (size_t)(seq & 3) * gridDim.x * NR;
#pragma unroll
        for (int i = 0; i < NR; ++i) {
            double v = part[i];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                v += __shfl_down_sync(0xffffffffu, v, off);
            if (lane == 0)
                s_red[warp * NR + i] = v;
        }
        __syncthreads();
        if (tid == 0) {
            for (int i = 0; i < n; ++i) {
                double t = 0.0;
                for (int w = 0; w < TB / 32; ++w)
                    t += s_red[w * NR + i];
                slot[(size_t)blockIdx.x * NR + i] = t;
            }   // n == 0: a plain grid barrier
            unsigned long long *bar = &a.st->gbar;
            const unsigned long long target = (unsigned long long)seq * gridDim.x;
            // release: the block's writes (ordered before this thread by the block barrier)
            // are visible to every block that acquires the count
            asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(bar) : "memory");
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
            if (blockIdx.x == 0 && kind >= 0) {   // kind < 0: timed with the next phase
                const unsigned long long t1 = global_ns();
                s_st.phase_ns[kind] += t1 - t_phase;
                s_st.phase_cnt[kind] += 1;
                t_phase = t1;
            }
        }
        __syncthreads();
        ++seq;
        return slot;
    };
    // Second half, warp 0 only: all blocks' partials of up to two slots, in block order (lane
    // l takes blocks l, l + 32, ...; then a fixed shuffle tree), into out[0..n) and
    // out[n..2n); the same arithmetic in every block.
    auto reduce_w0 = [&](const double *slot0, const double *slot1, int n, double *out) {
        double v[NR], w[NR];
#pragma unroll
        for (int i = 0; i < NR; ++i) {
            v[i] = 0.0;
            w[i] = 0.0;
        }
        for (int b = lane; b < (int)gridDim.x; b += 32) {
#pragma unroll
            for (int i = 0; i < NR; ++i)
                if (i < n) {
                    v[i] += __ldcg(&slot0[(size_t)b * NR + i]);
                    if (slot1)
                        w[i] += __ldcg(&slot1[(size_t)b * NR + i]);
                }
        }
#pragma unroll
        for (int i = 0; i < NR; ++i) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                v[i] += __shfl_down_sync(0xffffffffu, v[i], off);
                w[i] += __shfl_down_sync(0xffffffffu, w[i], off);
            }
        }
        if (lane == 0)
            for (int i = 0; i < n; ++i) {
                out[i] = v[i];
                if (slot1)
                    out[n + i] = w[i];
            }
        __syncwarp();
    };
    // thread 0, after finalising: stop when every column is done or a wait ran out
    auto quit_now = [&]() { return s_st.all_done || *abort || *(volatile int *)a.err; };

    double part[NR];
    auto zero = [&]() {
#pragma unroll
        for (int i = 0; i < NR; ++i)
            part[i] = 0.0;
    };

    // U_J over this block's rows: x += alpha p, r -= alpha q, z = D^-1 r; partials r.r
    // (0..K-1) and r.z (K..2K-1).  The block takes the rows of its run of slices.
    auto run_uj = [&](const VV *p) -> bool {
        zero();
        const int64_t r0 = a.A.n_slices * blockIdx.x / gridDim.x * 32;
        const int64_t r1 = min(a.A.n, a.A.n_slices * (blockIdx.x + 1) / gridDim.x * 32);
        for (int64_t i = r0 + tid; i < r1; i += TB)
            jacobi_row<VV, K>(i, a.x, a.ra, p, a.q, a.z, a.dinv, s_scal, s_scal + K, part);
        const double *sl = publish(part, 2 * K, PH_UJ);
        if (warp == 0) {
            reduce_w0(sl, nullptr, 2 * K, s_sum);
            if (lane == 0) {
                finalize_residual(&s_st, s_sum);
                finalize_beta(&s_st, s_sum + K);
                stage_q();
                s_quit = quit_now();
            }
        }
        __syncthreads();
        return s_quit != 0;
    };
    auto run_q = [&](bool odd) -> bool {
        zero();
        if constexpr (P::FORM_P) {
            // p_new = z + beta p_old over this block's rows, then a grid barrier
            VV *pn = odd ? a.pa : a.pb;
            const VV *po = odd ? a.pb : a.pa;
            const int64_t r0 = a.A.n_slices * blockIdx.x / gridDim.x * 32;
            const int64_t r1 = min(a.A.n, a.A.n_slices * (blockIdx.x + 1) / gridDim.x * 32);
            using IO = RowIO<VV, K>;
            for (int64_t i = r0 + tid; i < r1; i += TB) {
                VV zz[K], pp[K], o[K];
                IO::load(a.z + i * K, zz);
                IO::load(po + i * K, pp);
#pragma unroll
                for (int c = 0; c < K; ++c)
                    o[c] = vfma<VV>(s_scal[c], pp[c], zz[c]);
                IO::store(pn + i * K, o);
            }
            publish(part, 0, -1);
            sell_phase<K, VM, MAXL, TB, P::RS>(a.A, P::opQm(a, odd, &s_st), part, s_scal);
        } else {
            sell_phase<K, VM, MAXL, TB, P::RS>(a.A, P::opQ(a, odd, &s_st), part, s_scal);
        }
        const double *sl = publish(part, K, PH_Q);
        if (warp == 0) {
            reduce_w0(sl, nullptr, K, s_sum);
            if (lane == 0) {
                finalize_alpha(&s_st, s_sum);
                stage_update();
                s_quit = quit_now();
            }
        }
        __syncthreads();
        return s_quit != 0;
    };
    // U_S then Z.  Z needs U_S's vectors (the barrier) but not its scalar, so U_S's
    // partials are reduced together with Z's at Z's end; U_S's residual test then decides
    // as before (a stop there leaves Z's results unused: x, r and the counts are U_S's).
    auto run_us_z = [&](bool odd) -> bool {
        zero();
        sell_phase<K, VM, MAXL, TB, P::RS>(a.GT, P::opUS(a, odd, &s_st), part, s_scal);
        const double *slot_us = publish(part, K, PH_US);
        zero();
        sell_phase<K, VM, MAXL, TB, P::RS>(a.G, P::opZ(a, odd, &s_st), part, s_eps);
        const double *slot_z = publish(part, K, PH_Z);
        if (warp == 0) {
            reduce_w0(slot_us, slot_z, K, s_sum);
            if (lane == 0) {
                finalize_residual(&s_st, s_sum);
                signal_if_done(&s_st);
                if (!s_st.all_done)
                    finalize_beta(&s_st, s_sum + K);
                stage_q();
                s_quit = quit_now();
            }
        }
        __syncthreads();
        return s_quit != 0;
    };

    bool quit;
    if (a.spai)
        quit = run_us_z(true);
    else
        quit = run_uj(a.pa);
    for (int it = 0; !quit; ++it) {
        const bool odd = it & 1;
        if (run_q(odd))
            break;
        if (a.spai)
            quit = run_us_z(odd);
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
