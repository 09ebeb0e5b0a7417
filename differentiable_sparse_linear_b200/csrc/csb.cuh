// Column-sorted row segments: the SpMV engine for matrices whose rows gather their operands
// from scattered columns (a random graph's neighbours, the power-law system).
//
// In CSR order every stored entry gathers one operand from a random column, so each entry
// costs its own L2 request; measured on B200, a random 4-byte gather stream tops out near
// 270 G gathers/s, a third of what the matrix stream alone would allow.  Here the rows are
// cut into segments of consecutive rows (CSB_RMAX, or CSB_RMAX_F32 for fp32 values), and
// each segment's entries are stored in COLUMN order: the 32 lanes of a warp then gather from
// a few hundred neighbouring columns instead of 32 random ones, so one L2 request serves
// several entries.  The row sums are accumulated in shared memory (atomic adds into the
// segment's row slots, see "Row sums" below), and the fused row epilogue of the operation
// runs once the segment's entries are done.
//
// Storage (CsbPart): per segment its first row and first chunk; entries in chunks of 32
// (one warp load), per chunk the smallest column `base`, per entry a 32-bit word
// (column - base) << 16 | local row, padding marked by a flag bit (csb_pad_word), and the
// entry's value, gathered from the caller's CSR values by `perm` at the start of every
// solve (the values may change between solves; the pattern may not).  8 bytes per entry
// plus 4 per 32 entries, as CSR's value + column index.
//
// Row sums.  With fp32 values and vectors every product a_ij v_j is rounded to an integer
// on a per-segment fixed-point scale and the row sums are exact integer sums, kept as three
// 32-bit words per row: the integer's low lb bits, its next lb bits, and the signed rest,
// each added with a native 32-bit shared-memory atomic (fp64 shared atomics, a
// compare-and-swap loop on 8-byte slots that meet more bank conflicts, made the products
// over half again as slow on B200).  The scale 2^sc is chosen so that bound = (largest sum
// of |a_ij| over a row of the segment) x max_j |v_j| maps below 2^EB, EB = min(62, 2 lb +
// 30): every term fits an int64 (one fp64-to-integer conversion per entry) and no word's sum
// can overflow (lb is set from the longest row, so that row's lower words cannot carry out
// of 32 bits).  Each term is rounded once, to 2^-(EB+1) of the bound (about 1e-19 of it):
// rows far below their segment's bound keep about as many digits as fp64 sums give them.
// The result is the same whatever the order of the adds, so these products are
// bit-reproducible.  max |v_j| comes from k_vec_absmax launched right before (one partial
// per block); when it or the bound is not finite the segment falls back to fp64 atomic adds
// (as fp64-vector products always do), so a NaN or Inf still reaches the result.
#pragma once

#include <cuda_runtime.h>

#include <type_traits>

#include "sla_internal.cuh"
#include "pcg_ops.cuh"
#include "tile_engine.cuh"

namespace sla {

constexpr int CSB_RMAX = 16384;                // rows per segment with fp64 sums (8 bytes a row)
static_assert(CSB_RMAX <= 16384, "local rows must fit 14 bits (the pad flag is bit 15)");
// rows per segment with fp32 values (three 4-byte fixed-point words a row): 128 KB of sums
// leave the other half of the SM's 256 KB of L1/shared memory to cache the gathered
// operand lines (with 16384 rows, 192 KB of sums left 60 KB of L1 and the products ran 7 %
// slower on the power-law 4M system despite the denser segments)
constexpr int CSB_RMAX_F32 = 10922;
constexpr int CSB_WORDS = 3;
// A padding slot (past a chunk's last entry) has value 0, column offset 0, local row = its
// lane in a segment of at least 32 rows (else row 0), and the flag CSB_PADF: it gathers a
// valid operand and, with the fixed-point sums (finite operands only), adds 0 to a row of
// its own bank without a test; the fp64 sums skip it by the flag (0 x Inf would be NaN).
// Local rows are below 2^14 (CSB_RMAX), so the flag bit is free.
constexpr uint32_t CSB_PADF = 0x8000u;
constexpr uint32_t CSB_ROWM = 0x3FFFu;
__host__ __device__ inline uint32_t csb_pad_word(int lane, int seg_rows)
{
    return (seg_rows >= 32 ? (uint32_t)lane : 0u) | CSB_PADF;
}

template <typename VM>
struct CsbView {
    const int32_t *seg_row0;                   // n_seg + 1
    const int32_t *seg_ch0;                    // n_seg + 1
    const int32_t *cbase;                      // per chunk
    const uint32_t *pk;                        // per entry slot
    const VM *val;                             // per entry slot
    int n_seg;
    int rmax;                                  // rows of the largest segment
    const double *seg_bound;                   // per segment: max over rows of sum |a_ij|
    const float *vmax;                         // per-block max |v_j| of the operand, or null
    int vmax_n;
    int lb;                                    // bits of the fixed-point low word
};

constexpr int CSB_VMAX_T = 1024;               // threads of k_vec_absmax

// Per-block max |v_i| over v[0, n) into out[blockIdx.x]; +Inf if the block saw a value that
// is not finite.  16-byte loads where v is 16-byte aligned, four in flight per thread.
template <typename V>
__global__ void __launch_bounds__(CSB_VMAX_T) k_vec_absmax(int64_t n, const V *v, float *out, const PcgState *st)
{
    __shared__ float s_m[CSB_VMAX_T / 32];
    if (st && *(volatile const int *)&st->all_done)
        return;
    float m = 0.f;
    bool bad = false;
    auto take = [&](V x) {
        const float a = fabsf((float)x);
        bad |= !(a <= 3.0e38f);
        m = fmaxf(m, a);
    };
    const int64_t tid = (int64_t)blockIdx.x * CSB_VMAX_T + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * CSB_VMAX_T;
    constexpr int VW = 16 / sizeof(V);             // values per 16-byte load
    int64_t done = 0;
    if (((uintptr_t)v & 15) == 0) {
        using L = typename std::conditional<sizeof(V) == 4, float4, double2>::type;
        const L *v4 = reinterpret_cast<const L *>(v);
        const int64_t n4 = n / VW;
        constexpr int IL = 4;
        for (int64_t i = tid; i < n4; i += stride * IL) {
            L t[IL];
#pragma unroll
            for (int k = 0; k < IL; ++k)
                if (i + k * stride < n4)
                    t[k] = __ldg(&v4[i + k * stride]);
#pragma unroll
            for (int k = 0; k < IL; ++k)
                if (i + k * stride < n4) {
                    const V *e = reinterpret_cast<const V *>(&t[k]);
#pragma unroll
                    for (int j = 0; j < VW; ++j)
                        take(e[j]);
                }
        }
        done = n4 * VW;
    }
    for (int64_t i = done + tid; i < n; i += stride)
        take(v[i]);
    if (bad)
        m = __int_as_float(0x7f800000);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0)
        s_m[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int w = 0; w < CSB_VMAX_T / 32; ++w)
            t = fmaxf(t, s_m[w]);
        out[blockIdx.x] = t;
    }
}

// Per segment the largest row sum of |a_ij| (fp64), from the CSR values: a block per
// segment, a warp per row group of four rows summed together (four rows' loads in flight).
constexpr int CSB_BND_T = 1024;
template <typename VM>
__global__ void __launch_bounds__(CSB_BND_T) k_csb_bounds(int n_seg, const int32_t *seg_row0, const int32_t *rp,
                                                          const VM *val, double *bound)
{
    constexpr int NW = CSB_BND_T / 32, RU = 4;
    __shared__ double s_w[NW];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int sg = blockIdx.x; sg < n_seg; sg += gridDim.x) {
        const int r0 = seg_row0[sg], r1 = seg_row0[sg + 1];
        double wm = 0.0;
        for (int rb = r0 + warp * RU; rb < r1; rb += NW * RU) {
            int k[RU], k1[RU];
            double a[RU];
#pragma unroll
            for (int u = 0; u < RU; ++u) {
                const int r = rb + u;
                k[u] = r < r1 ? rp[r] + lane : 0;
                k1[u] = r < r1 ? rp[r + 1] : 0;
                a[u] = 0.0;
            }
            bool more = true;
            while (more) {
                more = false;
#pragma unroll
                for (int u = 0; u < RU; ++u)
                    if (k[u] < k1[u]) {
                        a[u] += fabs((double)val[k[u]]);
                        k[u] += 32;
                        more |= k[u] < k1[u];
                    }
            }
#pragma unroll
            for (int u = 0; u < RU; ++u) {
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
                    a[u] += __shfl_xor_sync(0xffffffffu, a[u], off);
                wm = fmax(wm, a[u]);
            }
        }
        if (lane == 0)
            s_w[warp] = wm;
        __syncthreads();
        if (threadIdx.x == 0) {
            double t = 0.0;
            for (int w = 0; w < NW; ++w)
                t = fmax(t, s_w[w]);
            bound[sg] = t;
        }
        __syncthreads();
    }
}

// 4 chunks per warp per round, the next round's loads in flight during this one's adds:
// 2 or 8 measured slower with the fixed-point sums (q = A p on the 4M system: 0.644 and
// 0.657 ms against 0.538).
struct CsbCfg {
    static constexpr int T = 1024;             // threads per block (one block per SM)
    static constexpr int U = 4;                // chunks per warp per round
};

// Shared-memory 32-bit add without a returned value (a native shared-memory atomic).
__device__ __forceinline__ void red_add_u32(uint32_t *p, uint32_t v)
{
    asm volatile("red.shared.add.u32 [%0], %1;" ::"r"((unsigned)__cvta_generic_to_shared(p)), "r"(v) : "memory");
}

// The matrix stream (chunk bases, packed words, values) is read once: loaded without L1
// allocation (ld_stream_*), so L1 keeps the gathered operand lines (q = A p on the
// power-law 4M system: 0.514 against 0.530 ms with L1-allocating loads; an L2 evict-first
// hint on top was slower, 0.579).
// One round's matrix data of a warp: U chunks (or padding past the segment's end).
template <typename VM, int U>
struct CsbRound {
    int base[U];
    uint32_t w[U];
    VM a[U];
    // chunks past the segment's last one read as padding (`pad` = csb_pad_word)
    __device__ __forceinline__ void load(const CsbView<VM> &c, int ch, int ch1, int lane, uint32_t pad)
    {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int cc = ch + u * (CsbCfg::T / 32);
            if (cc < ch1) {
                base[u] = (int)ld_stream_b32(&c.cbase[cc]);
                w[u] = ld_stream_b32(&c.pk[(int64_t)cc * 32 + lane]);
                a[u] = ld_stream_val(&c.val[(int64_t)cc * 32 + lane]);
            } else {
                base[u] = 0;
                w[u] = pad;
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
    __shared__ float s_vm[NW];
    // fixed-point row sums (see the top of this file): fp32 values and vectors only
    constexpr bool FIX = sizeof(VM) == 4 && sizeof(VV) == 4;
    // fixed point: high words s_w[0, R), middle words s_w[R, 2R), low words s_w[2R, 3R) of
    // the segment's R rows (s_y[0, R) of the fp64 path shares the first 2R words)
    uint32_t *s_w = reinterpret_cast<uint32_t *>(s_y);

    if (op.skip())
        return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0)
        op.stage(s_scal);
    float vmax = __int_as_float(0x7f800000);                // +Inf: no usable bound
    if (FIX && c.vmax) {
        float m = 0.f;
        for (int b = tid; b < c.vmax_n; b += T)
            m = fmaxf(m, c.vmax[b]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0)
            s_vm[warp] = m;
        __syncthreads();
        vmax = 0.f;
        for (int w = 0; w < NW; ++w)
            vmax = fmaxf(vmax, s_vm[w]);
    }
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
        // this segment's scale 2^sc (block-uniform), or the fp64 path
        bool fix = false;
        double scale = 1.0, unscale = 1.0;
        if (FIX && c.vmax) {
            const double bound = c.seg_bound[s] * (double)vmax;
            if (bound == 0.0) {
                fix = true;
            } else if (bound <= 1.0e300) {           // finite (and not NaN)
                const int eb = min(62, 2 * c.lb + 30);
                const int sc = min(eb - (ilogb(bound) + 1), 1000);
                scale = ldexp(1.0, sc);
                unscale = ldexp(1.0, -sc);
                fix = true;
            }
        }
        const uint32_t pad = csb_pad_word(lane, R);
        for (int i = tid; i < ((FIX && c.vmax) ? CSB_WORDS * R : 2 * R); i += T)
            s_w[i] = 0u;                               // fixed-point words, or s_y[0, R)
        const uint32_t lmask = (1u << c.lb) - 1u;
        // one round: gather the U chunks' operands, then add their products
        auto round = [&](const CsbRound<VM, U> &cr) {
            VV g[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                g[u] = op.operand((int64_t)cr.base[u] + (cr.w[u] >> 16), 0, s_scal);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t r = cr.w[u] & CSB_ROWM;
                if (FIX && fix) {
                    const long long v = __double2ll_rn((double)cr.a[u] * (double)g[u] * scale);
                    red_add_u32(&s_w[r], (uint32_t)(int32_t)(v >> (2 * c.lb)));
                    red_add_u32(&s_w[R + r], (uint32_t)(v >> c.lb) & lmask);
                    red_add_u32(&s_w[2 * R + r], (uint32_t)v & lmask);
                } else if (!(cr.w[u] & CSB_PADF)) {
                    atomicAdd(&s_y[r], (double)cr.a[u] * (double)g[u]);
                }
            }
        };
        // two round buffers in turn: the next round's loads go out before this round's work
        CsbRound<VM, U> ra, rb;
        ra.load(c, ch, ch1, lane, pad);
        __syncthreads();
        for (; ch < ch1; ch += 2 * U * NW) {
            rb.load(c, ch + U * NW, ch1, lane, pad);
            round(ra);
            if (ch + U * NW >= ch1)
                break;
            ra.load(c, ch + 2 * U * NW, ch1, lane, pad);
            round(rb);
        }
        __syncthreads();
        for (int i = tid; i < R; i += T) {
            double acc[1];
            if (FIX && fix) {
                // |sum| < 2^62 + 2^52: exact in int64, rounded once to fp64
                const long long t = (long long)(int32_t)s_w[i] * (1ll << (2 * c.lb)) +
                                    (long long)s_w[R + i] * (1ll << c.lb) + (long long)s_w[2 * R + i];
                acc[0] = (double)t * unscale;
            } else {
                acc[0] = s_y[i];
            }
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
