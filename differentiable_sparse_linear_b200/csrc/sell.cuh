// Sliced SpMV with fused row epilogues for the persistent solver (short-row matrices; the
// storage is described with SellPart).
//
// A warp owns a slice of 32 rows, one row per lane; a slot row of the slice is one
// coalesced 128-byte access of values (64 bytes of 16-bit column offsets in an index
// slice), and a lane's loop over its row's entries is fully unrolled up to MAXL with every
// load independent.  Operands are gathered through L1/L2
// (the vectors were written before the grid barrier that opened this phase); a block owns
// a contiguous run of slices and its warps take consecutive slices, so the lines that hold
// a row's vertical neighbours (a grid line away) were just brought in by the same warp.
// Row sums are fp32 when values and vectors are fp32 (at most MAXL terms), fp64 otherwise.
#pragma once

#include <type_traits>

#include "pcg_ops.cuh"

namespace sla {

template <typename VM>
struct SellView {
    const uint2 *desc;         // per slice: {first slot row << 5 | L, diagonal << 31 | full << 30 | offsets}
    const int32_t *offs;       // offset lists of the diagonal slices
    const uint8_t *lens;       // per row (index slices)
    const int16_t *idx16;      // column - row (rel16), or null
    const int32_t *idx32;      // columns, or null
    const VM *val;
    int64_t n;
    int64_t n_slices;
};

// Own-row vector values of a lane's row.
template <typename VV, int K, int NV>
struct LaneVals {
    VV v[NV > 0 ? NV : 1][K];
    __device__ __forceinline__ VV get(int vi, int64_t, int c) const { return v[vi][c]; }
};

// A slot's value: with 4 or more right-hand sides loaded without L1 allocation (the operand
// rows are wide and L1 is better left to them: the 8-RHS heat solve ran 59.0 against 61.4 us
// per iteration); with fewer, an L1-allocating load (the L2-resident 1024^2 SPAI solve ran
// 36.3 against 47.7 us with no-allocate loads).
template <int K, typename VM>
__device__ __forceinline__ VM sell_val(const VM *q)
{
    if constexpr (K >= 4)
        return ld_stream_val(q);
    else
        return *q;
}

// The slices [s0, s1) of this block, warps round-robin over consecutive slices, RS slices
// per round (their loads all in flight together); `part` takes the epilogue's dot-product
// partials in a fixed order.  In a diagonal slice the operand rows are row + offs[u]
// (shared by the warp), so the operand loads and the value loads go out together; a
// padding slot (value 0) reads a clamped row and adds 0.
template <int K, typename VM, int MAXL, int TB, int RS, class Op, int NR>
__device__ __forceinline__ void sell_phase(const SellView<VM> &m, const Op &op, double (&part)[NR],
                                           const double *s_scal)
{
    using VV = typename Op::VV;
    using Acc = typename std::conditional<sizeof(VM) == 4 && sizeof(VV) == 4, float, double>::type;
    constexpr int NV = Op::NV;
    constexpr int NW = TB / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t s0 = m.n_slices * blockIdx.x / gridDim.x;
    const int64_t s1 = m.n_slices * (blockIdx.x + 1) / gridDim.x;
    const int32_t nlast = (int32_t)m.n - 1;
    // descriptors are loaded one round ahead (L = 0 past the run: nothing to do)
    uint2 dn[RS];
#pragma unroll
    for (int q = 0; q < RS; ++q) {
        const int64_t sl = s0 + warp + (int64_t)q * NW;
        dn[q] = sl < s1 ? m.desc[sl] : make_uint2(0u, 0u);
    }
    for (int64_t sb = s0 + warp; sb < s1; sb += (int64_t)NW * RS) {
        uint2 d[RS];
#pragma unroll
        for (int q = 0; q < RS; ++q) {
            d[q] = dn[q];
            const int64_t sl = sb + (int64_t)(q + RS) * NW;
            dn[q] = sl < s1 ? m.desc[sl] : make_uint2(0u, 0u);
        }
        Acc s[RS][K];
        LaneVals<VV, K, NV> rv[RS];
#pragma unroll
        for (int q = 0; q < RS; ++q) {
            const int64_t sl = sb + (int64_t)q * NW;
            const int32_t row = (int32_t)(sl * 32 + lane);
            const bool live = sl < s1 && row < m.n;
            const int L = (int)(d[q].x & 31u);
            const int64_t e0 = (int64_t)(d[q].x >> 5) * 32 + lane;
#pragma unroll
            for (int v = 0; v < NV; ++v) {
                if (live) {
                    op.load_rv(v, row, rv[q].v[v]);
                } else {
#pragma unroll
                    for (int c = 0; c < K; ++c)
                        rv[q].v[v][c] = (VV)0;
                }
            }
#pragma unroll
            for (int c = 0; c < K; ++c)
                s[q][c] = (Acc)0;
            if (d[q].y >> 31) {
                const int32_t *of = m.offs + (d[q].y & 0x3fffffffu);
#pragma unroll
                for (int u = 0; u < MAXL; ++u) {
                    if (u < L) {
                        const int32_t j = min(max(row + of[u], 0), nlast);
                        const Acc av = (Acc)sell_val<K>(&m.val[e0 + u * 32]);
                        VV o[K];
                        op.operand_row(j, o, s_scal);
#pragma unroll
                        for (int c = 0; c < K; ++c)
                            s[q][c] = fma(av, (Acc)o[c], s[q][c]);
                    }
                }
            } else {
                const int len = sl < s1 ? m.lens[row] : 0;   // 0 past the last row
#pragma unroll
                for (int u = 0; u < MAXL; ++u) {
                    if (u < len) {
                        const int32_t j =
                            m.idx16 ? row + (int32_t)m.idx16[e0 + u * 32] : m.idx32[e0 + u * 32];
                        const Acc av = (Acc)sell_val<K>(&m.val[e0 + u * 32]);
                        VV o[K];
                        op.operand_row(j, o, s_scal);
#pragma unroll
                        for (int c = 0; c < K; ++c)
                            s[q][c] = fma(av, (Acc)o[c], s[q][c]);
                    }
                }
            }
        }
#pragma unroll
        for (int q = 0; q < RS; ++q) {
            const int64_t sl = sb + (int64_t)q * NW;
            const int32_t row = (int32_t)(sl * 32 + lane);
            if (sl < s1 && row < m.n) {
                double acc[K];
#pragma unroll
                for (int c = 0; c < K; ++c)
                    acc[c] = (double)s[q][c];
                op.emit(row, acc, part, s_scal, rv[q]);
            }
        }
    }
}

// y = A x straight from the caller's CSR arrays (K right-hand sides with leading dimension
// ld, columns c >= nc zero), using the slice descriptors only for the pattern: in a full
// diagonal slice entry u of row r is CSR entry row_ptr[r] + u and its column is
// r + offs[u], so the column indices are not read at all; other slices read them.  A warp
// owns a slice (lane = row), a block a contiguous run of slices; two slices per round.
constexpr int SPS_T = 256;

template <typename V, int K, int MAXL>
__global__ void __launch_bounds__(SPS_T)
k_spmv_slices(int64_t n, int64_t n_slices, const uint2 *__restrict__ desc, const int32_t *__restrict__ offs,
              const int32_t *__restrict__ rp, const int32_t *__restrict__ ci, const V *__restrict__ val,
              const V *__restrict__ x, V *__restrict__ y, int ld, int nc)
{
    constexpr int NW = SPS_T / 32, RS = 2;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t s0 = n_slices * blockIdx.x / gridDim.x;
    const int64_t s1 = n_slices * (blockIdx.x + 1) / gridDim.x;
    for (int64_t sb = s0 + warp; sb < s1; sb += (int64_t)NW * RS) {
        double acc[RS][K];
#pragma unroll
        for (int q = 0; q < RS; ++q) {
            const int64_t sl = sb + (int64_t)q * NW;
            const int64_t row = sl * 32 + lane;
            const bool live = sl < s1 && row < n;
            const uint2 d = sl < s1 ? desc[sl] : make_uint2(0u, 0u);
            const int L = (int)(d.x & 31u);
            const int32_t k0 = live ? rp[row] : 0;
#pragma unroll
            for (int c = 0; c < K; ++c)
                acc[q][c] = 0.0;
            if ((d.y >> 30) == 3u) {
                const int32_t *of = offs + (d.y & 0x3fffffffu);
#pragma unroll
                for (int u = 0; u < MAXL; ++u)
                    if (live && u < L) {
                        const int64_t j = row + of[u];
                        const double a = (double)val[k0 + u];
#pragma unroll
                        for (int c = 0; c < K; ++c)
                            if (c < nc)
                                acc[q][c] = fma(a, (double)__ldg(&x[j * ld + c]), acc[q][c]);
                    }
            } else {
                const int len = live ? rp[row + 1] - k0 : 0;
#pragma unroll
                for (int u = 0; u < MAXL; ++u)
                    if (u < len) {
                        const int64_t j = ci[k0 + u];
                        const double a = (double)val[k0 + u];
#pragma unroll
                        for (int c = 0; c < K; ++c)
                            if (c < nc)
                                acc[q][c] = fma(a, (double)__ldg(&x[j * ld + c]), acc[q][c]);
                    }
            }
        }
#pragma unroll
        for (int q = 0; q < RS; ++q) {
            const int64_t sl = sb + (int64_t)q * NW;
            const int64_t row = sl * 32 + lane;
            if (sl < s1 && row < n)
#pragma unroll
                for (int c = 0; c < K; ++c)
                    if (c < nc)
                        y[row * ld + c] = (V)acc[q][c];
        }
    }
}

// y = A x from the sliced copy of a short-row matrix whose values are declared static
// (SLA_STATIC_VALUES; the copy is refreshed when the caller reports a change): every slot row
// of a slice is one coalesced 128-byte access of values, diagonal slices read no column
// indices, and [n][K] operands move as whole rows.  The persistent solver's phase code, with
// the plain product as its row epilogue.
template <typename V, int K, int MAXL>
__global__ void __launch_bounds__(SPS_T)
k_spmv_sell(const SellView<V> m, const OpSpmv<V, K> op)
{
    double part[1] = {0.0};
    sell_phase<K, V, MAXL, SPS_T, (K <= 2 ? 2 : 1)>(m, op, part, nullptr);
}

}  // namespace sla
