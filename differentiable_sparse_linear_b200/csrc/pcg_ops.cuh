// Scalar finalisation of the PCG recurrence and the fused operations (row epilogues) the
// SpMV engines run: Q (p update, q = A p, p.q), U_S (x/r update, y = G^T r, r.r), Z
// (z = G y + eps r, r.z) and the plain SpMV.
#pragma once

#include <cuda_runtime.h>

#include <cmath>
#include <cstring>

#include "sla_internal.cuh"

namespace sla {

// ------------------------------------------------------------------ scalar finalisation
static __device__ __forceinline__ bool finite_d(double a) { return isfinite(a); }

static __device__ __noinline__ void signal_if_done(PcgState *st)
{
    int any = 0;
    for (int c = 0; c < st->k; ++c)
        any |= st->active[c];
    if (!any) {
        st->all_done = 1;
        if (st->has_cond)
            cudaGraphSetConditional((cudaGraphConditionalHandle)st->cond_handle, 0u);
    }
}

// After q = A p: alpha = rho / (p.q); p.q <= 0 or non-finite is a breakdown.
static __device__ __noinline__ void finalize_alpha(PcgState *st, const double *pq)
{
    if (st->profile)
        return;
    for (int c = 0; c < st->k; ++c) {
        if (!st->active[c])
            continue;
        const double d = pq[c];
        if (!(d > 0.0) || !finite_d(d)) {
            st->status[c] = SLA_BREAKDOWN;
            st->active[c] = 0;
        } else {
            st->alpha[c] = st->rho[c] / d;
        }
    }
    signal_if_done(st);
}

// After the x/r update: stopping test on ||r||/||b|| (initial pass: record ||b||).
static __device__ __noinline__ void finalize_residual(PcgState *st, const double *rr)
{
    if (st->profile)
        return;
    for (int c = 0; c < st->k; ++c) {
        if (!st->active[c])
            continue;
        if (st->phase0) {
            const double bn = sqrt(rr[c]);
            st->bnorm[c] = bn;
            st->relres[c] = bn > 0.0 ? 1.0 : 0.0;
            if (!finite_d(bn)) {
                st->status[c] = SLA_BREAKDOWN;
                st->active[c] = 0;
            } else if (bn == 0.0) {
                st->status[c] = SLA_SUCCESS;
                st->active[c] = 0;
            }
        } else {
            st->iters[c] += 1;
            const double rel = sqrt(rr[c]) / st->bnorm[c];
            st->relres[c] = rel;
            if (!finite_d(rel)) {
                st->status[c] = SLA_BREAKDOWN;
                st->active[c] = 0;
            } else if (rel <= st->tol) {
                st->status[c] = SLA_SUCCESS;
                st->active[c] = 0;
            } else if (st->iters[c] >= st->maxit) {
                st->status[c] = SLA_NOT_CONVERGED;
                st->active[c] = 0;
            }
        }
    }
}

// After z = M^-1 r: rho' = r.z, beta = rho'/rho (0 on the initial pass).
static __device__ __noinline__ void finalize_beta(PcgState *st, const double *rz)
{
    if (st->profile)
        return;
    for (int c = 0; c < st->k; ++c) {
        if (!st->active[c])
            continue;
        const double v = rz[c];
        if (!(v > 0.0) || !finite_d(v)) {
            st->status[c] = SLA_BREAKDOWN;
            st->active[c] = 0;
            continue;
        }
        st->beta[c] = st->phase0 ? 0.0 : v / st->rho[c];
        st->rho[c] = v;
    }
    st->phase0 = 0;
    signal_if_done(st);
}

// ------------------------------------------------------------------ operations
// a*b + c for vector elements: in fp32 (a rounded once) for fp32 vectors, fp64 otherwise.
// Every place that forms the same vector value uses it with the same operands, so values
// recomputed from gathered operands equal the stored ones bit for bit.
template <typename V>
__device__ __forceinline__ V vfma(double a, V b, V c);
template <>
__device__ __forceinline__ float vfma<float>(double a, float b, float c)
{
    return __fmaf_rn((float)a, b, c);
}
template <>
__device__ __forceinline__ double vfma<double>(double a, double b, double c)
{
    return __fma_rn(a, b, c);
}

// A row of K contiguous vector elements (the solver's [n][K] layout) moved with the widest
// access its size allows, up to 16 bytes; the row must be aligned to that width (the
// solver's vectors are 256-byte aligned and K is a power of two).  Plain loads: the data
// may have been written earlier in the same kernel by other blocks.
template <typename V, int K>
struct RowIO {
    static constexpr int BYTES = K * (int)sizeof(V);
    static constexpr int W = BYTES % 16 == 0 ? 16 : BYTES % 8 == 0 ? 8 : (int)sizeof(V);
    static constexpr int N = BYTES / W;          // accesses per row
    static constexpr int E = W / (int)sizeof(V); // elements per access
    __device__ static __forceinline__ void load(const V *p, V (&v)[K])
    {
        if constexpr (W == 16) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const uint4 u = reinterpret_cast<const uint4 *>(p)[i];
                memcpy(&v[i * E], &u, 16);
            }
        } else if constexpr (W == 8 && sizeof(V) == 4) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const uint2 u = reinterpret_cast<const uint2 *>(p)[i];
                memcpy(&v[i * E], &u, 8);
            }
        } else {
#pragma unroll
            for (int c = 0; c < K; ++c)
                v[c] = p[c];
        }
    }
    __device__ static __forceinline__ void store(V *p, const V (&v)[K])
    {
        if constexpr (W == 16) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                uint4 u;
                memcpy(&u, &v[i * E], 16);
                reinterpret_cast<uint4 *>(p)[i] = u;
            }
        } else if constexpr (W == 8 && sizeof(V) == 4) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                uint2 u;
                memcpy(&u, &v[i * E], 8);
                reinterpret_cast<uint2 *>(p)[i] = u;
            }
        } else {
#pragma unroll
            for (int c = 0; c < K; ++c)
                p[c] = v[c];
        }
    }
};

// Interface of an operation (the row epilogue an SpMV engine runs), for K right-hand sides:
//   NP dot products per column reduced over the grid, NS staged scalars, NV own-row
//   vectors the epilogue reads, NG gathered vectors combined into the SpMV operand;
//   operand(j, c) / operand_row(j, o): the operand at vector row j (global memory);
//   combine(g, c): the operand from the NG gathered values (shared-memory windows);
//   load_rv(v, i, o): own-row vector v at row i; emit(i, acc, part, s, rv): the epilogue of
//   row i with its row sums acc; finalize(sums): the scalar step after the grid reduction.

// y = A x for K right-hand sides with leading dimension ld (columns c >= nc are zero).
template <typename V, int K>
struct OpSpmv {
    using VV = V;
    static constexpr int NP = 0, NS = 0, NV = 0;
    static constexpr bool ANY_LD = true;
    static constexpr int NG = 1;
    const V *x;
    V *y;
    int ld, nc;
    // whole-row vector accesses: set by the host only when ld == nc == K and x, y are
    // aligned to the row width the access uses (RowIO)
    bool rows = false;
    __device__ const V *row_vec(int) const { return nullptr; }
    __host__ __device__ const V *gvec(int) const { return x; }
    __host__ __device__ int gstride() const { return ld; }
    static __device__ constexpr int rv_src(int) { return -1; }
    __device__ bool skip() const { return false; }
    __device__ void stage(double *) const {}
    __device__ __forceinline__ V combine(const V (&g)[NG], int c, const double *) const
    {
        return c < nc ? g[0] : (V)0;
    }
    __device__ __forceinline__ V operand(int64_t j, int c, const double *) const
    {
        return c < nc ? __ldg(&x[j * ld + c]) : (V)0;
    }
    // caller vectors: any leading dimension, so element by element (whole rows when the
    // host found the layout and alignment allow it)
    __device__ __forceinline__ void operand_row(int64_t j, V (&o)[K], const double *s) const
    {
        if (rows) {
            RowIO<V, K>::load(x + j * K, o);
            return;
        }
#pragma unroll
        for (int c = 0; c < K; ++c)
            o[c] = operand(j, c, s);
    }
    __device__ __forceinline__ void load_rv(int, int64_t, V (&o)[K]) const
    {
#pragma unroll
        for (int c = 0; c < K; ++c)
            o[c] = (V)0;
    }
    template <int N, class RV>
    __device__ __forceinline__ void emit(int64_t i, const double (&acc)[K], double (&)[N], const double *,
                                         const RV &) const
    {
        if (rows) {
            V v[K];
#pragma unroll
            for (int c = 0; c < K; ++c)
                v[c] = (V)acc[c];
            RowIO<V, K>::store(y + i * K, v);
            return;
        }
#pragma unroll
        for (int c = 0; c < K; ++c)
            if (c < nc)
                y[i * ld + c] = (V)acc[c];
    }
    __device__ void finalize(const double *) const {}
};

// Q: p_new = z + beta p_old, q = A p_new, partial p_new.q
template <typename V, int K>
struct OpQ {
    using VV = V;
    using IO = RowIO<V, K>;
    static constexpr int NP = 1, NS = K, NV = 2;
    const V *z;
    const V *p_old;
    V *p_new;
    V *q;
    PcgState *st;
    static constexpr int NG = 2;
    __device__ const V *row_vec(int v) const { return v == 0 ? p_old : z; }
    __host__ __device__ const V *gvec(int g) const { return g == 0 ? p_old : z; }
    __host__ __device__ int gstride() const { return K; }
    static __device__ constexpr int rv_src(int v) { return v; }
    __device__ bool skip() const { return *(volatile int *)&st->all_done; }
    __device__ void stage(double *s) const
    {
        for (int c = 0; c < K; ++c)
            s[c] = st->beta[c];
    }
    __device__ __forceinline__ V combine(const V (&g)[NG], int c, const double *s) const
    {
        return vfma<V>(s[c], g[0], g[1]);
    }
    __device__ __forceinline__ V operand(int64_t j, int c, const double *s) const
    {
        return vfma<V>(s[c], p_old[j * K + c], z[j * K + c]);
    }
    __device__ __forceinline__ void operand_row(int64_t j, V (&o)[K], const double *s) const
    {
        V p[K], zz[K];
        IO::load(p_old + j * K, p);
        IO::load(z + j * K, zz);
#pragma unroll
        for (int c = 0; c < K; ++c)
            o[c] = vfma<V>(s[c], p[c], zz[c]);
    }
    __device__ __forceinline__ void load_rv(int v, int64_t i, V (&o)[K]) const
    {
        IO::load(row_vec(v) + i * K, o);
    }
    template <int N, class RV>
    __device__ __forceinline__ void emit(int64_t i, const double (&acc)[K], double (&part)[N],
                                         const double *s, const RV &rv) const
    {
        V pn[K], qv[K];
#pragma unroll
        for (int c = 0; c < K; ++c) {
            pn[c] = vfma<V>(s[c], rv.get(0, i, c), rv.get(1, i, c));
            qv[c] = (V)acc[c];
            part[c] += (double)pn[c] * (double)qv[c];
        }
        IO::store(p_new + i * K, pn);
        IO::store(q + i * K, qv);
    }
    __device__ void finalize(const double *sums) const { finalize_alpha(st, sums); }
};

// U_S: r_new = r_old - alpha q, x += alpha p, y = G^T r_new, partial r_new.r_new.  Columns
// that have stopped keep r and x (x is rewritten with its own value).
template <typename V, int K>
struct OpUS {
    using VV = V;
    using IO = RowIO<V, K>;
    static constexpr int NP = 1, NS = 2 * K, NV = 4;
    const V *r_old;
    const V *q;
    const V *p;
    const V *x_in;
    V *r_new;
    V *x;
    V *y;
    PcgState *st;
    static constexpr int NG = 2;
    __device__ const V *row_vec(int v) const { return v == 0 ? r_old : v == 1 ? q : v == 2 ? p : x_in; }
    __host__ __device__ const V *gvec(int g) const { return g == 0 ? r_old : q; }
    __host__ __device__ int gstride() const { return K; }
    static __device__ constexpr int rv_src(int v) { return v < 2 ? v : -1; }
    __device__ bool skip() const { return *(volatile int *)&st->all_done; }
    __device__ void stage(double *s) const
    {
        for (int c = 0; c < K; ++c) {
            s[c] = st->alpha[c];
            s[K + c] = st->active[c] ? 1.0 : 0.0;
        }
    }
    __device__ __forceinline__ V rnew(V ro, V qv, int c, const double *s) const
    {
        return s[K + c] != 0.0 ? vfma<V>(-s[c], qv, ro) : ro;
    }
    __device__ __forceinline__ V combine(const V (&g)[NG], int c, const double *s) const
    {
        return rnew(g[0], g[1], c, s);
    }
    __device__ __forceinline__ V operand(int64_t j, int c, const double *s) const
    {
        return rnew(r_old[j * K + c], q[j * K + c], c, s);
    }
    __device__ __forceinline__ void operand_row(int64_t j, V (&o)[K], const double *s) const
    {
        V ro[K], qq[K];
        IO::load(r_old + j * K, ro);
        IO::load(q + j * K, qq);
#pragma unroll
        for (int c = 0; c < K; ++c)
            o[c] = rnew(ro[c], qq[c], c, s);
    }
    __device__ __forceinline__ void load_rv(int v, int64_t i, V (&o)[K]) const
    {
        IO::load(row_vec(v) + i * K, o);
    }
    template <int N, class RV>
    __device__ __forceinline__ void emit(int64_t i, const double (&acc)[K], double (&part)[N],
                                         const double *s, const RV &rv) const
    {
        V rn[K], xn[K], yv[K];
#pragma unroll
        for (int c = 0; c < K; ++c) {
            rn[c] = rnew(rv.get(0, i, c), rv.get(1, i, c), c, s);
            xn[c] = s[K + c] != 0.0 ? vfma<V>(s[c], rv.get(2, i, c), rv.get(3, i, c)) : rv.get(3, i, c);
            yv[c] = (V)acc[c];
            part[c] += (double)rn[c] * (double)rn[c];
        }
        IO::store(r_new + i * K, rn);
        IO::store(x + i * K, xn);
        IO::store(y + i * K, yv);
    }
    __device__ void finalize(const double *sums) const
    {
        if (st->profile)
            return;
        finalize_residual(st, sums);
        signal_if_done(st);
    }
};

// Z: z = G y + eps r, partial r.z
template <typename V, int K>
struct OpZ {
    using VV = V;
    using IO = RowIO<V, K>;
    static constexpr int NP = 1, NS = 1, NV = 1;
    const V *y;
    const V *r;
    V *z;
    PcgState *st;
    static constexpr int NG = 1;
    __device__ const V *row_vec(int) const { return r; }
    __host__ __device__ const V *gvec(int) const { return y; }
    __host__ __device__ int gstride() const { return K; }
    static __device__ constexpr int rv_src(int) { return -1; }
    __device__ bool skip() const { return *(volatile int *)&st->all_done; }
    __device__ void stage(double *s) const { s[0] = st->eps; }
    __device__ __forceinline__ V combine(const V (&g)[NG], int, const double *) const { return g[0]; }
    __device__ __forceinline__ V operand(int64_t j, int c, const double *) const
    {
        return y[j * K + c];
    }
    __device__ __forceinline__ void operand_row(int64_t j, V (&o)[K], const double *) const
    {
        IO::load(y + j * K, o);
    }
    __device__ __forceinline__ void load_rv(int, int64_t i, V (&o)[K]) const
    {
        IO::load(r + i * K, o);
    }
    template <int N, class RV>
    __device__ __forceinline__ void emit(int64_t i, const double (&acc)[K], double (&part)[N],
                                         const double *s, const RV &rv) const
    {
        V zv[K];
#pragma unroll
        for (int c = 0; c < K; ++c) {
            const V rv_ = rv.get(0, i, c);
            zv[c] = vfma<V>(s[0], rv_, (V)acc[c]);
            part[c] += (double)rv_ * (double)zv[c];
        }
        IO::store(z + i * K, zv);
    }
    __device__ void finalize(const double *sums) const { finalize_beta(st, sums); }
};

// Operations for matrices with long rows, whose SpMVs are bound by the random operand
// gathers: the operand vector is formed by an elementwise pass first (k_ep, k_er), so each
// stored entry gathers one value instead of two.
// Q': q = A p_new, partial p_new.q (p_new already formed).
template <typename V, int K>
struct OpQm {
    using VV = V;
    using IO = RowIO<V, K>;
    static constexpr int NP = 1, NS = 0, NV = 1, NG = 1;
    const V *pn;
    V *q;
    PcgState *st;
    __device__ const V *row_vec(int) const { return pn; }
    __host__ __device__ const V *gvec(int) const { return pn; }
    __host__ __device__ int gstride() const { return K; }
    static __device__ constexpr int rv_src(int) { return 0; }
    __device__ bool skip() const { return *(volatile int *)&st->all_done; }
    __device__ void stage(double *) const {}
    __device__ __forceinline__ V combine(const V (&g)[NG], int, const double *) const { return g[0]; }
    __device__ __forceinline__ V operand(int64_t j, int c, const double *) const { return pn[j * K + c]; }
    __device__ __forceinline__ void operand_row(int64_t j, V (&o)[K], const double *) const
    {
        IO::load(pn + j * K, o);
    }
    __device__ __forceinline__ void load_rv(int, int64_t i, V (&o)[K]) const { IO::load(pn + i * K, o); }
    template <int N, class RV>
    __device__ __forceinline__ void emit(int64_t i, const double (&acc)[K], double (&part)[N],
                                         const double *, const RV &rv) const
    {
        V qv[K];
#pragma unroll
        for (int c = 0; c < K; ++c) {
            qv[c] = (V)acc[c];
            part[c] += (double)rv.get(0, i, c) * (double)qv[c];
        }
        IO::store(q + i * K, qv);
    }
    __device__ void finalize(const double *sums) const { finalize_alpha(st, sums); }
};

// U_S': y = G^T r_new (r_new already formed, with the residual test).
template <typename V, int K>
struct OpUSm {
    using VV = V;
    using IO = RowIO<V, K>;
    static constexpr int NP = 0, NS = 0, NV = 0, NG = 1;
    const V *rn;
    V *y;
    PcgState *st;
    __device__ const V *row_vec(int) const { return nullptr; }
    __host__ __device__ const V *gvec(int) const { return rn; }
    __host__ __device__ int gstride() const { return K; }
    static __device__ constexpr int rv_src(int) { return -1; }
    __device__ bool skip() const { return *(volatile int *)&st->all_done; }
    __device__ void stage(double *) const {}
    __device__ __forceinline__ V combine(const V (&g)[NG], int, const double *) const { return g[0]; }
    __device__ __forceinline__ V operand(int64_t j, int c, const double *) const { return rn[j * K + c]; }
    __device__ __forceinline__ void operand_row(int64_t j, V (&o)[K], const double *) const
    {
        IO::load(rn + j * K, o);
    }
    __device__ __forceinline__ void load_rv(int, int64_t, V (&o)[K]) const
    {
#pragma unroll
        for (int c = 0; c < K; ++c)
            o[c] = (V)0;
    }
    template <int N, class RV>
    __device__ __forceinline__ void emit(int64_t i, const double (&acc)[K], double (&)[N], const double *,
                                         const RV &) const
    {
        V yv[K];
#pragma unroll
        for (int c = 0; c < K; ++c)
            yv[c] = (V)acc[c];
        IO::store(y + i * K, yv);
    }
    __device__ void finalize(const double *) const {}
};

// U_J on row i: x += alpha p and r -= alpha q in the active columns, z = D^-1 r; adds r.r
// to part[c] and r.z to part[K + c].  Stopped columns are rewritten with their own values.
template <typename V, int K>
__device__ __forceinline__ void jacobi_row(int64_t i, V *x, V *r, const V *p, const V *q, V *z,
                                           const V *dinv, const double *alpha, const double *on,
                                           double (&part)[2 * K])
{
    using IO = RowIO<V, K>;
    V xr[K], rr[K], pr[K], qr[K], zr[K];
    const double di = (double)dinv[i];
    IO::load(x + i * K, xr);
    IO::load(r + i * K, rr);
    IO::load(p + i * K, pr);
    IO::load(q + i * K, qr);
#pragma unroll
    for (int c = 0; c < K; ++c) {
        if (on[c] != 0.0) {
            xr[c] = vfma<V>(alpha[c], pr[c], xr[c]);
            rr[c] = vfma<V>(-alpha[c], qr[c], rr[c]);
        }
        const double rv = (double)rr[c];
        zr[c] = (V)(rv * di);
        part[c] += rv * rv;
        part[K + c] += rv * (double)zr[c];
    }
    IO::store(x + i * K, xr);
    IO::store(r + i * K, rr);
    IO::store(z + i * K, zr);
}

}  // namespace sla
