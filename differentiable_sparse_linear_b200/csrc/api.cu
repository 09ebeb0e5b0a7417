// C ABI of libsla: argument checks, handles, tile partitions, solve plans.
#include <cuda_runtime.h>

#include <algorithm>
#include <map>
#include <memory>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "sla.h"
#include "sla_internal.cuh"

#define SLA_VERSION_STRING "sla-b200 0.1.0 (sm_100a)"

namespace sla {

static thread_local std::string g_last_error;

void set_error(const std::string &msg) { g_last_error = msg; }

sla_status fail(sla_status code, const std::string &msg)
{
    set_error(msg);
    return code;
}

sla_status cuda_fail(cudaError_t e, const char *what)
{
    std::string m = std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
    set_error(m);
    return e == cudaErrorMemoryAllocation ? SLA_ERR_OOM : SLA_ERR_CUDA;
}

static size_t vbytes(sla_dtype d) { return d == SLA_F32 ? 4 : 8; }

// Rows grouped into tiles of at most D items (rows + entries) and at most RMAX rows; a row
// with D or more entries forms a tile of its own.  desc[t] = {first row, first entry}.
sla_status ensure_tiles(sla_csr *A, int D, int RMAX, cudaStream_t s, const TilePart **out)
{
    const int key = D * 65536 + RMAX;
    auto it = A->tiles.find(key);
    if (it != A->tiles.end()) {
        *out = &it->second;
        return SLA_SUCCESS;
    }
    std::vector<int32_t> t;
    t.reserve((size_t)(A->n + A->nnz) / (size_t)D + (size_t)A->n / (size_t)RMAX + 16);
    t.push_back(0);
    int64_t items = 0, rows = 0;
    for (int64_t r = 0; r < A->n; ++r) {
        const int64_t len = (int64_t)A->h_rp[r + 1] - A->h_rp[r];
        if (len + 1 > D) {
            if (items > 0) {
                t.push_back((int32_t)r);
                items = rows = 0;
            }
            t.push_back((int32_t)(r + 1));
            continue;
        }
        if (items + len + 1 > D || rows + 1 > RMAX) {
            t.push_back((int32_t)r);
            items = rows = 0;
        }
        items += len + 1;
        rows += 1;
    }
    if (items > 0)
        t.push_back((int32_t)A->n);
    std::vector<int2> desc(t.size());
    for (size_t i = 0; i < t.size(); ++i)
        desc[i] = make_int2(t[i], A->h_rp[(size_t)t[i]]);
    TilePart tp;
    tp.D = D;
    tp.RMAX = RMAX;
    tp.n_tiles = (int)t.size() - 1;
    SLA_CUDA_TRY(cudaMalloc((void **)&tp.d_desc, desc.size() * sizeof(int2)));
    SLA_CUDA_TRY(cudaMemcpyAsync(tp.d_desc, desc.data(), desc.size() * sizeof(int2),
                                 cudaMemcpyHostToDevice, s));
    SLA_CUDA_TRY(cudaStreamSynchronize(s));
    auto ins = A->tiles.emplace(key, tp);
    *out = &ins.first->second;
    return SLA_SUCCESS;
}

static sla_status fetch_host_cols(sla_csr *A, cudaStream_t s)
{
    if (A->h_ci.size() != (size_t)A->nnz) {
        A->h_ci.resize((size_t)A->nnz);
        if (A->nnz > 0) {
            SLA_CUDA_TRY(cudaMemcpyAsync(A->h_ci.data(), A->ci, (size_t)A->nnz * sizeof(int32_t),
                                         cudaMemcpyDeviceToHost, s));
            SLA_CUDA_TRY(cudaStreamSynchronize(s));
        }
    }
    return SLA_SUCCESS;
}

// Operand window of rows [r0, r1): the rows of the gathered vectors their columns (and the
// rows themselves) touch, as at most WSEG 4-row-aligned ranges totalling at most wmax rows
// and ending at most at row_limit; false when they do not fit.  Gaps of up to 32 rows are
// bridged.
static bool window_for_rows(const sla_csr *A, int64_t r0, int64_t r1, int wmax, int64_t row_limit,
                            WinDesc *out)
{
    const int64_t GAP = 32;
    WinDesc w{};
    *out = w;
    int64_t lo[8], hi[8];   // closed ranges
    int ns = 0;
    bool ok = wmax > 0;
    auto add = [&](int64_t j) {
        for (int i = 0; i < ns; ++i)
            if (j >= lo[i] - GAP && j <= hi[i] + GAP) {
                lo[i] = std::min(lo[i], j);
                hi[i] = std::max(hi[i], j);
                return;
            }
        if (ns == 8) {
            ok = false;
            return;
        }
        lo[ns] = hi[ns] = j;
        ++ns;
    };
    for (int64_t r = r0; ok && r < r1; ++r)   // the rows themselves (own-row values)
        add(r);
    for (int64_t k = A->h_rp[(size_t)r0]; ok && k < (int64_t)A->h_rp[(size_t)r1]; ++k)
        add(A->h_ci[(size_t)k]);
    if (!ok)
        return false;
    // sort, align to 4 rows, merge
    int64_t L[8], H[8];
    int m = 0;
    for (int i = 0; i < ns; ++i) {
        int b = i;
        for (int jdx = i + 1; jdx < ns; ++jdx)
            if (lo[jdx] < lo[b])
                b = jdx;
        std::swap(lo[i], lo[b]);
        std::swap(hi[i], hi[b]);
    }
    for (int i = 0; i < ns; ++i) {
        const int64_t a = lo[i] & ~(int64_t)3, e = (hi[i] + 1 + 3) & ~(int64_t)3;
        if (m > 0 && a <= H[m - 1] + GAP)
            H[m - 1] = std::max(H[m - 1], e);
        else {
            L[m] = a;
            H[m] = e;
            ++m;
        }
    }
    int64_t total = 0;
    for (int i = 0; i < m; ++i)
        total += H[i] - L[i];
    if (m > WSEG || total > wmax || (m > 0 && H[m - 1] > row_limit))
        return false;
    w.nseg = m;
    for (int i = 0; i < m; ++i) {
        w.a[i] = (int)L[i];
        w.l[i] = (int)(H[i] - L[i]);
    }
    *out = w;
    return true;
}

sla_status ensure_groups(sla_csr *A, cudaStream_t s, const GroupPart **out)
{
    if (A->groups) {
        *out = A->groups;
        return SLA_SUCCESS;
    }
    std::vector<int32_t> bin_rows[GBINS];
    const int64_t per_lane = A->bdim > 1 ? 2 : 4;   // items a lane takes per pass
    const int64_t nrows = pattern_rows(A);
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t len = (int64_t)A->h_rp[(size_t)r + 1] - A->h_rp[(size_t)r];
        int b = GBINS - 1;                  // G = 1
        while (b > 0 && per_lane * (int64_t(1) << (GBINS - 1 - b)) < len)
            --b;
        bin_rows[b].push_back((int32_t)r);
    }
    auto len_of = [&](int32_t r) { return A->h_rp[(size_t)r + 1] - A->h_rp[(size_t)r]; };
    std::stable_sort(bin_rows[0].begin(), bin_rows[0].end(),
                     [&](int32_t a, int32_t b) { return len_of(a) > len_of(b); });
    auto gp = std::make_unique<GroupPart>();
    std::vector<int4> rows;
    rows.reserve((size_t)A->n);
    int tasks = 0;
    for (int b = 0; b < GBINS; ++b) {
        const int per_task = 1 << b;        // 32 / G rows per warp task
        gp->task0[b] = tasks;
        gp->pos0[b] = (int)rows.size();
        tasks += (int)((bin_rows[b].size() + per_task - 1) / per_task);
        for (int32_t r : bin_rows[b])
            rows.push_back(make_int4(r, A->h_rp[(size_t)r], A->h_rp[(size_t)r + 1], 0));
    }
    gp->task0[GBINS] = tasks;
    gp->pos0[GBINS] = (int)rows.size();
    gp->n_tasks = tasks;
    if (!rows.empty()) {
        SLA_CUDA_TRY(cudaMalloc((void **)&gp->d_rows, rows.size() * sizeof(int4)));
        SLA_CUDA_TRY(cudaMemcpyAsync(gp->d_rows, rows.data(), rows.size() * sizeof(int4),
                                     cudaMemcpyHostToDevice, s));
        SLA_CUDA_TRY(cudaStreamSynchronize(s));
    }
    A->groups = gp.release();
    *out = A->groups;
    return SLA_SUCCESS;
}

// Operand windows of every tile of a partition (tiles that do not fit get nseg = 0 and
// gather from global memory).  Windows end inside the vectors (row n at most), since the
// gathered vectors can be the caller's.
sla_status ensure_windows(sla_csr *A, const TilePart *tp_c, int wmax, cudaStream_t s)
{
    TilePart *tp = const_cast<TilePart *>(tp_c);
    if (tp->win_rows == wmax)
        return SLA_SUCCESS;
    SLA_TRY(fetch_host_cols(A, s));
    std::vector<int2> desc((size_t)tp->n_tiles + 1);
    if (tp->n_tiles > 0)
        SLA_CUDA_TRY(cudaMemcpy(desc.data(), tp->d_desc, desc.size() * sizeof(int2), cudaMemcpyDeviceToHost));
    std::vector<WinDesc> win((size_t)std::max(tp->n_tiles, 1));
    for (int t = 0; t < tp->n_tiles; ++t)
        window_for_rows(A, desc[t].x, desc[t + 1].x, wmax, A->n, &win[(size_t)t]);
    if (!tp->d_win)
        SLA_CUDA_TRY(cudaMalloc((void **)&tp->d_win, win.size() * sizeof(WinDesc)));
    SLA_CUDA_TRY(cudaMemcpyAsync(tp->d_win, win.data(), win.size() * sizeof(WinDesc), cudaMemcpyHostToDevice, s));
    SLA_CUDA_TRY(cudaStreamSynchronize(s));
    tp->win_rows = wmax;
    return SLA_SUCCESS;
}

// Sliced copy (see SellPart).
sla_status ensure_sell(sla_csr *A, cudaStream_t s, const SellPart **out)
{
    // offsets per diagonal slice at most: the matrix's own row-length class (a kernel that
    // reads the layout unrolls to at least this)
    const int maxl = A->max_row_len <= 8 ? 8 : 16;
    if (A->sell && A->sell->maxl == maxl) {
        *out = A->sell;
        return SLA_SUCCESS;
    }
    SLA_TRY(fetch_host_cols(A, s));
    const int64_t n = A->n;
    const int64_t nsl = (n + 31) / 32;
    std::vector<uint2> desc((size_t)std::max<int64_t>(nsl, 1));
    std::vector<uint8_t> lens((size_t)std::max<int64_t>(nsl * 32, 1), 0);
    std::vector<int32_t> offs;
    std::vector<std::vector<int64_t>> slice_offs((size_t)nsl);
    std::map<std::vector<int64_t>, uint32_t> list_pos;
    bool rel16 = true;
    int64_t slot_rows = 0, n_diag = 0;
    for (int64_t sl = 0; sl < nsl; ++sl) {
        int64_t L = 0;
        std::vector<int64_t> u;
        bool diag = true;
        for (int64_t r = sl * 32; r < std::min(n, sl * 32 + 32); ++r) {
            const int64_t len = (int64_t)A->h_rp[(size_t)r + 1] - A->h_rp[(size_t)r];
            lens[(size_t)r] = (uint8_t)len;
            L = std::max(L, len);
            for (int64_t k = A->h_rp[(size_t)r]; k < (int64_t)A->h_rp[(size_t)r + 1]; ++k) {
                const int64_t d = (int64_t)A->h_ci[(size_t)k] - r;
                if (d < -32768 || d > 32767)
                    rel16 = false;
                if (diag && std::find(u.begin(), u.end(), d) == u.end()) {
                    u.push_back(d);
                    if ((int64_t)u.size() > maxl)
                        diag = false;
                }
            }
        }
        if (slot_rows >= ((int64_t)1 << 27) || (int64_t)offs.size() >= ((int64_t)1 << 30) - maxl)
            return fail(SLA_ERR_UNSUPPORTED, "matrix too large for the sliced layout");
        uint32_t w1 = 0;
        // a diagonal slice is "full" when every row holds every offset of the list: entry u of
        // row r is then CSR entry row_ptr[r] + u, so the product can skip the column indices
        bool full = true;
        if (diag && !u.empty())
            for (int64_t r = sl * 32; r < std::min(n, sl * 32 + 32); ++r)
                if ((int64_t)A->h_rp[(size_t)r + 1] - A->h_rp[(size_t)r] != (int64_t)u.size())
                    full = false;
        if (diag && !u.empty()) {
            std::sort(u.begin(), u.end());
            // slices with the same offsets share one list (a stencil has a handful)
            auto it = list_pos.find(u);
            if (it == list_pos.end()) {
                it = list_pos.emplace(u, (uint32_t)offs.size()).first;
                for (int64_t d : u)
                    offs.push_back((int32_t)d);
            }
            w1 = (1u << 31) | (full ? (1u << 30) : 0u) | it->second;
            L = (int64_t)u.size();
            slice_offs[(size_t)sl] = u;
            ++n_diag;
        }
        desc[(size_t)sl] = make_uint2((uint32_t)(slot_rows << 5) | (uint32_t)L, w1);
        slot_rows += L;
    }
    const int64_t slots = slot_rows * 32;
    std::vector<int32_t> perm((size_t)std::max<int64_t>(slots, 1), -1);
    std::vector<int16_t> i16;
    std::vector<int32_t> i32;
    if (rel16)
        i16.assign((size_t)std::max<int64_t>(slots, 1), 0);
    else
        i32.assign((size_t)std::max<int64_t>(slots, 1), 0);
    for (int64_t sl = 0; sl < nsl; ++sl) {
        const int64_t e0 = (int64_t)(desc[(size_t)sl].x >> 5) * 32;
        const bool diag = desc[(size_t)sl].y >> 31;
        const std::vector<int64_t> &u = slice_offs[(size_t)sl];
        for (int64_t l = 0; l < 32; ++l) {
            const int64_t r = sl * 32 + l;
            if (r >= n)
                break;
            const int64_t k0 = A->h_rp[(size_t)r], len = (int64_t)A->h_rp[(size_t)r + 1] - k0;
            for (int64_t t = 0; t < len; ++t) {
                const int64_t j = A->h_ci[(size_t)(k0 + t)];
                // slot row of this entry: its offset's position (diagonal), else its rank
                const int64_t pos = diag ? (int64_t)(std::lower_bound(u.begin(), u.end(), j - r) - u.begin()) : t;
                const size_t e = (size_t)(e0 + pos * 32 + l);
                perm[e] = (int32_t)(k0 + t);
                if (rel16)
                    i16[e] = (int16_t)(j - r);
                else
                    i32[e] = (int32_t)j;
            }
        }
    }
    if (A->groups) {
        cudaFree(A->groups->d_rows);
        delete A->groups;
        A->groups = nullptr;
    }
    if (A->sell) {
        cudaFree(A->sell->d_desc);
        cudaFree(A->sell->d_offs);
        cudaFree(A->sell->d_lens);
        cudaFree(A->sell->d_idx);
        cudaFree(A->sell->d_perm);
        cudaFree(A->sell->d_val);
        delete A->sell;
        A->sell = nullptr;
    }
    SellPart *sp = new SellPart();
    A->sell_vals_current = 0;
    sp->n_slices = nsl;
    sp->n_slots = slots;
    sp->rel16 = rel16 ? 1 : 0;
    sp->maxl = maxl;
    sp->n_diag = n_diag;
    const size_t vsz = vbytes(A->dtype);
    const size_t isz = rel16 ? 2 : 4;
    auto cleanup = [&](cudaError_t e, const char *what) {
        cudaFree(sp->d_desc);
        cudaFree(sp->d_offs);
        cudaFree(sp->d_lens);
        cudaFree(sp->d_idx);
        cudaFree(sp->d_perm);
        cudaFree(sp->d_val);
        delete sp;
        return cuda_fail(e, what);
    };
    cudaError_t e = cudaMalloc((void **)&sp->d_desc, desc.size() * sizeof(uint2));
    if (e == cudaSuccess)
        e = cudaMalloc((void **)&sp->d_offs, std::max<size_t>(offs.size(), 1) * sizeof(int32_t));
    if (e == cudaSuccess)
        e = cudaMalloc((void **)&sp->d_lens, lens.size());
    if (e == cudaSuccess)
        e = cudaMalloc(&sp->d_idx, perm.size() * isz);
    if (e == cudaSuccess)
        e = cudaMalloc((void **)&sp->d_perm, perm.size() * 4);
    if (e == cudaSuccess)
        e = cudaMalloc(&sp->d_val, perm.size() * vsz);
    if (e != cudaSuccess)
        return cleanup(e, "sliced layout");
    e = cudaMemcpyAsync(sp->d_desc, desc.data(), desc.size() * sizeof(uint2), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && !offs.empty())
        e = cudaMemcpyAsync(sp->d_offs, offs.data(), offs.size() * sizeof(int32_t), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(sp->d_lens, lens.data(), lens.size(), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(sp->d_idx, rel16 ? (const void *)i16.data() : (const void *)i32.data(),
                            perm.size() * isz, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(sp->d_perm, perm.data(), perm.size() * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(s);
    if (e != cudaSuccess)
        return cleanup(e, "sliced layout upload");
    A->sell = sp;
    *out = sp;
    return SLA_SUCCESS;
}

static size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

static size_t vec_bytes(const sla_csr *A, int vec64) { return vec64 ? 8 : vbytes(A->dtype); }

size_t plan_bytes(const sla_csr *A, const sla_precond *M, int K, int vec64)
{
    (void)M;
    const size_t vec = align256((size_t)A->n * (size_t)K * vec_bytes(A, vec64));
    const size_t parts = align256((size_t)A->num_sms * 32 * 2 * KMAX * sizeof(double));
    return 8 * vec + parts + align256(sizeof(PcgState));
}

void destroy_plan(Plan *p)
{
    if (!p)
        return;
    if (p->exec)
        cudaGraphExecDestroy(p->exec);
    if (p->graph)
        cudaGraphDestroy(p->graph);
    if (p->cs)
        cudaStreamDestroy(p->cs);
    if (p->cs2)
        cudaStreamDestroy(p->cs2);
    if (p->ws)
        cudaFree(p->ws);
    if (p->h_st)
        cudaFreeHost(p->h_st);
    delete p;
}

sla_status get_plan(sla_csr *A, const sla_precond *M, int K, int vec64, Plan **out)
{
    vec64 = (vec64 && A->dtype == SLA_F32) ? 1 : 0;
    for (Plan *p : A->plans)
        if (p->M == M && p->K == K && p->vec64 == vec64) {
            *out = p;
            return SLA_SUCCESS;
        }
    Plan *p = new Plan();
    p->M = M;
    p->K = K;
    p->vec64 = vec64;
    p->kind = M ? M->kind : 0;
    p->ws_bytes = plan_bytes(A, M, K, vec64);
    auto cleanup = [&](sla_status st) {
        destroy_plan(p);
        return st;
    };
    cudaError_t e = cudaMalloc(&p->ws, p->ws_bytes);
    if (e != cudaSuccess)
        return cleanup(cuda_fail(e, "solver workspace"));
    e = cudaMallocHost((void **)&p->h_st, sizeof(PcgState));
    if (e != cudaSuccess)
        return cleanup(cuda_fail(e, "pinned solver state"));
    const size_t vec = align256((size_t)A->n * (size_t)K * vec_bytes(A, vec64));
    char *b = (char *)p->ws;
    void **vs[8] = {&p->x, &p->ra, &p->rb, &p->pa, &p->pb, &p->q, &p->z, &p->y};
    for (int i = 0; i < 8; ++i) {
        *vs[i] = b;
        b += vec;
    }
    p->partials = (double *)b;
    b += align256((size_t)A->num_sms * 32 * 2 * KMAX * sizeof(double));
    p->st = (PcgState *)b;
    e = cudaStreamCreateWithFlags(&p->cs, cudaStreamNonBlocking);
    if (e == cudaSuccess)
        e = cudaStreamCreateWithFlags(&p->cs2, cudaStreamNonBlocking);
    if (e != cudaSuccess)
        return cleanup(cuda_fail(e, "capture streams"));
    sla_status st = capture_plan_graph(A, p);
    if (st != SLA_SUCCESS)
        return cleanup(st);
    A->plans.push_back(p);
    *out = p;
    return SLA_SUCCESS;
}

static sla_status current_device(sla_csr *A)
{
    SLA_CUDA_TRY(cudaGetDevice(&A->device));
    SLA_CUDA_TRY(cudaDeviceGetAttribute(&A->num_sms, cudaDevAttrMultiProcessorCount, A->device));
    SLA_CUDA_TRY(cudaMalloc((void **)&A->d_err, sizeof(int)));
    SLA_CUDA_TRY(cudaMemset(A->d_err, 0, sizeof(int)));
    return SLA_SUCCESS;
}

// Copy row_ptr to the host, check it (always: the kernels rely on it), and optionally
// check the column pattern on the device.
static sla_status setup_pattern(sla_csr *A, uint32_t flags, cudaStream_t s)
{
    const int64_t np = pattern_rows(A);
    A->h_rp.resize((size_t)np + 1);
    SLA_CUDA_TRY(cudaMemcpyAsync(A->h_rp.data(), A->rp, ((size_t)np + 1) * sizeof(int32_t),
                                 cudaMemcpyDeviceToHost, s));
    SLA_CUDA_TRY(cudaStreamSynchronize(s));
    if (A->h_rp[0] != 0)
        return fail(SLA_ERR_INVALID_CSR, "row_ptr[0] must be 0");
    if ((int64_t)A->h_rp[(size_t)np] != pattern_nnz(A))
        return fail(SLA_ERR_INVALID_CSR, "row_ptr[n] must equal nnz");
    int64_t mx = 0;
    for (int64_t r = 0; r < np; ++r) {
        const int64_t len = (int64_t)A->h_rp[r + 1] - A->h_rp[r];
        if (len < 0)
            return fail(SLA_ERR_INVALID_CSR, "row_ptr must be non-decreasing (row " + std::to_string(r) + ")");
        mx = std::max(mx, len);
    }
    A->max_row_len = mx * A->bdim;          // scalar entries of the longest row
    if (flags & SLA_VALIDATE) {
        int *d_err = nullptr;
        SLA_CUDA_TRY(cudaMallocAsync((void **)&d_err, sizeof(int), s));
        SLA_CUDA_TRY(cudaMemsetAsync(d_err, 0, sizeof(int), s));
        sla_status st = launch_validate(A, d_err, s);
        int h_err = 0;
        if (st == SLA_SUCCESS) {
            cudaError_t e = cudaMemcpyAsync(&h_err, d_err, sizeof(int), cudaMemcpyDeviceToHost, s);
            if (e == cudaSuccess)
                e = cudaStreamSynchronize(s);
            if (e != cudaSuccess)
                st = cuda_fail(e, "validation");
        }
        cudaFreeAsync(d_err, s);
        if (st != SLA_SUCCESS)
            return st;
        if (h_err)
            return fail(SLA_ERR_INVALID_CSR,
                        "column index out of range, unsorted or repeated within a row");
    }
    return SLA_SUCCESS;
}

static void drop_plans_of(sla_csr *A, const sla_precond *M)
{
    std::vector<Plan *> keep;
    for (Plan *p : A->plans) {
        if (p->M == M)
            destroy_plan(p);
        else
            keep.push_back(p);
    }
    A->plans.swap(keep);
}

static void unlink(std::vector<sla_precond *> &v, const sla_precond *M)
{
    v.erase(std::remove(v.begin(), v.end(), M), v.end());
}

static void free_csr(sla_csr *A)
{
    if (!A)
        return;
    // detach the preconditioners that refer to A: their plans live in their matrix and
    // may reference A's arrays (as A or as G), so they go first
    for (sla_precond *M : A->dependents) {
        if (M->A && M->A != A)
            drop_plans_of(const_cast<sla_csr *>(M->A), M);
        if (M->A == A)
            M->A = nullptr;
        if (M->G == A)
            M->G = nullptr;   // a SPAI preconditioner without G refuses further use
    }
    A->dependents.clear();
    for (cudaEvent_t &ev : A->list_ev)
        if (ev) {
            cudaEventDestroy(ev);
            ev = nullptr;
        }
    for (Plan *p : A->plans)
        destroy_plan(p);
    A->plans.clear();
    for (auto &kv : A->tiles) {
        cudaFree(kv.second.d_desc);
        if (kv.second.d_win)
            cudaFree(kv.second.d_win);
    }
    if (A->sell) {
        cudaFree(A->sell->d_desc);
        cudaFree(A->sell->d_offs);
        cudaFree(A->sell->d_lens);
        cudaFree(A->sell->d_idx);
        cudaFree(A->sell->d_perm);
        cudaFree(A->sell->d_val);
        delete A->sell;
        A->sell = nullptr;
    }
    if (A->groups) {
        cudaFree(A->groups->d_rows);
        delete A->groups;
        A->groups = nullptr;
    }
    free_csb(A);
    if (A->d_err)
        cudaFree(A->d_err);
    if (A->d_sys_off)
        cudaFree(A->d_sys_off);
    if (A->own_rp)
        cudaFree(A->own_rp);
    if (A->own_ci)
        cudaFree(A->own_ci);
    if (A->own_val)
        cudaFree(A->own_val);
    delete A;
}

}  // namespace sla

using namespace sla;

extern "C" {

const char *sla_version(void) { return SLA_VERSION_STRING; }

const char *sla_status_string(sla_status s)
{
    switch (s) {
    case SLA_SUCCESS: return "SLA_SUCCESS";
    case SLA_NOT_CONVERGED: return "SLA_NOT_CONVERGED";
    case SLA_BREAKDOWN: return "SLA_BREAKDOWN";
    case SLA_ERR_INVALID_ARG: return "SLA_ERR_INVALID_ARG";
    case SLA_ERR_INVALID_CSR: return "SLA_ERR_INVALID_CSR";
    case SLA_ERR_CUDA: return "SLA_ERR_CUDA";
    case SLA_ERR_OOM: return "SLA_ERR_OOM";
    case SLA_ERR_UNSUPPORTED: return "SLA_ERR_UNSUPPORTED";
    default: return "SLA_UNKNOWN_STATUS";
    }
}

const char *sla_last_error(void) { return g_last_error.c_str(); }

sla_status sla_csr_create(sla_csr **out, int64_t n_rows, int64_t n_cols, int64_t nnz,
                          const int32_t *d_row_ptr, const int32_t *d_col, const void *d_val,
                          sla_dtype dtype, uint32_t flags, void *stream)
{
    if (!out)
        return fail(SLA_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (n_rows < 0 || nnz < 0 || n_rows != n_cols)
        return fail(SLA_ERR_INVALID_ARG, "matrix must be square with n >= 0 and nnz >= 0");
    if (n_rows >= (int64_t)INT32_MAX || nnz >= (int64_t)INT32_MAX)
        return fail(SLA_ERR_INVALID_ARG, "n and nnz must fit int32 indices");
    if (dtype != SLA_F32 && dtype != SLA_F64)
        return fail(SLA_ERR_INVALID_ARG, "dtype must be SLA_F32 or SLA_F64");
    if (!d_row_ptr || (nnz > 0 && (!d_col || !d_val)))
        return fail(SLA_ERR_INVALID_ARG, "NULL row_ptr, col or val");
    // the SpMV pipeline streams these arrays with 16-byte-aligned bulk copies
    if (((uintptr_t)d_row_ptr & 15) || ((uintptr_t)d_col & 15) || ((uintptr_t)d_val & 15))
        return fail(SLA_ERR_INVALID_ARG, "row_ptr, col and val must be 16-byte aligned device pointers");
    cudaStream_t s = (cudaStream_t)stream;
    sla_csr *A = new sla_csr();
    A->n = n_rows;
    A->nnz = nnz;
    A->dtype = dtype;
    A->flags = flags;
    A->rp = d_row_ptr;
    A->ci = d_col;
    A->val = d_val;
    A->max_sys_n = n_rows;
    A->max_sys_nnz = nnz;
    sla_status st = current_device(A);
    if (st == SLA_SUCCESS)
        st = setup_pattern(A, flags, s);
    if (st != SLA_SUCCESS) {
        free_csr(A);
        return st;
    }
    *out = A;
    return SLA_SUCCESS;
}

sla_status sla_bsr_create(sla_csr **out, int64_t n_block_rows, int32_t block_dim, int64_t nnzb,
                          const int32_t *d_row_ptr, const int32_t *d_col, const void *d_val,
                          sla_dtype dtype, uint32_t flags, void *stream)
{
    if (!out)
        return fail(SLA_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (block_dim < 2 || block_dim > 4)
        return fail(SLA_ERR_INVALID_ARG, "block_dim must be 2, 3 or 4 (use sla_csr_create for 1)");
    if (n_block_rows < 0 || nnzb < 0)
        return fail(SLA_ERR_INVALID_ARG, "n_block_rows and nnzb must be >= 0");
    const int64_t b = block_dim;
    if (n_block_rows * b >= (int64_t)INT32_MAX || nnzb * b * b >= (int64_t)INT32_MAX)
        return fail(SLA_ERR_INVALID_ARG, "scalar rows and values must fit int32 indices");
    if (dtype != SLA_F32 && dtype != SLA_F64)
        return fail(SLA_ERR_INVALID_ARG, "dtype must be SLA_F32 or SLA_F64");
    if (!d_row_ptr || (nnzb > 0 && (!d_col || !d_val)))
        return fail(SLA_ERR_INVALID_ARG, "NULL row_ptr, col or val");
    if (((uintptr_t)d_row_ptr & 15) || ((uintptr_t)d_col & 15) || ((uintptr_t)d_val & 15))
        return fail(SLA_ERR_INVALID_ARG, "row_ptr, col and val must be 16-byte aligned device pointers");
    cudaStream_t s = (cudaStream_t)stream;
    sla_csr *A = new sla_csr();
    A->bdim = block_dim;
    A->n = n_block_rows * b;
    A->nnz = nnzb * b * b;
    A->dtype = dtype;
    A->flags = flags;
    A->rp = d_row_ptr;
    A->ci = d_col;
    A->val = d_val;
    A->max_sys_n = A->n;
    A->max_sys_nnz = A->nnz;
    sla_status st = current_device(A);
    if (st == SLA_SUCCESS)
        st = setup_pattern(A, flags, s);
    if (st != SLA_SUCCESS) {
        free_csr(A);
        return st;
    }
    *out = A;
    return SLA_SUCCESS;
}

sla_status sla_csr_create_list(sla_csr **out, int32_t batch, const int64_t *h_sys_row_off,
                               int64_t nnz_total, const int32_t *d_row_ptr, const int32_t *d_col,
                               const void *d_val, sla_dtype dtype, uint32_t flags, void *stream)
{
    if (!out)
        return fail(SLA_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (batch < 1 || !h_sys_row_off)
        return fail(SLA_ERR_INVALID_ARG, "batch must be >= 1 with system offsets");
    if (h_sys_row_off[0] != 0)
        return fail(SLA_ERR_INVALID_ARG, "system offsets must start at 0");
    for (int32_t i = 0; i < batch; ++i)
        if (h_sys_row_off[i + 1] < h_sys_row_off[i])
            return fail(SLA_ERR_INVALID_ARG, "system offsets must be non-decreasing");
    const int64_t n = h_sys_row_off[batch];
    sla_csr *A = nullptr;
    sla_status st = sla_csr_create(&A, n, n, nnz_total, d_row_ptr, d_col, d_val, dtype,
                                   flags & ~SLA_VALIDATE, stream);
    if (st != SLA_SUCCESS)
        return st;
    cudaStream_t s = (cudaStream_t)stream;
    A->batch = batch;
    A->sys_off.assign(h_sys_row_off, h_sys_row_off + batch + 1);
    A->max_sys_n = 0;
    A->max_sys_nnz = 0;
    for (int32_t i = 0; i < batch; ++i) {
        A->max_sys_n = std::max<int64_t>(A->max_sys_n, h_sys_row_off[i + 1] - h_sys_row_off[i]);
        A->max_sys_nnz = std::max<int64_t>(
            A->max_sys_nnz, (int64_t)A->h_rp[(size_t)h_sys_row_off[i + 1]] - A->h_rp[(size_t)h_sys_row_off[i]]);
    }
    cudaError_t e = cudaMalloc((void **)&A->d_sys_off, sizeof(int64_t) * (size_t)(batch + 1));
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(A->d_sys_off, h_sys_row_off, sizeof(int64_t) * (size_t)(batch + 1),
                            cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
        st = cuda_fail(e, "system offsets");
        free_csr(A);
        return st;
    }
    if (flags & SLA_VALIDATE) {
        A->flags = flags;
        st = setup_pattern(A, flags, s);
        if (st != SLA_SUCCESS) {
            free_csr(A);
            return st;
        }
    }
    *out = A;
    return SLA_SUCCESS;
}

sla_status sla_csr_destroy(sla_csr *A)
{
    free_csr(A);
    return SLA_SUCCESS;
}

sla_status sla_csr_shape(const sla_csr *A, int64_t *n_rows, int64_t *nnz, int32_t *batch)
{
    if (!A)
        return fail(SLA_ERR_INVALID_ARG, "NULL handle");
    if (n_rows)
        *n_rows = A->n;
    if (nnz)
        *nnz = A->nnz;
    if (batch)
        *batch = A->batch;
    return SLA_SUCCESS;
}

sla_status sla_spmv(const sla_csr *A, const void *d_x, void *d_y, void *stream)
{
    if (!A)
        return fail(SLA_ERR_INVALID_ARG, "NULL handle");
    if (A->n > 0 && (!d_x || !d_y))
        return fail(SLA_ERR_INVALID_ARG, "NULL vector");
    if (A->n > 0 && d_x == d_y)
        return fail(SLA_ERR_INVALID_ARG, "x and y must not overlap");
    return launch_spmv(A, 1, d_x, d_y, (cudaStream_t)stream);
}

sla_status sla_spmv_multi(const sla_csr *A, int32_t nrhs, const void *d_X, void *d_Y, void *stream)
{
    if (!A)
        return fail(SLA_ERR_INVALID_ARG, "NULL handle");
    if (nrhs < 1 || nrhs > KMAX)
        return fail(SLA_ERR_INVALID_ARG, "nrhs must be in [1, 16]");
    if (A->bdim > 1 && nrhs > BSR_KMAX)
        return fail(SLA_ERR_INVALID_ARG, "a BSR matrix takes at most 4 right-hand sides");
    if (A->n > 0 && (!d_X || !d_Y || d_X == d_Y))
        return fail(SLA_ERR_INVALID_ARG, "NULL or overlapping X/Y");
    return launch_spmv(A, nrhs, d_X, d_Y, (cudaStream_t)stream);
}

// ------------------------------------------------------------------ preconditioners
static sla_status jacobi_setup(sla_precond *M, cudaStream_t s)
{
    const sla_csr *A = M->A;
    int *d_err = nullptr;
    SLA_CUDA_TRY(cudaMallocAsync((void **)&d_err, sizeof(int), s));
    SLA_CUDA_TRY(cudaMemsetAsync(d_err, 0, sizeof(int), s));
    sla_status st = launch_jacobi_dinv(A, M->d_dinv64, M->d_dinv, d_err, s);
    int h_err = 0;
    if (st == SLA_SUCCESS) {
        cudaError_t e = cudaMemcpyAsync(&h_err, d_err, sizeof(int), cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess)
            e = cudaStreamSynchronize(s);
        if (e != cudaSuccess)
            st = cuda_fail(e, "Jacobi set-up");
    }
    cudaFreeAsync(d_err, s);
    if (st != SLA_SUCCESS)
        return st;
    if (h_err)
        return fail(SLA_ERR_INVALID_ARG, "Jacobi needs a stored, positive diagonal entry in every row");
    return SLA_SUCCESS;
}

sla_status sla_precond_jacobi(sla_precond **out, const sla_csr *A, void *stream)
{
    if (!out || !A)
        return fail(SLA_ERR_INVALID_ARG, "NULL argument");
    *out = nullptr;
    cudaStream_t s = (cudaStream_t)stream;
    sla_precond *M = new sla_precond();
    M->kind = 1;
    M->A = A;
    const size_t nb = (size_t)std::max<int64_t>(A->n, 1);
    cudaError_t e = cudaMalloc(&M->d_dinv64, nb * sizeof(double));
    if (e == cudaSuccess && A->dtype == SLA_F32)
        e = cudaMalloc(&M->d_dinv, nb * sizeof(float));
    if (e != cudaSuccess) {
        cudaFree(M->d_dinv64);
        delete M;
        return cuda_fail(e, "Jacobi D^-1");
    }
    sla_status st = jacobi_setup(M, s);
    if (st != SLA_SUCCESS) {
        cudaFree(M->d_dinv64);
        if (M->d_dinv)
            cudaFree(M->d_dinv);
        delete M;
        return st;
    }
    const_cast<sla_csr *>(A)->dependents.push_back(M);
    *out = M;
    return SLA_SUCCESS;
}

// G^T on the device (device_transpose: a stable sort of G's entries by column): row j of
// G^T lists the rows i of G holding column j in increasing i.  perm[k] = position in G of
// the k-th entry of G^T, so a later change of G's values is one device gather.  Only G^T's
// row pointers come back to the host (for the row partitions, like every handle's).
static sla_status spai_transpose(sla_precond *M, cudaStream_t s)
{
    const sla_csr *G = M->G;
    const int64_t n = G->n, nnz = G->nnz;
    sla_csr *GT = new sla_csr();
    GT->n = n;
    GT->nnz = nnz;
    GT->dtype = G->dtype;
    GT->device = G->device;
    GT->num_sms = G->num_sms;
    GT->max_sys_n = n;
    M->GT = GT;
    SLA_CUDA_TRY(cudaMalloc((void **)&GT->own_rp, ((size_t)n + 1) * sizeof(int32_t)));
    SLA_CUDA_TRY(cudaMalloc((void **)&GT->own_ci, (size_t)std::max<int64_t>(nnz, 1) * sizeof(int32_t)));
    SLA_CUDA_TRY(cudaMalloc(&GT->own_val, (size_t)std::max<int64_t>(nnz, 1) * vbytes(G->dtype)));
    SLA_CUDA_TRY(cudaMalloc((void **)&M->d_perm, (size_t)std::max<int64_t>(nnz, 1) * sizeof(int32_t)));
    GT->rp = GT->own_rp;
    GT->ci = GT->own_ci;
    GT->val = GT->own_val;
    SLA_TRY(device_transpose(G, GT->own_rp, GT->own_ci, M->d_perm, s));
    GT->h_rp.resize((size_t)n + 1);
    SLA_CUDA_TRY(cudaMemcpyAsync(GT->h_rp.data(), GT->own_rp, ((size_t)n + 1) * sizeof(int32_t),
                                 cudaMemcpyDeviceToHost, s));
    SLA_TRY(refresh_transpose_values(G, GT, M->d_perm, s));
    SLA_CUDA_TRY(cudaStreamSynchronize(s));
    int64_t mx = 0;
    for (int64_t j = 0; j < n; ++j)
        mx = std::max<int64_t>(mx, (int64_t)GT->h_rp[(size_t)j + 1] - GT->h_rp[(size_t)j]);
    GT->max_row_len = mx;
    return SLA_SUCCESS;
}

static void free_precond(sla_precond *M)
{
    if (!M)
        return;
    if (M->A) {
        sla_csr *A = const_cast<sla_csr *>(M->A);
        drop_plans_of(A, M);
        unlink(A->dependents, M);
    }
    if (M->G)
        unlink(const_cast<sla_csr *>(M->G)->dependents, M);
    if (M->d_dinv)
        cudaFree(M->d_dinv);
    if (M->d_dinv64)
        cudaFree(M->d_dinv64);
    if (M->d_perm)
        cudaFree(M->d_perm);
    if (M->GT)
        free_csr(M->GT);
    delete M;
}

sla_status sla_precond_spai(sla_precond **out, const sla_csr *A, const sla_csr *G, double eps,
                            void *stream)
{
    if (!out || !A || !G)
        return fail(SLA_ERR_INVALID_ARG, "NULL argument");
    *out = nullptr;
    if (G->n != A->n || G->dtype != A->dtype)
        return fail(SLA_ERR_INVALID_ARG, "G must match A's size and dtype");
    if (G->bdim > 1)
        return fail(SLA_ERR_INVALID_ARG, "G must be a CSR matrix (A may be BSR)");
    if (!(eps >= 0.0))
        return fail(SLA_ERR_INVALID_ARG, "eps must be >= 0");
    if (A->d_sys_off)       // a list: the list kernel reads G's columns as local indices
        SLA_TRY(check_list_blocks(A, G, (cudaStream_t)stream));
    sla_precond *M = new sla_precond();
    M->kind = 2;
    M->A = A;
    M->G = G;
    M->eps = eps;
    sla_status st = spai_transpose(M, (cudaStream_t)stream);
    if (st != SLA_SUCCESS) {
        M->A = nullptr;
        M->G = nullptr;
        free_precond(M);
        return st;
    }
    const_cast<sla_csr *>(A)->dependents.push_back(M);
    if (G != A)
        const_cast<sla_csr *>(G)->dependents.push_back(M);
    *out = M;
    return SLA_SUCCESS;
}

sla_status sla_precond_refresh(sla_precond *M, void *stream)
{
    if (!M)
        return fail(SLA_ERR_INVALID_ARG, "NULL preconditioner");
    cudaStream_t s = (cudaStream_t)stream;
    if (!M->A || (M->kind == 2 && !M->G))
        return fail(SLA_ERR_INVALID_ARG, "a handle this preconditioner was built from was destroyed");
    if (M->kind == 1)
        return jacobi_setup(M, s);
    SLA_TRY(refresh_transpose_values(M->G, M->GT, M->d_perm, s));
    SLA_CUDA_TRY(cudaStreamSynchronize(s));
    return SLA_SUCCESS;
}

sla_status sla_precond_destroy(sla_precond *M)
{
    free_precond(M);
    return SLA_SUCCESS;
}

// ------------------------------------------------------------------ solves
static sla_status check_solve(const sla_csr *A, const sla_precond *M)
{
    if (!A)
        return fail(SLA_ERR_INVALID_ARG, "NULL matrix handle");
    if (M && M->A != A)
        return fail(SLA_ERR_INVALID_ARG, "the preconditioner was built for another matrix handle");
    if (M && M->kind == 2 && !M->G)
        return fail(SLA_ERR_INVALID_ARG, "the SPAI factor G of this preconditioner was destroyed");
    return SLA_SUCCESS;
}

sla_status sla_pcg_solve(const sla_csr *A, const sla_precond *M, const void *d_b, void *d_x,
                         const sla_pcg_opts *opts, sla_pcg_info *info, void *stream)
{
    SLA_TRY(check_solve(A, M));
    if (A->batch > 1)
        return fail(SLA_ERR_INVALID_ARG, "list handles are solved with sla_pcg_solve_batched");
    if (A->n > 0 && (!d_b || !d_x || d_b == d_x))
        return fail(SLA_ERR_INVALID_ARG, "NULL or overlapping b/x");
    if (A->n == 0) {
        if (info) {
            info->iters = 0;
            info->relres = 0.0;
            info->status = SLA_SUCCESS;
        }
        return SLA_SUCCESS;
    }
    Plan *p = nullptr;
    SLA_TRY(get_plan(const_cast<sla_csr *>(A), M, 1, opts ? opts->vector_f64 : 0, &p));
    return run_plan(const_cast<sla_csr *>(A), p, 1, d_b, d_x, opts, info, nullptr, nullptr,
                    (cudaStream_t)stream);
}

sla_status sla_pcg_adjoint(const sla_csr *A, const sla_precond *M, const void *d_x,
                           const void *d_dLdx, void *d_dLdb, void *d_dLdA,
                           const sla_pcg_opts *opts, sla_pcg_info *info, void *stream)
{
    SLA_TRY(check_solve(A, M));
    if (A->batch > 1)
        return fail(SLA_ERR_INVALID_ARG, "list handles use sla_pcg_adjoint_batched");
    if (A->n > 0 && (!d_x || !d_dLdx || !d_dLdb || d_dLdx == d_dLdb))
        return fail(SLA_ERR_INVALID_ARG, "NULL or overlapping adjoint vectors");
    if (A->n == 0)
        return SLA_SUCCESS;
    Plan *p = nullptr;
    SLA_TRY(get_plan(const_cast<sla_csr *>(A), M, 1, opts ? opts->vector_f64 : 0, &p));
    return run_plan(const_cast<sla_csr *>(A), p, 1, d_dLdx, d_dLdb, opts, info, d_x, d_dLdA,
                    (cudaStream_t)stream);
}

sla_status sla_pcg_solve_batched(const sla_csr *A, const sla_precond *M, int32_t nrhs,
                                 const void *d_B, void *d_X, const sla_pcg_opts *opts,
                                 sla_pcg_info *h_info, void *stream)
{
    SLA_TRY(check_solve(A, M));
    if (!h_info)
        return fail(SLA_ERR_INVALID_ARG, "h_info is required");
    if (A->n > 0 && (!d_B || !d_X || d_B == d_X))
        return fail(SLA_ERR_INVALID_ARG, "NULL or overlapping B/X");
    cudaStream_t s = (cudaStream_t)stream;
    if (A->batch > 1 || A->d_sys_off) {
        if (nrhs != 1)
            return fail(SLA_ERR_INVALID_ARG, "list handles take nrhs = 1");
        return run_list_solve(A, M, d_B, d_X, nullptr, nullptr, opts, h_info, s);
    }
    if (nrhs < 1 || nrhs > KMAX)
        return fail(SLA_ERR_INVALID_ARG, "nrhs must be in [1, 16]");
    if (A->bdim > 1 && nrhs > BSR_KMAX)
        return fail(SLA_ERR_INVALID_ARG, "a BSR matrix takes at most 4 right-hand sides");
    if (A->n == 0) {
        for (int c = 0; c < nrhs; ++c)
            h_info[c] = sla_pcg_info{0, 0.0, SLA_SUCCESS, 0};
        return SLA_SUCCESS;
    }
    int K = 1;
    while (K < nrhs)
        K <<= 1;
    Plan *p = nullptr;
    SLA_TRY(get_plan(const_cast<sla_csr *>(A), M, K, opts ? opts->vector_f64 : 0, &p));
    return run_plan(const_cast<sla_csr *>(A), p, nrhs, d_B, d_X, opts, h_info, nullptr, nullptr,
                    s);
}

sla_status sla_pcg_adjoint_batched(const sla_csr *A, const sla_precond *M, int32_t nrhs,
                                   const void *d_X, const void *d_dLdX, void *d_dLdB,
                                   void *d_dLdA, const sla_pcg_opts *opts, sla_pcg_info *h_info,
                                   void *stream)
{
    SLA_TRY(check_solve(A, M));
    if (!h_info)
        return fail(SLA_ERR_INVALID_ARG, "h_info is required");
    if (A->n > 0 && (!d_X || !d_dLdX || !d_dLdB || d_dLdX == d_dLdB))
        return fail(SLA_ERR_INVALID_ARG, "NULL or overlapping adjoint blocks");
    cudaStream_t s = (cudaStream_t)stream;
    if (A->batch > 1 || A->d_sys_off) {
        if (nrhs != 1)
            return fail(SLA_ERR_INVALID_ARG, "list handles take nrhs = 1");
        return run_list_solve(A, M, d_dLdX, d_dLdB, d_X, d_dLdA, opts, h_info, s);
    }
    if (nrhs < 1 || nrhs > KMAX)
        return fail(SLA_ERR_INVALID_ARG, "nrhs must be in [1, 16]");
    if (A->bdim > 1 && nrhs > BSR_KMAX)
        return fail(SLA_ERR_INVALID_ARG, "a BSR matrix takes at most 4 right-hand sides");
    if (A->n == 0)
        return SLA_SUCCESS;
    int K = 1;
    while (K < nrhs)
        K <<= 1;
    Plan *p = nullptr;
    SLA_TRY(get_plan(const_cast<sla_csr *>(A), M, K, opts ? opts->vector_f64 : 0, &p));
    return run_plan(const_cast<sla_csr *>(A), p, nrhs, d_dLdX, d_dLdB, opts, h_info, d_X, d_dLdA,
                    s);
}

sla_status sla_pattern_grad(const sla_csr *A, int32_t nrhs, const void *d_lam, const void *d_x,
                            void *d_g, void *stream)
{
    if (!A)
        return fail(SLA_ERR_INVALID_ARG, "NULL handle");
    if (nrhs < 1)
        return fail(SLA_ERR_INVALID_ARG, "nrhs must be >= 1");
    if (A->nnz > 0 && (!d_lam || !d_x || !d_g))
        return fail(SLA_ERR_INVALID_ARG, "NULL vector");
    if (A->nnz == 0)
        return SLA_SUCCESS;
    return launch_pattern_grad(A, nrhs, 0, d_lam, d_x, d_g, (cudaStream_t)stream);
}

sla_status sla_pcg_kernel_times(const sla_csr *A, const sla_precond *M, int32_t nrhs,
                                int32_t vector_f64, int32_t reps, double *h_ms, void *stream)
{
    SLA_TRY(check_solve(A, M));
    if (!h_ms || reps < 1)
        return fail(SLA_ERR_INVALID_ARG, "h_ms is required and reps must be >= 1");
    if (A->batch > 1)
        return fail(SLA_ERR_UNSUPPORTED, "kernel timing covers the single-matrix solver");
    if (nrhs < 1 || nrhs > KMAX)
        return fail(SLA_ERR_INVALID_ARG, "nrhs must be in [1, 16]");
    if (A->n == 0)
        return fail(SLA_ERR_INVALID_ARG, "empty matrix");
    int K = 1;
    while (K < nrhs)
        K <<= 1;
    Plan *p = nullptr;
    SLA_TRY(get_plan(const_cast<sla_csr *>(A), M, K, vector_f64, &p));
    return kernel_times(const_cast<sla_csr *>(A), p, nrhs, reps, h_ms, (cudaStream_t)stream);
}

sla_status sla_pcg_phase_times(const sla_csr *A, const sla_precond *M, int32_t nrhs,
                               int32_t vector_f64, double *h_ms, int64_t *h_count, void *stream)
{
    SLA_TRY(check_solve(A, M));
    if (!h_ms || !h_count)
        return fail(SLA_ERR_INVALID_ARG, "h_ms and h_count are required");
    if (A->batch > 1)
        return fail(SLA_ERR_UNSUPPORTED, "phase timing covers the single-matrix solver");
    if (nrhs < 1 || nrhs > KMAX)
        return fail(SLA_ERR_INVALID_ARG, "nrhs must be in [1, 16]");
    int K = 1;
    while (K < nrhs)
        K <<= 1;
    Plan *p = nullptr;
    SLA_TRY(get_plan(const_cast<sla_csr *>(A), M, K, vector_f64, &p));
    cudaStream_t s = (cudaStream_t)stream;
    SLA_CUDA_TRY(cudaMemcpyAsync(p->h_st, p->st, sizeof(PcgState), cudaMemcpyDeviceToHost, s));
    SLA_CUDA_TRY(cudaStreamSynchronize(s));
    if (!p->h_st->persistent)
        return fail(SLA_ERR_INVALID_ARG, "the last solve of this solver did not run on the persistent engine");
    for (int i = 0; i < 4; ++i) {
        h_count[i] = p->h_st->phase_cnt[i];
        h_ms[i] = h_count[i] > 0 ? 1e-6 * (double)p->h_st->phase_ns[i] / (double)h_count[i] : 0.0;
    }
    return SLA_SUCCESS;
}

size_t sla_workspace_bytes(const sla_csr *A, const sla_precond *M, int32_t nrhs, int32_t vector_f64)
{
    if (!A || nrhs < 1 || nrhs > KMAX)
        return 0;
    int K = 1;
    while (K < nrhs)
        K <<= 1;
    return plan_bytes(A, M, K, (vector_f64 && A->dtype == SLA_F32) ? 1 : 0);
}

}  // extern "C"
