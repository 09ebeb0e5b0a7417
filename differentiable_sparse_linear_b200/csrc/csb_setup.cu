// Set-up of the column-sorted row segments (csb.cuh) on the host, once per matrix pattern.
//
// Segments: contiguous rows with about equal (entries + rows), at most CSB_RMAX rows each
// (their sums live in shared memory) and as few as that allows -- the larger a segment, the
// closer its sorted columns lie -- rounded up to a multiple of the SpMV's grid (one block
// per SM), so that every block takes the same number of segments.  Each segment's
// entries are sorted by (column, row) -- the segments are independent and are sorted on all
// host threads -- and cut into chunks of 32; a chunk also ends early when its next column
// would lie 65536 or more past the chunk's first column (the column offset is 16 bits), and
// the rest of its slots are padding.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <memory>
#include <thread>
#include <vector>

#include "sla.h"
#include "sla_internal.cuh"
#include "csb.cuh"

namespace sla {

namespace {


struct SegOut {
    std::vector<int32_t> cbase;
    std::vector<uint32_t> pk;
    std::vector<int32_t> perm;
};

// Sort one segment's entries by (column, row) and cut them into chunks.
void build_segment(const int32_t *rp, const int32_t *ci, int64_t r0, int64_t r1, SegOut &o)
{
    const int64_t k0 = rp[r0], k1 = rp[r1];
    std::vector<uint64_t> key((size_t)(k1 - k0));
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t k = rp[r]; k < rp[r + 1]; ++k)   // column in the high bits, local row below
            key[(size_t)(k - k0)] = ((uint64_t)(uint32_t)ci[k] << 32) | (uint64_t)(uint32_t)(r - r0);
    // (column, row) pairs are distinct, so the order is unique
    std::vector<int64_t> pos((size_t)(k1 - k0));
    for (size_t i = 0; i < pos.size(); ++i)
        pos[i] = (int64_t)i;
    std::sort(pos.begin(), pos.end(), [&](int64_t a, int64_t b) { return key[(size_t)a] < key[(size_t)b]; });
    o.cbase.clear();
    o.pk.clear();
    o.perm.clear();
    size_t i = 0;
    while (i < pos.size()) {
        const int64_t first = pos[i];
        const uint32_t base = (uint32_t)(key[(size_t)first] >> 32);
        o.cbase.push_back((int32_t)base);
        int l = 0;
        for (; l < 32 && i < pos.size(); ++l) {
            const int64_t e = pos[i];
            const uint32_t col = (uint32_t)(key[(size_t)e] >> 32);
            if (col - base > 0xFFFFu)
                break;
            const uint32_t row = (uint32_t)(key[(size_t)e] & 0xFFFFFFFFu);
            o.pk.push_back(((col - base) << 16) | row);
            o.perm.push_back((int32_t)(k0 + e));
            ++i;
        }
        for (; l < 32; ++l) {
            o.pk.push_back(CSB_PAD);
            o.perm.push_back(-1);
        }
    }
}

}  // namespace

void free_csb(sla_csr *A)
{
    if (!A->csb)
        return;
    cudaFree(A->csb->d_seg_row0);
    cudaFree(A->csb->d_seg_ch0);
    cudaFree(A->csb->d_cbase);
    cudaFree(A->csb->d_pk);
    cudaFree(A->csb->d_perm);
    cudaFree(A->csb->d_val);
    delete A->csb;
    A->csb = nullptr;
}

sla_status ensure_csb(sla_csr *A, cudaStream_t s, const CsbPart **out)
{
    if (A->csb) {
        *out = A->csb;
        return SLA_SUCCESS;
    }
    if (A->bdim != 1 || A->n > 0x7FFFFFFF || A->nnz >= ((int64_t)1 << 31))
        return fail(SLA_ERR_UNSUPPORTED, "column-sorted segments: CSR matrices with int32 sizes only");
    const int64_t n = A->n;
    std::vector<int32_t> h_ci((size_t)A->nnz);
    if (A->nnz > 0) {
        SLA_CUDA_TRY(cudaMemcpyAsync(h_ci.data(), A->ci, (size_t)A->nnz * sizeof(int32_t), cudaMemcpyDeviceToHost, s));
        SLA_CUDA_TRY(cudaStreamSynchronize(s));
    }
    const int32_t *rp = A->h_rp.data();
    // segment boundaries: equal shares of (entries + rows), at most CSB_RMAX rows
    const int64_t total = A->nnz + n;
    const int64_t grid = std::max(1, A->num_sms);
    const int64_t nseg_min = std::max<int64_t>(1, (n + CSB_RMAX - 1) / CSB_RMAX);
    int64_t nseg = (nseg_min + grid - 1) / grid * grid;
    // segments of the row budget but with a few rows more than an equal share of the
    // cost would give are still under CSB_RMAX: allow that much slack before splitting
    nseg = std::min<int64_t>(nseg, std::max<int64_t>(1, n));
    std::vector<int32_t> row0;
    row0.push_back(0);
    {
        int64_t r = 0;
        for (int64_t sgi = 1; sgi < nseg && r < n; ++sgi) {
            const int64_t target = total * sgi / nseg;
            int64_t lo = r, hi = n;          // first row whose prefix cost reaches the target
            while (lo < hi) {
                const int64_t mid = (lo + hi) / 2;
                if ((int64_t)rp[mid] + mid < target)
                    lo = mid + 1;
                else
                    hi = mid;
            }
            int64_t cut = std::max(lo, r + 1);
            cut = std::min(cut, r + (int64_t)CSB_RMAX);
            if (cut >= n)
                break;
            row0.push_back((int32_t)cut);
            r = cut;
        }
        // the last segment may still exceed CSB_RMAX rows: split it
        while (n - row0.back() > CSB_RMAX)
            row0.push_back(row0.back() + CSB_RMAX);
        row0.push_back((int32_t)n);
    }
    nseg = (int64_t)row0.size() - 1;
    std::vector<SegOut> segs((size_t)nseg);
    const unsigned hw = std::max(1u, std::thread::hardware_concurrency());
    const unsigned nth = (unsigned)std::min<int64_t>(hw, nseg);
    {
        std::vector<std::thread> th;
        for (unsigned t = 0; t < nth; ++t)
            th.emplace_back([&, t] {
                for (int64_t sgi = t; sgi < nseg; sgi += nth)
                    build_segment(rp, h_ci.data(), row0[(size_t)sgi], row0[(size_t)sgi + 1], segs[(size_t)sgi]);
            });
        for (auto &x : th)
            x.join();
    }
    std::vector<int32_t> ch0((size_t)nseg + 1, 0);
    int rmax = 0;
    for (int64_t sgi = 0; sgi < nseg; ++sgi) {
        ch0[(size_t)sgi + 1] = ch0[(size_t)sgi] + (int32_t)segs[(size_t)sgi].cbase.size();
        rmax = std::max(rmax, row0[(size_t)sgi + 1] - row0[(size_t)sgi]);
    }
    const int64_t nch = ch0.back();
    auto cp = std::make_unique<CsbPart>();
    cp->n_seg = (int)nseg;
    cp->rmax = rmax;
    cp->n_chunks = nch;
    const size_t vb = A->dtype == SLA_F32 ? 4 : 8;
    auto fail_free = [&](cudaError_t e) {
        A->csb = cp.release();
        free_csb(A);
        return cuda_fail(e, "column-sorted segments: device allocation");
    };
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess) e = cudaMalloc((void **)&cp->d_seg_row0, sizeof(int32_t) * (size_t)(nseg + 1));
    if (e == cudaSuccess) e = cudaMalloc((void **)&cp->d_seg_ch0, sizeof(int32_t) * (size_t)(nseg + 1));
    if (e == cudaSuccess) e = cudaMalloc((void **)&cp->d_cbase, sizeof(int32_t) * (size_t)std::max<int64_t>(nch, 1));
    if (e == cudaSuccess) e = cudaMalloc((void **)&cp->d_pk, sizeof(uint32_t) * 32 * (size_t)std::max<int64_t>(nch, 1));
    if (e == cudaSuccess) e = cudaMalloc((void **)&cp->d_perm, sizeof(int32_t) * 32 * (size_t)std::max<int64_t>(nch, 1));
    if (e == cudaSuccess) e = cudaMalloc(&cp->d_val, vb * 32 * (size_t)std::max<int64_t>(nch, 1));
    if (e != cudaSuccess)
        return fail_free(e);
    // gather the per-segment pieces into whole host arrays, then one copy each
    std::vector<int32_t> cb((size_t)nch);
    std::vector<uint32_t> pk((size_t)nch * 32);
    std::vector<int32_t> perm((size_t)nch * 32);
    for (int64_t sgi = 0; sgi < nseg; ++sgi) {
        const SegOut &o = segs[(size_t)sgi];
        const size_t c0 = (size_t)ch0[(size_t)sgi];
        if (!o.cbase.empty()) {
            std::memcpy(&cb[c0], o.cbase.data(), o.cbase.size() * sizeof(int32_t));
            std::memcpy(&pk[c0 * 32], o.pk.data(), o.pk.size() * sizeof(uint32_t));
            std::memcpy(&perm[c0 * 32], o.perm.data(), o.perm.size() * sizeof(int32_t));
        }
    }
    segs.clear();
    e = cudaMemcpyAsync(cp->d_seg_row0, row0.data(), sizeof(int32_t) * row0.size(), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(cp->d_seg_ch0, ch0.data(), sizeof(int32_t) * ch0.size(), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && nch) e = cudaMemcpyAsync(cp->d_cbase, cb.data(), sizeof(int32_t) * cb.size(), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && nch) e = cudaMemcpyAsync(cp->d_pk, pk.data(), sizeof(uint32_t) * pk.size(), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && nch) e = cudaMemcpyAsync(cp->d_perm, perm.data(), sizeof(int32_t) * perm.size(), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess)
        return fail_free(e);
    A->csb = cp.release();
    A->csb_vals_current = 0;
    *out = A->csb;
    return SLA_SUCCESS;
}

sla_status launch_csb_values(const sla_csr *A, cudaStream_t s)
{
    const CsbPart *cp = A->csb;
    if (!cp || cp->n_chunks == 0)
        return SLA_SUCCESS;
    const int64_t slots = cp->n_chunks * 32;
    const int grid = (int)std::min<int64_t>((slots + 255) / 256, (int64_t)A->num_sms * 16);
    if (A->dtype == SLA_F32)
        k_csb_values<float><<<grid, 256, 0, s>>>(slots, cp->d_perm, (const float *)A->val, (float *)cp->d_val);
    else
        k_csb_values<double><<<grid, 256, 0, s>>>(slots, cp->d_perm, (const double *)A->val, (double *)cp->d_val);
    SLA_CUDA_TRY(cudaGetLastError());
    const_cast<sla_csr *>(A)->csb_vals_current = 1;
    return SLA_SUCCESS;
}

}  // namespace sla

using namespace sla;

extern "C" sla_status sla_csr_values_changed(sla_csr *A, void *stream)
{
    (void)stream;
    if (!A)
        return fail(SLA_ERR_INVALID_ARG, "NULL handle");
    A->csb_vals_current = 0;
    A->sell_vals_current = 0;
    return SLA_SUCCESS;
}
