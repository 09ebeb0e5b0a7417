// Set-up of the column-sorted row segments (csb.cuh), once per matrix pattern.
//
// Segments (on the host, from the row pointers): contiguous rows with about equal
// (entries + rows), at most CSB_RMAX rows each (CSB_RMAX_F32 for fp32 values; their sums
// live in shared memory) and as few as that allows -- the larger a segment, the closer its
// sorted columns lie -- rounded up to a multiple of the SpMV's grid (one block per SM), so
// that every block takes the same number of segments.
//
// The entries (on the device): every entry gets the key (segment, column, local row), the
// keys are sorted with the radix sort of radix_sort.cuh, and one warp per segment cuts the
// segment's sorted entries into chunks of 32; a chunk also ends early when its next column
// would lie 65536 or more past the chunk's first column (the column offset is 16 bits), and
// the rest of its slots are padding.  A first walk counts each segment's chunks, a second
// writes them.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <memory>
#include <vector>

#include "sla.h"
#include "sla_internal.cuh"
#include "csb.cuh"
#include "radix_sort.cuh"

namespace sla {

namespace {

constexpr int CSB_RB = 14;                      // bits of a local row in the sort key
static_assert(CSB_RMAX <= (1 << CSB_RB), "local rows must fit the key's row field");

// key[k] = (segment << (cb + CSB_RB)) | (column << CSB_RB) | local row, val[k] = k; one warp
// per row, its segment found by binary search over the segments' first rows.
__global__ void k_csb_keys(int64_t n, const int32_t *rp, const int32_t *ci, const int32_t *seg_row0, int nseg,
                           int cb, uint64_t *key, int32_t *val)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; i < n; i += warps) {
        int lo = 0, hi = nseg - 1;              // last segment whose first row is <= i
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (seg_row0[mid] <= i)
                lo = mid;
            else
                hi = mid - 1;
        }
        const uint64_t hi_bits = ((uint64_t)lo << (cb + CSB_RB)) | (uint64_t)(i - seg_row0[lo]);
        for (int64_t k = rp[i] + lane; k < rp[i + 1]; k += 32) {
            key[k] = hi_bits | ((uint64_t)(uint32_t)ci[k] << CSB_RB);
            val[k] = (int32_t)k;
        }
    }
}

// One warp per segment walks its sorted entries chunk by chunk: a chunk takes the next
// entries up to 32 whose column lies within 65535 of the first one (a prefix of the 32 read,
// since the columns ascend).  WRITE = false: chunk counts; true: the chunks themselves,
// from the segment's first chunk ch0[s].
template <bool WRITE>
__global__ void k_csb_chunks(int nseg, const int32_t *seg_row0, const int32_t *rp, const uint64_t *key,
                             const int32_t *val, int cb, int32_t *cnt, const int32_t *ch0, int32_t *cbase,
                             uint32_t *pk, int32_t *perm)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    const uint64_t colmask = (cb >= 32) ? 0xFFFFFFFFull : ((1ull << cb) - 1ull);
    for (int64_t sg = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; sg < nseg; sg += warps) {
        const int64_t e0 = rp[seg_row0[sg]], e1 = rp[seg_row0[sg + 1]];
        const int r_seg = seg_row0[sg + 1] - seg_row0[sg];
        int64_t ch = WRITE ? (int64_t)ch0[sg] : 0;
        for (int64_t pos = e0; pos < e1;) {
            const int64_t t = pos + lane;
            const bool in = t < e1;
            const uint64_t kk = in ? key[t] : 0ull;
            const uint32_t col = (uint32_t)((kk >> CSB_RB) & colmask);
            const uint32_t base = __shfl_sync(0xffffffffu, col, 0);
            const bool ok = in && col - base <= 0xFFFFu;
            const int take = __popc(__ballot_sync(0xffffffffu, ok));
            if (WRITE) {
                const uint32_t lr = (uint32_t)(kk & ((1u << CSB_RB) - 1u));
                pk[ch * 32 + lane] = lane < take ? ((col - base) << 16) | lr : csb_pad_word(lane, r_seg);
                perm[ch * 32 + lane] = lane < take ? val[t] : -1;
                if (lane == 0)
                    cbase[ch] = (int32_t)base;
            }
            ++ch;
            pos += take;
        }
        if (!WRITE && lane == 0)
            cnt[sg] = (int32_t)ch;
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
    cudaFree(A->csb->d_seg_bound);
    cudaFree(A->csb->d_vmax);
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
    const int32_t *rp = A->h_rp.data();
    // segment boundaries: equal shares of (entries + rows), at most RMX rows
    const int64_t total = A->nnz + n;
    const int64_t grid = std::max(1, A->num_sms);
    const int64_t RMX = A->dtype == SLA_F32 ? CSB_RMAX_F32 : CSB_RMAX;
    const int64_t nseg_min = std::max<int64_t>(1, (n + RMX - 1) / RMX);
    int64_t nseg = (nseg_min + grid - 1) / grid * grid;
    // segments of the row budget but with a few rows more than an equal share of the
    // cost would give are still under RMX: allow that much slack before splitting
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
            cut = std::min(cut, r + RMX);
            if (cut >= n)
                break;
            row0.push_back((int32_t)cut);
            r = cut;
        }
        // the last segment may still exceed RMX rows: split it
        while (n - row0.back() > RMX)
            row0.push_back(row0.back() + (int32_t)RMX);
        row0.push_back((int32_t)n);
    }
    nseg = (int64_t)row0.size() - 1;
    int rmax = 0;
    for (int64_t sgi = 0; sgi < nseg; ++sgi)
        rmax = std::max(rmax, row0[(size_t)sgi + 1] - row0[(size_t)sgi]);
    const int cb = std::max(1, bits_for((uint64_t)std::max<int64_t>(n - 1, 0)));
    const int sb = bits_for((uint64_t)(nseg - 1));
    if (sb + cb + CSB_RB > 64)
        return fail(SLA_ERR_UNSUPPORTED, "column-sorted segments: sort key wider than 64 bits");
    const int64_t nnz = A->nnz;
    auto cp = std::make_unique<CsbPart>();
    cp->n_seg = (int)nseg;
    cp->rmax = rmax;
    cudaError_t e = cudaMalloc((void **)&cp->d_seg_row0, sizeof(int32_t) * (size_t)(nseg + 1));
    if (e == cudaSuccess) e = cudaMalloc((void **)&cp->d_seg_ch0, sizeof(int32_t) * (size_t)(nseg + 1));
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(cp->d_seg_row0, row0.data(), sizeof(int32_t) * row0.size(), cudaMemcpyHostToDevice, s);
    // sort (segment, column, local row) keys with the entry positions
    uint64_t *k0 = nullptr, *k1 = nullptr, *ks = nullptr;
    int32_t *v0 = nullptr, *v1 = nullptr, *vs = nullptr, *d_cnt = nullptr;
    const size_t ne = (size_t)std::max<int64_t>(nnz, 1);
    if (e == cudaSuccess) e = cudaMallocAsync((void **)&k0, sizeof(uint64_t) * ne, s);
    if (e == cudaSuccess) e = cudaMallocAsync((void **)&k1, sizeof(uint64_t) * ne, s);
    if (e == cudaSuccess) e = cudaMallocAsync((void **)&v0, sizeof(int32_t) * ne, s);
    if (e == cudaSuccess) e = cudaMallocAsync((void **)&v1, sizeof(int32_t) * ne, s);
    if (e == cudaSuccess) e = cudaMallocAsync((void **)&d_cnt, sizeof(int32_t) * (size_t)nseg, s);
    const int rgrid = (int)std::max<int64_t>(1, std::min<int64_t>((n + 7) / 8, (int64_t)A->num_sms * 16));
    const int sgrid = (int)std::max<int64_t>(1, (nseg + 7) / 8);
    if (e == cudaSuccess && n > 0) {
        k_csb_keys<<<rgrid, 256, 0, s>>>(n, A->rp, A->ci, cp->d_seg_row0, (int)nseg, cb, k0, v0);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess)
        e = radix_sort_pairs<uint64_t>(k0, v0, k1, v1, nnz, sb + cb + CSB_RB, &ks, &vs, s);
    if (e == cudaSuccess) {
        k_csb_chunks<false><<<sgrid, 256, 0, s>>>((int)nseg, cp->d_seg_row0, A->rp, ks, vs, cb, d_cnt, nullptr,
                                                  nullptr, nullptr, nullptr);
        e = cudaGetLastError();
    }
    std::vector<int32_t> cnt((size_t)nseg);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(cnt.data(), d_cnt, sizeof(int32_t) * (size_t)nseg, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(s);
    std::vector<int32_t> ch0((size_t)nseg + 1, 0);
    for (int64_t sgi = 0; sgi < nseg; ++sgi)
        ch0[(size_t)sgi + 1] = ch0[(size_t)sgi] + cnt[(size_t)sgi];
    const int64_t nch = ch0.back();
    cp->n_chunks = nch;
    const size_t vb = A->dtype == SLA_F32 ? 4 : 8;
    const size_t nc = (size_t)std::max<int64_t>(nch, 1);
    if (e == cudaSuccess) e = cudaMalloc((void **)&cp->d_cbase, sizeof(int32_t) * nc);
    if (e == cudaSuccess) e = cudaMalloc((void **)&cp->d_pk, sizeof(uint32_t) * 32 * nc);
    if (e == cudaSuccess) e = cudaMalloc((void **)&cp->d_perm, sizeof(int32_t) * 32 * nc);
    if (e == cudaSuccess) e = cudaMalloc(&cp->d_val, vb * 32 * nc);
    // fixed-point row sums: per-segment bounds (with the values), operand maxima, low-word
    // bits such that the longest row's low words cannot carry out of 32 bits
    cp->vmax_n = std::max(1, A->num_sms);
    cp->lb = std::max(1, std::min(20, 32 - bits_for((uint64_t)std::max<int64_t>(A->max_row_len, 0))));
    if (e == cudaSuccess) e = cudaMalloc((void **)&cp->d_seg_bound, sizeof(double) * (size_t)std::max<int64_t>(nseg, 1));
    if (e == cudaSuccess) e = cudaMalloc((void **)&cp->d_vmax, sizeof(float) * (size_t)cp->vmax_n);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(cp->d_seg_bound, 0, sizeof(double) * (size_t)std::max<int64_t>(nseg, 1), s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(cp->d_seg_ch0, ch0.data(), sizeof(int32_t) * ch0.size(), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && nch > 0) {
        k_csb_chunks<true><<<sgrid, 256, 0, s>>>((int)nseg, cp->d_seg_row0, A->rp, ks, vs, cb, nullptr,
                                                 cp->d_seg_ch0, cp->d_cbase, cp->d_pk, cp->d_perm);
        e = cudaGetLastError();
    }
    for (void *p : {(void *)k0, (void *)k1, (void *)v0, (void *)v1, (void *)d_cnt})
        if (p)
            cudaFreeAsync(p, s);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
        A->csb = cp.release();
        free_csb(A);
        return cuda_fail(e, "column-sorted segments: device build");
    }
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
    if (A->dtype == SLA_F32) {
        k_csb_values<float><<<grid, 256, 0, s>>>(slots, cp->d_perm, (const float *)A->val, (float *)cp->d_val);
        k_csb_bounds<float><<<cp->n_seg, CSB_BND_T, 0, s>>>(cp->n_seg, cp->d_seg_row0, A->rp, (const float *)A->val,
                                                      cp->d_seg_bound);
    } else {
        k_csb_values<double><<<grid, 256, 0, s>>>(slots, cp->d_perm, (const double *)A->val, (double *)cp->d_val);
        k_csb_bounds<double><<<cp->n_seg, CSB_BND_T, 0, s>>>(cp->n_seg, cp->d_seg_row0, A->rp, (const double *)A->val,
                                                       cp->d_seg_bound);
    }
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
