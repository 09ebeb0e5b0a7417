// Stable least-significant-digit radix sort of (key, int32 value) pairs on the device, and an
// exclusive prefix sum: the set-up steps that reorder a matrix pattern (the explicit G^T of
// the SPAI preconditioner, the column-sorted row segments) without a round trip through
// host memory.
//
// One pass per 8-bit digit, three launches each:
//   1. k_rs_hist: every tile of RS_TILE items counts its digits (shared-memory counters) and
//      writes them digit-major: hist[d * tiles + tile].
//   2. an exclusive prefix sum over hist: offs[d * tiles + tile] = items with a smaller digit
//      anywhere + items with digit d in earlier tiles, i.e. the first output slot of that
//      tile's digit-d items.
//   3. k_rs_scatter: the tile's items are split among its warps in order (warp w takes the
//      w-th run of RS_WARP_ITEMS); a first walk counts each warp's digits, the counts become
//      per-warp starting slots (tile offset + earlier warps' counts), and a second walk in the
//      same order places every item at its warp's slot for its digit + its rank among the
//      lanes of its round that share the digit (__match_any_sync).  Items keep their input
//      order among equal digits, so the sort is stable and its output is unique.
// Counts and slots are 32-bit: at most 2^32 - 1 items.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <utility>

namespace sla {

constexpr int RS_BITS = 8;
constexpr int RS_DIGITS = 1 << RS_BITS;
constexpr int RS_T = 256;                          // threads per block
constexpr int RS_TILE = 4096;                      // items per block
constexpr int RS_WARPS = RS_T / 32;
constexpr int RS_WARP_ITEMS = RS_TILE / RS_WARPS;  // items per warp, in rounds of 32

template <typename K>
__global__ void __launch_bounds__(RS_T) k_rs_hist(const K *keys, int64_t n, int shift, uint32_t *hist,
                                                  int64_t tiles)
{
    __shared__ uint32_t cnt[RS_DIGITS];
    for (int d = threadIdx.x; d < RS_DIGITS; d += RS_T)
        cnt[d] = 0;
    __syncthreads();
    const int64_t t0 = (int64_t)blockIdx.x * RS_TILE;
    const int64_t t1 = n < t0 + RS_TILE ? n : t0 + RS_TILE;
    for (int64_t t = t0 + threadIdx.x; t < t1; t += RS_T)
        atomicAdd(&cnt[(uint32_t)(keys[t] >> shift) & (RS_DIGITS - 1)], 1u);
    __syncthreads();
    for (int d = threadIdx.x; d < RS_DIGITS; d += RS_T)
        hist[(int64_t)d * tiles + blockIdx.x] = cnt[d];
}

template <typename K>
__global__ void __launch_bounds__(RS_T) k_rs_scatter(const K *kin, const int32_t *vin, K *kout, int32_t *vout,
                                                     int64_t n, int shift, const uint32_t *offs, int64_t tiles)
{
    __shared__ uint32_t wc[RS_WARPS][RS_DIGITS];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < RS_WARPS * RS_DIGITS; i += RS_T)
        (&wc[0][0])[i] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * RS_TILE + (int64_t)w * RS_WARP_ITEMS;
    const uint32_t lower = (1u << lane) - 1u;     // lanes below this one
    // this warp's count of each digit (RS_DIGITS marks a slot past the end)
    for (int r = 0; r < RS_WARP_ITEMS / 32; ++r) {
        const int64_t t = base + r * 32 + lane;
        const uint32_t d = t < n ? (uint32_t)(kin[t] >> shift) & (RS_DIGITS - 1) : (uint32_t)RS_DIGITS;
        const uint32_t peers = __match_any_sync(0xffffffffu, d);
        if (d < RS_DIGITS && (peers & lower) == 0)
            wc[w][d] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // per-warp first slots: the tile's offset for the digit, then the earlier warps' counts
    for (int d = threadIdx.x; d < RS_DIGITS; d += RS_T) {
        uint32_t run = offs[(int64_t)d * tiles + blockIdx.x];
        for (int j = 0; j < RS_WARPS; ++j) {
            const uint32_t c = wc[j][d];
            wc[j][d] = run;
            run += c;
        }
    }
    __syncthreads();
    for (int r = 0; r < RS_WARP_ITEMS / 32; ++r) {
        const int64_t t = base + r * 32 + lane;
        K k = 0;
        int32_t v = 0;
        uint32_t d = RS_DIGITS;
        if (t < n) {
            k = kin[t];
            v = vin[t];
            d = (uint32_t)(k >> shift) & (RS_DIGITS - 1);
        }
        const uint32_t peers = __match_any_sync(0xffffffffu, d);
        if (d < RS_DIGITS) {
            const uint32_t pos = wc[w][d] + __popc(peers & lower);
            kout[pos] = k;
            vout[pos] = v;
        }
        __syncwarp();
        if (d < RS_DIGITS && (peers & lower) == 0)
            wc[w][d] += __popc(peers);
        __syncwarp();
    }
}

// Exclusive prefix sum in place, tiles of SC_TILE values: each tile is scanned by one block
// and its total goes to sums[tile]; the totals are scanned the same way (recursively) and
// added back.
constexpr int SC_T = 1024;
constexpr int SC_ITEMS = 4;
constexpr int SC_TILE = SC_T * SC_ITEMS;

static __global__ void __launch_bounds__(SC_T) k_scan_tiles(uint32_t *a, int64_t len, uint32_t *sums)
{
    __shared__ uint32_t s_w[SC_T / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t t0 = (int64_t)blockIdx.x * SC_TILE + (int64_t)threadIdx.x * SC_ITEMS;
    uint32_t v[SC_ITEMS], tot = 0;
#pragma unroll
    for (int i = 0; i < SC_ITEMS; ++i) {
        v[i] = t0 + i < len ? a[t0 + i] : 0u;
        tot += v[i];
    }
    uint32_t x = tot;                              // inclusive scan of the threads' totals
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off)
            x += y;
    }
    if (lane == 31)
        s_w[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t y = s_w[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t z = __shfl_up_sync(0xffffffffu, y, off);
            if (lane >= off)
                y += z;
        }
        s_w[lane] = y;
    }
    __syncthreads();
    uint32_t run = x - tot + (warp > 0 ? s_w[warp - 1] : 0u);
#pragma unroll
    for (int i = 0; i < SC_ITEMS; ++i) {
        if (t0 + i < len)
            a[t0 + i] = run;
        run += v[i];
    }
    if (threadIdx.x == 0 && sums)
        sums[blockIdx.x] = s_w[SC_T / 32 - 1];
}

static __global__ void __launch_bounds__(SC_T) k_scan_add(uint32_t *a, int64_t len, const uint32_t *sums)
{
    const int64_t t0 = (int64_t)blockIdx.x * SC_TILE + (int64_t)threadIdx.x * SC_ITEMS;
    const uint32_t add = sums[blockIdx.x];
#pragma unroll
    for (int i = 0; i < SC_ITEMS; ++i)
        if (t0 + i < len)
            a[t0 + i] += add;
}

inline cudaError_t scan_exclusive(uint32_t *a, int64_t len, cudaStream_t s)
{
    if (len <= 0)
        return cudaSuccess;
    const int64_t nt = (len + SC_TILE - 1) / SC_TILE;
    if (nt == 1) {
        k_scan_tiles<<<1, SC_T, 0, s>>>(a, len, nullptr);
        return cudaGetLastError();
    }
    uint32_t *sums = nullptr;
    cudaError_t e = cudaMallocAsync((void **)&sums, sizeof(uint32_t) * (size_t)nt, s);
    if (e != cudaSuccess)
        return e;
    k_scan_tiles<<<(unsigned)nt, SC_T, 0, s>>>(a, len, sums);
    e = cudaGetLastError();
    if (e == cudaSuccess)
        e = scan_exclusive(sums, nt, s);
    if (e == cudaSuccess) {
        k_scan_add<<<(unsigned)nt, SC_T, 0, s>>>(a, len, sums);
        e = cudaGetLastError();
    }
    cudaFreeAsync(sums, s);
    return e;
}

// Sort n pairs by bits [0, end_bit) of their keys.  (k0, v0) hold the input; (k1, v1) are
// scratch of the same sizes.  On return *out_k / *out_v point to whichever pair of buffers
// holds the sorted result.
template <typename K>
cudaError_t radix_sort_pairs(K *k0, int32_t *v0, K *k1, int32_t *v1, int64_t n, int end_bit, K **out_k,
                             int32_t **out_v, cudaStream_t s)
{
    *out_k = k0;
    *out_v = v0;
    if (n <= 0 || end_bit <= 0)
        return cudaSuccess;
    if (n > (int64_t)0xFFFFFFFF)
        return cudaErrorInvalidValue;
    const int64_t tiles = (n + RS_TILE - 1) / RS_TILE;
    uint32_t *hist = nullptr;
    cudaError_t e = cudaMallocAsync((void **)&hist, sizeof(uint32_t) * (size_t)(tiles * RS_DIGITS), s);
    if (e != cudaSuccess)
        return e;
    K *ki = k0, *ko = k1;
    int32_t *vi = v0, *vo = v1;
    for (int shift = 0; shift < end_bit && e == cudaSuccess; shift += RS_BITS) {
        k_rs_hist<K><<<(unsigned)tiles, RS_T, 0, s>>>(ki, n, shift, hist, tiles);
        e = cudaGetLastError();
        if (e == cudaSuccess)
            e = scan_exclusive(hist, tiles * RS_DIGITS, s);
        if (e == cudaSuccess) {
            k_rs_scatter<K><<<(unsigned)tiles, RS_T, 0, s>>>(ki, vi, ko, vo, n, shift, hist, tiles);
            e = cudaGetLastError();
        }
        std::swap(ki, ko);
        std::swap(vi, vo);
    }
    cudaFreeAsync(hist, s);
    *out_k = ki;
    *out_v = vi;
    return e;
}

// Number of bits needed to hold values 0 .. v.
inline int bits_for(uint64_t v)
{
    int b = 0;
    while (b < 64 && (v >> b) != 0)
        ++b;
    return b;
}

}  // namespace sla
