// Batched list solve that allocates nothing.
//
// Some callers cannot allocate device memory while they solve: code running under a
// memory pool or budget that owns every byte on the device, embedded hosts that forbid
// runtime allocation after start-up, or code that must not pay the synchronisation an
// allocation or free can imply.  The regular list solve takes a small device buffer for the
// per-system results from the stream-ordered allocator on every call; this entry point
// writes them into a fixed array in this library's own device memory instead.
//
// The array is a file-scope __device__ array of NOALLOC_MAX_SYSTEMS results (1.5 MiB); every
// GPU that loads the library holds it until the process exits.  Host code only holds a
// stand-in for its name, so every call looks its device address up with
// cudaGetSymbolAddress on the current device.  The address is not cached: a context that is
// torn down and created again (cudaDeviceReset) can place the array elsewhere.  Every call
// on a device shares the array: calls that overlap on the GPU (different streams, or
// different host threads) race on it and must be serialised by the caller.
#include <cuda_runtime.h>

#include <algorithm>

#include "sla.h"
#include "sla_internal.cuh"

namespace sla {

sla_status launch_list_kernel(const sla_csr *A, const sla_precond *M, const void *B, void *X,
                              const sla_pcg_opts *opts, sla_pcg_info *d_info, cudaStream_t s);

namespace {

constexpr int NOALLOC_MAX_SYSTEMS = 65536;
static __device__ __align__(256) sla_pcg_info g_noalloc_info[NOALLOC_MAX_SYSTEMS];

// Device address of g_noalloc_info in the current device's context (a host-side lookup).
sla_status noalloc_scratch(sla_pcg_info **out)
{
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_info);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetSymbolAddress of the fixed result array");
    *out = (sla_pcg_info *)p;
    return SLA_SUCCESS;
}

}  // namespace
}  // namespace sla

using namespace sla;

extern "C" sla_status sla_pcg_solve_batched_noalloc(const sla_csr *A, const sla_precond *M, const void *d_B,
                                                    void *d_X, const sla_pcg_opts *opts,
                                                    sla_pcg_info *h_info, void *stream)
{
    if (!A)
        return fail(SLA_ERR_INVALID_ARG, "NULL matrix handle");
    if (!A->d_sys_off)
        return fail(SLA_ERR_INVALID_ARG, "the no-allocation solve takes a list handle (sla_csr_create_list)");
    if (M && M->A != A)
        return fail(SLA_ERR_INVALID_ARG, "the preconditioner was built for another matrix handle");
    if (!h_info)
        return fail(SLA_ERR_INVALID_ARG, "h_info is required");
    if (A->n > 0 && (!d_B || !d_X || d_B == d_X))
        return fail(SLA_ERR_INVALID_ARG, "NULL or overlapping B/X");
    if (A->batch > NOALLOC_MAX_SYSTEMS)
        return fail(SLA_ERR_INVALID_ARG, "the no-allocation solve handles at most 65536 systems per call");
    cudaStream_t s = (cudaStream_t)stream;
    sla_pcg_info *d_info = nullptr;
    SLA_TRY(noalloc_scratch(&d_info));
    // the array keeps the previous call's results: fill this call's slots with a value that
    // is no solver outcome (status -1), so a slot the kernel left unwritten cannot pass for
    // a converged solve
    SLA_CUDA_TRY(cudaMemsetAsync(d_info, 0xFF, sizeof(sla_pcg_info) * (size_t)A->batch, s));
    SLA_TRY(launch_list_kernel(A, M, d_B, d_X, opts, d_info, s));
    SLA_CUDA_TRY(cudaMemcpyAsync(h_info, d_info, sizeof(sla_pcg_info) * (size_t)A->batch,
                                 cudaMemcpyDeviceToHost, s));
    SLA_CUDA_TRY(cudaStreamSynchronize(s));
    sla_status worst = SLA_SUCCESS;
    for (int i = 0; i < A->batch; ++i) {
        if (h_info[i].status < 0)
            return fail(SLA_ERR_CUDA, "the list solve left a system's result unwritten");
        worst = std::max(worst, (sla_status)h_info[i].status);
    }
    return worst;
}
