// PCG solver instantiations for float matrix values with double vectors.
#include "pcg_impl.cuh"

namespace sla {

#define SLA_DISPATCH_K(K_, FN, ...)                                                    \
    switch (K_) {                                                                      \
    case 1: return FN<float, double, 1>(__VA_ARGS__);                                      \
    case 2: return FN<float, double, 2>(__VA_ARGS__);                                      \
    case 4: return FN<float, double, 4>(__VA_ARGS__);                                      \
    case 8: return FN<float, double, 8>(__VA_ARGS__);                                      \
    case 16: return FN<float, double, 16>(__VA_ARGS__);                                    \
    default: return fail(SLA_ERR_INVALID_ARG, "unsupported right-hand-side count");    \
    }

sla_status capture_fd(sla_csr *A, Plan *p) { SLA_DISPATCH_K(p->K, capture_k, A, p) }

sla_status times_fd(sla_csr *A, Plan *p, int nrhs, int reps, double *h_ms, cudaStream_t s)
{
    SLA_DISPATCH_K(p->K, times_k, A, p, nrhs, reps, h_ms, s)
}

sla_status run_fd(sla_csr *A, Plan *p, int nrhs, const void *B, void *X, double tol, long long maxit,
                      int engine, cudaStream_t s)
{
    SLA_DISPATCH_K(p->K, run_k, A, p, nrhs, B, X, tol, maxit, engine, s)
}

sla_status grad_fd(const sla_csr *A, int nrhs, const void *lam, const void *x, void *g, double scale,
                   cudaStream_t s)
{
    return grad_v<float, double>(A, nrhs, lam, x, g, scale, s);
}

}  // namespace sla
