// PCG solver instantiations for double matrix values with double vectors.
#include "pcg_impl.cuh"

namespace sla {

#define SLA_DISPATCH_K(K_, FN, ...)                                                    \
    switch (K_) {                                                                      \
    case 1: return FN<double, double, 1>(__VA_ARGS__);                                      \
    case 2: return FN<double, double, 2>(__VA_ARGS__);                                      \
    case 4: return FN<double, double, 4>(__VA_ARGS__);                                      \
    case 8: return FN<double, double, 8>(__VA_ARGS__);                                      \
    case 16: return FN<double, double, 16>(__VA_ARGS__);                                    \
    default: return fail(SLA_ERR_INVALID_ARG, "unsupported right-hand-side count");    \
    }

sla_status capture_dd(sla_csr *A, Plan *p) { SLA_DISPATCH_K(p->K, capture_k, A, p) }

sla_status times_dd(sla_csr *A, Plan *p, int nrhs, int reps, double *h_ms, cudaStream_t s)
{
    SLA_DISPATCH_K(p->K, times_k, A, p, nrhs, reps, h_ms, s)
}

sla_status run_dd(sla_csr *A, Plan *p, int nrhs, const void *B, void *X, double tol, long long maxit,
                      int engine, cudaStream_t s)
{
    SLA_DISPATCH_K(p->K, run_k, A, p, nrhs, B, X, tol, maxit, engine, s)
}

sla_status grad_dd(const sla_csr *A, int nrhs, const void *lam, const void *x, void *g, double scale,
                   cudaStream_t s)
{
    return grad_v<double, double>(A, nrhs, lam, x, g, scale, s);
}

static int pad_k(int nrhs)
{
    int K = 1;
    while (K < nrhs)
        K <<= 1;
    return K;
}

sla_status spmv_dd(const sla_csr *A, int nrhs, const void *x, void *y, cudaStream_t s)
{
    switch (pad_k(nrhs)) {
    case 1: return spmv_k<double, 1>(A, nrhs, x, y, s);
    case 2: return spmv_k<double, 2>(A, nrhs, x, y, s);
    case 4: return spmv_k<double, 4>(A, nrhs, x, y, s);
    case 8: return spmv_k<double, 8>(A, nrhs, x, y, s);
    case 16: return spmv_k<double, 16>(A, nrhs, x, y, s);
    default: return fail(SLA_ERR_INVALID_ARG, "nrhs must be in [1, 16]");
    }
}

}  // namespace sla
