// Internal declarations of libsla: handles, device solver state, launch helpers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <map>
#include <string>
#include <vector>

#include "sla.h"

namespace sla {

// ------------------------------------------------------------------ error reporting
void set_error(const std::string &msg);
sla_status fail(sla_status code, const std::string &msg);
sla_status cuda_fail(cudaError_t e, const char *what);

#define SLA_CUDA_TRY(expr)                                                   \
    do {                                                                     \
        cudaError_t _e = (expr);                                             \
        if (_e != cudaSuccess) return ::sla::cuda_fail(_e, #expr);           \
    } while (0)

#define SLA_TRY(expr)                                                        \
    do {                                                                     \
        sla_status _s = (expr);                                              \
        if (_s != SLA_SUCCESS) return _s;                                    \
    } while (0)

// ------------------------------------------------------------------ limits
constexpr int KMAX = 16;            // right-hand sides handled by one solve
constexpr int BSR_KMAX = 4;         // ... with a BSR matrix
constexpr int NPMAX = 2;            // dot products one kernel reduces per right-hand side

// ------------------------------------------------------------------ device solver state
// One per solve plan.  Scalars of the recurrence (fp64), per right-hand side, plus the
// loop control the device reads: `active` per RHS, `all_done`, and the last-block ticket.
struct PcgState {
    double rho[KMAX];
    double alpha[KMAX];
    double beta[KMAX];
    double bnorm[KMAX];
    double relres[KMAX];
    long long iters[KMAX];
    int status[KMAX];
    int active[KMAX];
    int all_done;
    int phase0;             // 1 while the initial (k = 0) pass runs
    unsigned int ticket;    // completed-block counter of the running reduction kernel
    int k;                  // number of RHS slots in use (<= KMAX)
    double tol;
    long long maxit;
    double eps;             // SPAI shift
    unsigned long long cond_handle;   // cudaGraphConditionalHandle of the solve loop
    int has_cond;
    int profile;            // 1: kernels run for timing only; finalisation is skipped
    int error;              // nonzero: a pipeline wait ran out of time (results invalid)
    int vec64;              // vectors are fp64 (matrix may be fp32)
    int persistent;         // 1: the last solve ran in the persistent kernel
    unsigned long long gbar;            // grid-barrier arrivals of the persistent kernel
    unsigned long long phase_ns[4];     // persistent kernel: device time per phase kind
    long long phase_cnt[4];             //   (Q, U_S, Z, U_J) and phases run, last solve
};

// ------------------------------------------------------------------ tiles
// Row partition for the load-balanced SpMV: tile t holds rows [desc[t].x, desc[t+1].x) and
// entries [desc[t].y, desc[t+1].y).  A tile holds at most D "items" (rows + stored entries)
// and at most RMAX rows, unless it is one single row with D or more entries (a "long row"
// tile, streamed in chunks and reduced by the whole block).
struct TilePart {
    int D = 0;
    int RMAX = 0;
    int n_tiles = 0;
    int2 *d_desc = nullptr;
    struct WinDesc *d_win = nullptr;       // operand windows per tile (see ensure_windows)
    int win_rows = -1;                     // WMAX the windows were built for (-1: not built)
};

// Rows of a long-row matrix grouped by length for the lane-group SpMV: a row of len entries
// goes to a group of G lanes, G the smallest power of two with 4 G >= len (G = 1 up to 32;
// rows longer than 128 entries get a whole warp).  For a BSR matrix the rows are block rows,
// len counts blocks and the factor is 2 (a lane takes two blocks per pass).  The rows of one G form a bin; bins are
// ordered G = 32, 16, ..., 1, and a warp task is 32 / G consecutive rows of one bin.  In
// the G = 32 bin rows are ordered by length, longest first, elsewhere by index.
constexpr int GBINS = 6;
struct GroupPart {
    int n_tasks = 0;
    int task0[GBINS + 1] = {};             // first task of each bin; task0[GBINS] = n_tasks
    int pos0[GBINS + 1] = {};              // first row position of each bin
    int4 *d_rows = nullptr;                // per position: {row, first entry, end entry, 0}
};

// Operand window of a tile of a banded matrix: the tile's columns (and its own rows) lie in
// nseg ranges of rows [a[s], a[s] + l[s]) of the gathered vectors, 4-row aligned; nseg = 0
// means the tile gathers from global memory.
constexpr int WSEG = 4;
struct __align__(16) WinDesc {
    int nseg;
    int a[WSEG];
    int l[WSEG];
    int pad[16 - 1 - 2 * WSEG];
};

// Sliced storage (slices of 32 rows) of a short-row matrix for the persistent solver.
// Slice s holds rows [32 s, 32 s + 32); its entries sit in L_s slot rows of 32 (slot row u,
// lane l: entry u of row 32 s + l), so a warp reads slot row u of its slice with one
// coalesced access.  Two slice kinds:
//   diagonal slice: every row's columns lie at offsets (column - row) from one sorted list
//     of L_s offsets shared by the slice (a stencil's ±1, ±line, 0 ...); slot row u holds
//     the values at offset u (0 where a row has no entry there), so no column index is
//     stored per entry and the operand addresses need no per-entry load;
//   index slice: slot row u holds entry u of each row, with its column as a 16-bit offset
//     from the row (rel16, when every offset of the matrix fits) or a 32-bit column, and
//     per-row lengths.
// desc[s] = {first slot row << 5 | L_s, diagonal << 31 | full << 30 | position of its
// offsets}; "full": every row of the slice holds every offset of the list, so entry u of row
// r is CSR entry row_ptr[r] + u (the CSR-direct product uses that).  Values
// are gathered from the CSR arrays by `perm` (slot -> CSR position, -1 for padding) before
// each solve, so values changed in place are picked up.
struct SellPart {
    int64_t n_slices = 0;
    int64_t n_slots = 0;                 // entry slots (32 per slot row), padding included
    int rel16 = 0;
    int maxl = 0;                        // offsets per diagonal slice at most
    int64_t n_diag = 0;                  // diagonal slices
    uint2 *d_desc = nullptr;
    int32_t *d_offs = nullptr;           // offset lists of the diagonal slices
    uint8_t *d_lens = nullptr;           // row lengths, n_slices * 32 (0 past the last row)
    void *d_idx = nullptr;               // int16 offsets (rel16) or int32 columns
    int32_t *d_perm = nullptr;
    void *d_val = nullptr;               // the matrix's type
};

// Column-sorted row segments of a long-row matrix (csb.cuh): segment s holds rows
// [seg_row0[s], seg_row0[s+1]) (at most CSB_RMAX) and chunks [seg_ch0[s], seg_ch0[s+1]) of
// 32 entry slots, its entries in ascending (column, row) order; per chunk the smallest
// column, per slot (column - base) << 16 | local row (0xFFFF: padding), the CSR position of
// the entry (-1: padding) and its value (gathered from the CSR values before each solve).
// Loads of data read once (a matrix stream), without L1 allocation: L1 is left to data that
// is read again (gathered operand lines).
__device__ __forceinline__ uint32_t ld_stream_b32(const void *q)
{
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.b32 %0, [%1];" : "=r"(v) : "l"(q));
    return v;
}
__device__ __forceinline__ uint64_t ld_stream_b64(const void *q)
{
    uint64_t v;
    asm volatile("ld.global.nc.L1::no_allocate.b64 %0, [%1];" : "=l"(v) : "l"(q));
    return v;
}
template <typename VM>
__device__ __forceinline__ VM ld_stream_val(const VM *q)
{
    if constexpr (sizeof(VM) == 4)
        return __uint_as_float(ld_stream_b32(q));
    else
        return __longlong_as_double((long long)ld_stream_b64(q));
}

struct CsbPart {
    int n_seg = 0;
    int rmax = 0;                        // rows of the largest segment
    int64_t n_chunks = 0;
    int32_t *d_seg_row0 = nullptr;
    int32_t *d_seg_ch0 = nullptr;
    int32_t *d_cbase = nullptr;
    uint32_t *d_pk = nullptr;
    int32_t *d_perm = nullptr;
    void *d_val = nullptr;               // the matrix's type
    // exact fixed-point row sums (csb.cuh): per segment the largest row sum of |a_ij| (with
    // the values), the operand's per-block |v| maxima, the low word's bits
    double *d_seg_bound = nullptr;
    float *d_vmax = nullptr;
    int vmax_n = 0;
    int lb = 20;
};

// Read-only view of a CSR matrix passed to kernels.
template <typename V>
struct MatView {
    const int32_t *rp;
    const int32_t *ci;
    const V *val;
    const int2 *desc;
    int n_tiles;
    int64_t n;
    int64_t nnz;
};

struct Plan;

}  // namespace sla

// ------------------------------------------------------------------ public handle types
struct sla_csr {
    int64_t n = 0, nnz = 0;
    sla_dtype dtype = SLA_F64;
    uint32_t flags = 0;
    const int32_t *rp = nullptr;
    const int32_t *ci = nullptr;
    const void *val = nullptr;
    // block sparse rows: rp / ci index bdim x bdim blocks (row-major values), n and nnz count
    // scalar rows and values; 1 for CSR
    int32_t bdim = 1;
    // owned arrays (used by the internal G^T handle)
    int32_t *own_rp = nullptr, *own_ci = nullptr;
    void *own_val = nullptr;
    // list of systems (block diagonal)
    int32_t batch = 1;
    std::vector<int64_t> sys_off;          // host, batch+1
    int64_t *d_sys_off = nullptr;          // device copy
    int64_t max_sys_n = 0;
    int64_t max_sys_nnz = 0;
    // host copy of row_ptr, for partition building
    std::vector<int32_t> h_rp;
    std::vector<int32_t> h_ci;             // host copy of col (short-row matrices, for windows)
    std::map<int, sla::TilePart> tiles;    // by item budget D
    sla::SellPart *sell = nullptr;         // sliced ELL copy (persistent solver)
    sla::GroupPart *groups = nullptr;      // rows grouped by length (long-row matrices)
    sla::CsbPart *csb = nullptr;           // column-sorted row segments (long-row matrices)
    int csb_vals_current = 0;              // csb's value copy matches the CSR values
    int sell_vals_current = 0;             // sell's value copy matches the CSR values
    int device = 0;
    int num_sms = 148;
    std::vector<sla::Plan *> plans;
    int64_t max_row_len = 0;
    int *d_err = nullptr;                  // pipeline error word of kernels without a plan
    // preconditioners built on this handle (as A or as G); they are detached when it is
    // destroyed, whatever the order the caller destroys handles in
    std::vector<sla_precond *> dependents;
    // device time of the last list solve's kernel (CUDA events around its launch)
    cudaEvent_t list_ev[2] = {nullptr, nullptr};
    int list_ev_recorded = 0;
};

struct sla_precond {
    int kind = 0;                          // 1 Jacobi, 2 SPAI
    const sla_csr *A = nullptr;
    const sla_csr *G = nullptr;            // borrowed (SPAI)
    sla_csr *GT = nullptr;                 // owned explicit transpose (SPAI)
    double eps = 0.0;
    void *d_dinv = nullptr;                // Jacobi: 1 / A_ii in fp32 (fp32 matrices only)
    void *d_dinv64 = nullptr;              // Jacobi: 1 / A_ii in fp64
    int32_t *d_perm = nullptr;             // SPAI: position in G of each G^T entry
};

namespace sla {

// Rows and entries of the stored pattern (blocks for a BSR matrix).
inline int64_t pattern_rows(const sla_csr *A) { return A->n / A->bdim; }
inline int64_t pattern_nnz(const sla_csr *A) { return A->nnz / ((int64_t)A->bdim * A->bdim); }

// Solve plan: workspace + captured graph for one (A, M, K) combination.
struct Plan {
    const sla_precond *M = nullptr;
    int K = 1;
    int vec64 = 0;                         // fp64 vectors with an fp32 matrix
    int kind = 0;                          // 0 none, 1 Jacobi, 2 SPAI
    void *ws = nullptr;                    // one device allocation
    size_t ws_bytes = 0;
    void *x = nullptr, *ra = nullptr, *rb = nullptr, *pa = nullptr, *pb = nullptr;
    void *q = nullptr, *z = nullptr, *y = nullptr;
    double *partials = nullptr;
    PcgState *st = nullptr;
    PcgState *h_st = nullptr;              // pinned host mirror for the final read
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    cudaStream_t cs = nullptr, cs2 = nullptr;
    int grid_tiles_A = 0, grid_tiles_G = 0, grid_tiles_GT = 0, grid_vec = 0;
    unsigned long long cond = 0;           // conditional handle of the loop node
    int persist_grid = 0;                  // persistent engine: blocks (0: not set up yet)
};

// ------------------------------------------------------------------ internal entry points
sla_status ensure_tiles(sla_csr *A, int D, int RMAX, cudaStream_t s, const TilePart **out);
// Build (once) the operand windows of a tile partition, at most wmax rows per tile.
sla_status ensure_windows(sla_csr *A, const TilePart *tp, int wmax, cudaStream_t s);
// Build (once) the sliced copy of a short-row matrix (diagonal slices of at most 8 offsets,
// 16 for rows of 9 to 16 entries); gather its values.
sla_status ensure_sell(sla_csr *A, cudaStream_t s, const SellPart **out);
// Build (once) the length-grouped row list of a matrix.
sla_status ensure_groups(sla_csr *A, cudaStream_t s, const GroupPart **out);
sla_status launch_sell_values(const sla_csr *A, const SellPart *sp, cudaStream_t s);
// Build (once) the column-sorted segments of a long-row CSR matrix; gather their values
// from the CSR values (every solve); free them.
sla_status ensure_csb(sla_csr *A, cudaStream_t s, const CsbPart **out);
sla_status launch_csb_values(const sla_csr *A, cudaStream_t s);
void free_csb(sla_csr *A);
size_t plan_bytes(const sla_csr *A, const sla_precond *M, int K, int vec64);
sla_status get_plan(sla_csr *A, const sla_precond *M, int K, int vec64, Plan **out);
void destroy_plan(Plan *p);

// launchers implemented in the .cu files
sla_status launch_spmv(const sla_csr *A, int K, const void *x, void *y, cudaStream_t s);
// g_k = scale * sum_c lam[row(k)][c] x[col(k)][c] on A's pattern (scale -1: the adjoint's
// dL/dA; +1: the eigenvalue gradient).
sla_status launch_pattern_grad(const sla_csr *A, int K, int vec64, const void *lam, const void *x,
                               void *g, cudaStream_t s, double scale = -1.0);
sla_status launch_validate(const sla_csr *A, int *d_err, cudaStream_t s);
sla_status launch_jacobi_dinv(const sla_csr *A, void *dinv64, void *dinv32, int *d_err, cudaStream_t s);
// G^T of a CSR matrix on the device: row pointers (n+1), columns and perm (nnz each, perm[t] =
// position in G of G^T's t-th entry), all caller-allocated.  SLA_ERR_INVALID_CSR for a
// column of G outside [0, n).  Synchronises s.
sla_status device_transpose(const sla_csr *G, int32_t *rpT, int32_t *ciT, int32_t *perm, cudaStream_t s);
sla_status refresh_transpose_values(const sla_csr *G, sla_csr *GT, const int32_t *d_perm,
                                    cudaStream_t s);
sla_status capture_plan_graph(sla_csr *A, Plan *p);
// Solve with the plan; with grad_out set, also form dL/dA = -X (x) grad_x on A's pattern
// (X = lambda) before the single final synchronisation.
sla_status run_plan(sla_csr *A, Plan *p, int nrhs, const void *B, void *X,
                    const sla_pcg_opts *opts, sla_pcg_info *info, const void *grad_x,
                    void *grad_out, cudaStream_t s);
sla_status kernel_times(sla_csr *A, Plan *p, int nrhs, int reps, double *h_ms, cudaStream_t s);

// per-precision instantiations: ff = fp32 values/vectors, dd = fp64, fd = fp32 values with
// fp64 vectors
#define SLA_COMBO_DECL(T)                                                                            \
    sla_status capture_##T(sla_csr *A, Plan *p);                                                    \
    sla_status times_##T(sla_csr *A, Plan *p, int nrhs, int reps, double *h_ms, cudaStream_t s);     \
    sla_status run_##T(sla_csr *A, Plan *p, int nrhs, const void *B, void *X, double tol,            \
                       long long maxit, int engine, cudaStream_t s);                                \
    sla_status grad_##T(const sla_csr *A, int nrhs, const void *lam, const void *x, void *g,         \
                        double scale, cudaStream_t s);
SLA_COMBO_DECL(ff)
SLA_COMBO_DECL(dd)
SLA_COMBO_DECL(fd)
#undef SLA_COMBO_DECL
sla_status spmv_ff(const sla_csr *A, int nrhs, const void *x, void *y, cudaStream_t s);
sla_status spmv_dd(const sla_csr *A, int nrhs, const void *x, void *y, cudaStream_t s);
// Fails unless every row of M keeps its columns inside its system of the list handle A.
sla_status check_list_blocks(const sla_csr *A, const sla_csr *M, cudaStream_t s);
sla_status run_list_solve(const sla_csr *A, const sla_precond *M, const void *B, void *X,
                          const void *Xfwd, void *G, const sla_pcg_opts *opts, sla_pcg_info *info,
                          cudaStream_t s);

}  // namespace sla
