/*
 * sla.h -- C ABI of the B200 (sm_100a) sparse SPD solver library `libsla`.
 *
 * The library solves A x = b for a sparse symmetric positive definite A stored in CSR by
 * the preconditioned conjugate-gradient method, and provides the adjoint (backward) pass:
 *
 *   forward   x = A^-1 b                                   (PCG, Jacobi or SPAI preconditioner)
 *   backward  A^T lambda = dL/dx,  dL/db = lambda,  dL/dA_ij = -lambda_i x_j on A's pattern
 *
 * Sources (page title, section):
 *   [TS]   "torch-sla: Differentiable Sparse Linear Algebra with Adjoint Solvers and Sparse
 *          Tensor Parallelism for PyTorch": Methodology §1 (the .solve / .matvec API; the
 *          Jacobi-preconditioned native iterative backend; SparseTensor = one matrix or a
 *          batch sharing one pattern, SparseTensorList = a batch with distinct patterns),
 *          Methodology §2 "Linear Systems" (the adjoint), Complexity (O(1) graph nodes,
 *          O(n + nnz) memory, independent of the iteration count).
 *   [SPAI] "Learning Sparse Approximate Inverse Preconditioners for Conjugate Gradient
 *          Solvers on GPUs": Approach (M^-1 = G G^T + eps I, G on A's pattern, two SpMVs
 *          per CG step) and the epsilon ablation (default eps = 3e-3).
 *
 * Conventions common to every call
 *   - Pointers prefixed d_ are DEVICE pointers on the current CUDA device; h_ are HOST
 *     pointers.  Indices are int32 (row_ptr, col); values are fp32 or fp64 (sla_dtype).
 *     Vectors have the matrix's value type: fp32 matrices use fp32 vectors with all dot
 *     products, norms and the scalars alpha, beta, rho in fp64.
 *   - Multi-right-hand-side blocks are [n][nrhs] row-major ("interleaved"): entry (i, c)
 *     is at i * nrhs + c.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  All
 *     device work is enqueued on it.  Calls that return solver results (sla_pcg_*)
 *     synchronise that stream once, at the end, to fill the info structs; no call
 *     synchronises per iteration.
 *   - Ownership: the caller owns every d_ buffer and keeps the arrays passed to
 *     sla_csr_create alive and unchanged (pattern) for the handle's lifetime; values may be
 *     changed in place between calls (then call sla_precond_refresh).  The library owns its
 *     handles, workspaces, the explicit G^T, Jacobi's D^-1 and the captured CUDA graphs; the
 *     matching _destroy call frees them.
 *   - Errors: every call returns an sla_status.  Negative values are errors and leave
 *     outputs unspecified; sla_last_error() gives a thread-local message.  Solver outcomes
 *     SLA_NOT_CONVERGED and SLA_BREAKDOWN are positive: the outputs hold the last iterate.
 *   - Handles are not thread-safe: one host thread at a time per handle.  Work queued on
 *     one handle to different streams must not overlap in time (order the streams): the
 *     handle's layout copies and scratch (value copies, per-segment bounds, operand maxima
 *     of the column-sorted products) are shared by its calls.
 *   - Products of fp32 values with fp32 vectors on the column-sorted segments (long-row
 *     single-RHS solves, and sla_spmv on SLA_STATIC_VALUES handles) sum each row exactly in
 *     fixed point after rounding every term to 2^-63 of its segment's bound (largest row sum
 *     of |a_ij| times max |v_j|): results are bit-reproducible run to run.
 */
#ifndef SLA_H
#define SLA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SLA_API __attribute__((visibility("default")))
#else
#define SLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t sla_status;
#define SLA_SUCCESS 0
#define SLA_NOT_CONVERGED 1       /* maxit reached; x holds the last iterate           */
#define SLA_BREAKDOWN 2           /* p.q <= 0, r.z <= 0 or a non-finite value: A or M   */
                                  /* is not SPD (or the input holds NaN/Inf)            */
#define SLA_ERR_INVALID_ARG (-1)  /* null pointer, bad size, dtype or handle mismatch   */
#define SLA_ERR_INVALID_CSR (-2)  /* SLA_VALIDATE found a malformed pattern             */
#define SLA_ERR_CUDA (-3)         /* a CUDA runtime call failed                         */
#define SLA_ERR_OOM (-4)          /* device or host allocation failed                   */
#define SLA_ERR_UNSUPPORTED (-5)  /* valid request outside what this build implements   */

typedef enum { SLA_F32 = 0, SLA_F64 = 1 } sla_dtype;

/* Flags for sla_csr_create*. */
#define SLA_SPD 1u        /* caller asserts A is symmetric positive definite (needed by PCG) */
#define SLA_VALIDATE 2u   /* check the pattern on the device: row_ptr[0] = 0, row_ptr non-  */
                          /* decreasing, row_ptr[n] = nnz, columns in range, strictly        */
                          /* ascending in each row (so duplicates are rejected, not summed)  */
#define SLA_STATIC_VALUES 4u /* the caller does not change the values after creation, or    */
                          /* calls sla_csr_values_changed after it does: single-vector       */
                          /* products (sla_spmv) may then read a copy of the values kept in  */
                          /* the library's own layout (solves re-read the values anyway)     */

typedef struct sla_csr sla_csr;
typedef struct sla_precond sla_precond;

/* Solver options.  Zero-initialised fields take the defaults given. */
typedef struct {
    double rtol;        /* stop when ||r_k||_2 / ||b||_2 <= rtol on the recursive residual;
                           0 -> 1e-10 for fp64, 1e-6 for fp32                              */
    int64_t maxit;      /* iteration cap per right-hand side; 0 -> 10 * n (n of the system) */
    int32_t vector_f64; /* nonzero with an fp32 matrix: mixed precision -- b, x, the adjoint's
                           dL/dx and dL/db and all solver vectors are fp64 (dL/dA stays fp32);
                           the default tolerance is then 1e-10.  Ignored for fp64 matrices
                           and for list handles. */
    int32_t engine;     /* how the solve loop runs (SLA_ENGINE_*); 0 -> automatic */
} sla_pcg_opts;

/* Solve engines.  Both run every step of the method on the GPU with the same fused
 * operations and the same stopping test; the dot products are summed over different
 * block partitions (each in a fixed order, so each engine is deterministic), so their
 * iterates agree to rounding, not bit for bit.
 *   SLA_ENGINE_GRAPH: one kernel per fused operation, the iteration loop a CUDA graph with
 *     a device-side conditional (while) node -- any row-length mix.
 *   SLA_ENGINE_PERSISTENT: the whole solve in one cooperative launch; the fused operations
 *     are phases separated by grid barriers, and the matrix stream of the next phase is
 *     prefetched while the current one runs.  For single systems whose matrices (A, and G
 *     and G^T with SPAI) hold at most 8 entries per row, with at most 8 right-hand sides
 *     (fp64 vectors: at most 4); fp32 vectors with at most 2 right-hand sides also allow
 *     rows of up to 16 entries.
 *   SLA_ENGINE_AUTO (0): persistent where it applies, graph otherwise.
 * Asking for SLA_ENGINE_PERSISTENT where it does not apply fails with SLA_ERR_INVALID_ARG.
 * List handles always use the one-block-per-system list kernel (SLA_ENGINE_LIST). */
#define SLA_ENGINE_AUTO 0
#define SLA_ENGINE_GRAPH 1
#define SLA_ENGINE_PERSISTENT 2
#define SLA_ENGINE_LIST 3

/* Per right-hand side (or per system of a list) solver outcome. */
typedef struct {
    int64_t iters;      /* number of products q = A p taken (0 when b = 0)                   */
    double relres;      /* ||r||/||b|| of the recursive residual at exit (0 when b = 0)      */
    int32_t status;     /* SLA_SUCCESS, SLA_NOT_CONVERGED or SLA_BREAKDOWN                   */
    int32_t engine;     /* the engine that ran the solve (SLA_ENGINE_GRAPH, _PERSISTENT, _LIST) */
} sla_pcg_info;

/* ---------------------------------------------------------------- library */
SLA_API const char *sla_version(void);
SLA_API const char *sla_status_string(sla_status s);
/* Message of the last failing call on this host thread ("" if none). */
SLA_API const char *sla_last_error(void);

/* ---------------------------------------------------------------- matrices */
/* One square CSR matrix ([TS] Methodology §1, SparseTensor).
 * n_rows == n_cols is required (the solver works on square SPD systems); nnz = row_ptr[n].
 * d_row_ptr (n+1), d_col (nnz), d_val (nnz, `dtype`) are borrowed, not copied, and must be
 * 16-byte aligned (SLA_ERR_INVALID_ARG otherwise): the SpMV streams them by bulk copies.
 * The pattern (d_row_ptr, d_col) must not change while the handle lives: the library
 * derives row partitions and sliced layouts from it at first use.  The values may change
 * between calls; every product and solve reads the current values. 
 * Set-up work (load-balanced tile partition of the rows, optional validation) runs on
 * `stream` and is synchronised before return.  Returns SLA_ERR_INVALID_CSR on a pattern
 * that fails SLA_VALIDATE. */
SLA_API sla_status sla_csr_create(sla_csr **out, int64_t n_rows, int64_t n_cols, int64_t nnz,
                          const int32_t *d_row_ptr, const int32_t *d_col, const void *d_val,
                          sla_dtype dtype, uint32_t flags, void *stream);

/* A batch of independent systems with distinct patterns ([TS] Methodology §1,
 * SparseTensorList), stored as ONE block-diagonal CSR of n_total rows: system s owns rows
 * and columns [h_sys_row_off[s], h_sys_row_off[s+1]); h_sys_row_off (host, batch+1 entries,
 * h_sys_row_off[0] = 0, last = n_total) is copied.  Column indices are global and must lie in
 * the owning system's range (checked by SLA_VALIDATE).  sla_spmv works on the whole block
 * matrix; sla_pcg_solve_batched / sla_pcg_adjoint_batched solve every system on its own,
 * each with its own stopping test and info entry (one block per system: its vectors in
 * shared memory, or in a workspace the call allocates when the largest system's do not fit;
 * Jacobi, SPAI or no preconditioner). */
SLA_API sla_status sla_csr_create_list(sla_csr **out, int32_t batch, const int64_t *h_sys_row_off,
                               int64_t nnz_total, const int32_t *d_row_ptr, const int32_t *d_col,
                               const void *d_val, sla_dtype dtype, uint32_t flags, void *stream);

/* One square block sparse row (BSR) matrix: dense block_dim x block_dim blocks on a CSR
 * pattern of blocks ([SM] "Efficient Sparse Matrix Algebra in Python for Mathematics", Key
 * sparse formats and memory tradeoffs; Block sparse patterns and sharding strategies: one
 * index per dense block).  block_dim is 2, 3 or 4 (SLA_ERR_INVALID_ARG otherwise; use
 * sla_csr_create for 1).  d_row_ptr (n_block_rows+1) and d_col (nnzb) index blocks, with
 * nnzb = row_ptr[n_block_rows]; d_val holds nnzb*block_dim^2 values of `dtype`, block k
 * row-major at d_val[k*block_dim^2], so scalar entry (I*b + r, col[k]*b + c) is
 * d_val[k*b*b + r*b + c].  The scalar system has n = n_block_rows*block_dim rows and
 * nnz = nnzb*block_dim^2 stored values (what sla_csr_shape reports, and the length of a
 * gradient on the pattern, aligned with d_val).  Borrowing, alignment, immutability of the
 * pattern and SLA_VALIDATE (on the block pattern) are as for sla_csr_create.  The handle
 * works with sla_spmv, sla_spmv_multi and the batched solves up to 4 right-hand sides,
 * sla_precond_jacobi (the scalar diagonal) and as A of sla_precond_spai (G must be CSR),
 * the solves and adjoints (graph engine), and sla_pattern_grad. */
SLA_API sla_status sla_bsr_create(sla_csr **out, int64_t n_block_rows, int32_t block_dim, int64_t nnzb,
                          const int32_t *d_row_ptr, const int32_t *d_col, const void *d_val,
                          sla_dtype dtype, uint32_t flags, void *stream);

SLA_API sla_status sla_csr_destroy(sla_csr *A);

/* For a handle created with SLA_STATIC_VALUES: the caller changed the values in place, so
 * copies of them held in the library's layouts must be refreshed before the next product
 * (done lazily, on `stream`, by that product).  Harmless on other handles. */
SLA_API sla_status sla_csr_values_changed(sla_csr *A, void *stream);

/* n_rows, nnz and batch (1 for a single matrix) of a handle; any output may be NULL. */
SLA_API sla_status sla_csr_shape(const sla_csr *A, int64_t *n_rows, int64_t *nnz, int32_t *batch);

/* y = A x ([TS] Methodology §1, .matvec).  d_x, d_y: n vectors of A's dtype, must not
 * overlap.  Accumulates each row in fp64 and rounds once to the value type. */
SLA_API sla_status sla_spmv(const sla_csr *A, const void *d_x, void *d_y, void *stream);

/* Y = A X for nrhs right-hand sides in [n][nrhs] layout (1 <= nrhs <= 16; a BSR handle
 * takes at most 4, SLA_ERR_INVALID_ARG above). */
SLA_API sla_status sla_spmv_multi(const sla_csr *A, int32_t nrhs, const void *d_X, void *d_Y, void *stream);

/* ---------------------------------------------------------------- preconditioners */
/* Jacobi: M^-1 = D^-1, D = diag(A) ([TS] Methodology §1, the native backend's
 * preconditioner).  Every row must store a positive diagonal entry, else
 * SLA_ERR_INVALID_ARG.  The preconditioner belongs to A and must be used with A only. */
SLA_API sla_status sla_precond_jacobi(sla_precond **out, const sla_csr *A, void *stream);

/* SPAI: M^-1 = G G^T + eps I ([SPAI] Approach).  G is a square CSR of A's size (it normally
 * carries A's lower-triangular pattern; any pattern is accepted), borrowed like A; the
 * library forms and owns G^T explicitly so each apply is two plain SpMVs.  For a list
 * handle A, G must be block-diagonal with the same blocks (checked on the device:
 * SLA_ERR_INVALID_ARG otherwise). */
SLA_API sla_status sla_precond_spai(sla_precond **out, const sla_csr *A, const sla_csr *G, double eps,
                            void *stream);

/* Recompute what the preconditioner derives from A's or G's values (D^-1, G^T values)
 * after the caller changed them in place. */
SLA_API sla_status sla_precond_refresh(sla_precond *M, void *stream);

SLA_API sla_status sla_precond_destroy(sla_precond *M);

/* ---------------------------------------------------------------- solves */
/* x = A^-1 b by PCG from x0 = 0 ([TS] Methodology §1 .solve; [SPAI] Approach).
 * M may be NULL (plain CG).  d_b, d_x: n vectors; may not overlap.  On SLA_SUCCESS,
 * ||r||/||b|| <= rtol for the recursive residual r.  b = 0 gives x = 0 and iters = 0.
 * info may be NULL.  Workspace is O(n) and does not grow with the iteration count. */
SLA_API sla_status sla_pcg_solve(const sla_csr *A, const sla_precond *M, const void *d_b, void *d_x,
                         const sla_pcg_opts *opts, sla_pcg_info *info, void *stream);

/* Adjoint of x = A^-1 b ([TS] Methodology §2, Linear Systems): solves A^T lambda = dL/dx
 * with the same PCG and preconditioner (A is SPD, so A^T = A), writes dL/db = lambda (n)
 * and dL/dA_k = -lambda_row(k) * x_col(k) for every stored entry k (nnz, aligned with A's
 * values).  d_x is the forward solution.  d_dLdA may be NULL to skip the gradient. */
SLA_API sla_status sla_pcg_adjoint(const sla_csr *A, const sla_precond *M, const void *d_x,
                           const void *d_dLdx, void *d_dLdb, void *d_dLdA,
                           const sla_pcg_opts *opts, sla_pcg_info *info, void *stream);

/* Batched solve.  For a single matrix: nrhs (1..16) right-hand sides in [n][nrhs] layout
 * sharing A, each with its own stopping test; h_info has nrhs entries.  For a list handle:
 * nrhs must be 1, d_B/d_X are the concatenated n_total vectors and h_info has `batch`
 * entries. */
SLA_API sla_status sla_pcg_solve_batched(const sla_csr *A, const sla_precond *M, int32_t nrhs,
                                 const void *d_B, void *d_X, const sla_pcg_opts *opts,
                                 sla_pcg_info *h_info, void *stream);

/* Batched adjoint.  Single matrix: Lambda (= dL/dB) per RHS, dL/dA summed over the RHS
 * (sum_c -lambda_c,i x_c,j).  List handle: per system, concatenated (each system's block
 * of dL/dA is its own gradient). */
SLA_API sla_status sla_pcg_adjoint_batched(const sla_csr *A, const sla_precond *M, int32_t nrhs,
                                   const void *d_X, const void *d_dLdX, void *d_dLdB,
                                   void *d_dLdA, const sla_pcg_opts *opts, sla_pcg_info *h_info,
                                   void *stream);

/* dL/dA_k = -sum_c lambda_c,row(k) * x_c,col(k) on A's pattern, for nrhs vectors in
 * [n][nrhs] layout ([TS] Methodology §2; with lambda = x = v it is the Hellmann-Feynman
 * eigenvalue gradient of the same section up to sign).  For a BSR handle k runs over the
 * stored scalar values in d_val order (nnzb*b*b of them). */
SLA_API sla_status sla_pattern_grad(const sla_csr *A, int32_t nrhs, const void *d_lam, const void *d_x,
                            void *d_g, void *stream);

/* Eigenvalue gradient by the Hellmann-Feynman theorem ([TS] Methodology §2, Eigenvalue
 * Problems): for a simple eigenvalue mu of a symmetric A with unit eigenvector v,
 * d mu / d A_ij = v_i v_j, formed on A's pattern only.  d_V holds nvec (>= 1) unit
 * eigenvectors in [n][nvec] layout, A's dtype; d_g (nnz, aligned with A's values) receives
 * g_k = sum_c V[row(k)][c] V[col(k)][c], the gradient of the sum of those eigenvalues.  The
 * eigenvectors come from the caller (this library has no eigensolver).  Same kernel as
 * sla_pattern_grad with the opposite sign; BSR handles give g in d_val order. */
SLA_API sla_status sla_eigen_grad(const sla_csr *A, int32_t nvec, const void *d_V, void *d_g, void *stream);

/* d_val_out = the values of A + diag(d_c) on A's pattern ([TS] Methodology §2, Nonlinear
 * Systems: the Jacobian J = dF/du of F(u) = A u + N(u) - b with an elementwise N is
 * A + diag(N'(u))).  d_c: n values of A's dtype; d_val_out: nnz values (caller-owned, not A's
 * own array), usually the value array of a handle J created once on A's pattern arrays.
 * Every row must store its diagonal (SLA_ERR_INVALID_ARG otherwise); CSR and list handles
 * (SLA_ERR_UNSUPPORTED for BSR).  Synchronises `stream`.  A Jacobi preconditioner built on
 * J must be refreshed (sla_precond_refresh) after J's values change. */
SLA_API sla_status sla_csr_add_diagonal(const sla_csr *A, const void *d_c, void *d_val_out, void *stream);

/* Backward pass of a nonlinear system F(u, theta) = 0 solved by the caller ([TS] Methodology
 * §2, Nonlinear Systems): one adjoint solve J^T lambda = dL/du with the Jacobian J = dF/du at
 * the solution u (J SPD, so the same PCG as sla_pcg_solve, with M built on J), then the
 * vector-Jacobian product for F = A u + N(u) - b: dL/dA_k = -lambda_row(k) u_col(k) on A's
 * pattern (A's values are the parameters) and dL/db = lambda.  d_lambda (n) receives lambda;
 * A and d_dLdA may be NULL to skip the product; A must match J's size, dtype and batch (J
 * may share A's pattern arrays).  The work does not depend on how many nonlinear iterations
 * the forward solve took.  Single systems; vector types as sla_pcg_solve (opts->vector_f64). */
SLA_API sla_status sla_nonlinear_adjoint(const sla_csr *J, const sla_precond *M, const sla_csr *A,
                                         const void *d_u, const void *d_dLdu, void *d_lambda,
                                         void *d_dLdA, const sla_pcg_opts *opts, sla_pcg_info *info,
                                         void *stream);

/* ---------------------------------------------------------------- iteration steps
 * The vector steps of one PCG iteration as separate calls, for solvers that drive the
 * iteration from the host between collectives: the row-block distributed PCG of [TS]
 * Methodology §3 (each rank owns a contiguous block of rows, exchanges halo values before
 * each product and all-reduces the scalars).  dtype is the vectors' type (SLA_F32 or
 * SLA_F64); all vectors are device arrays of n elements; reductions are fp64, summed in a
 * fixed order (deterministic) and written to DEVICE memory, so they can feed a collective
 * without a host round trip.  fp32 updates round the scalar to fp32 once and use one fused
 * multiply-add, as the single-GPU solve engines do.  None synchronises `stream`. */

/* d_out[0] = sum_i x_i y_i (fp64). */
SLA_API sla_status sla_vec_dot(int32_t dtype, int64_t n, const void *d_x, const void *d_y, double *d_out,
                               void *stream);

/* The update after q = A p ([TS] Methodology §1 CG step): x += alpha p, r -= alpha q,
 * z = D^-1 r (d_dinv: n values of 1/A_ii in the vector type; NULL: z = r), and
 * d_out2[0] = r.r, d_out2[1] = r.z of the updated r (fp64). */
SLA_API sla_status sla_pcg_update(int32_t dtype, int64_t n, double alpha, const void *d_p, const void *d_q,
                                  void *d_x, void *d_r, const void *d_dinv, void *d_z, double *d_out2,
                                  void *stream);

/* p = z + beta p. */
SLA_API sla_status sla_pcg_direction(int32_t dtype, int64_t n, double beta, const void *d_z, void *d_p,
                                     void *stream);

/* d_dst[k] = d_src[d_idx[k]] for k < n (packing the values a neighbour needs; indices must
 * lie inside d_src). */
SLA_API sla_status sla_vec_gather(int32_t dtype, int64_t n, const int32_t *d_idx, const void *d_src,
                                  void *d_dst, void *stream);

/* d_dst[d_idx[k]] += d_src[k] for k < n (summing received halo contributions into their
 * owner's entries); the indices of one call must be distinct (no atomics: the result is
 * deterministic), and lie inside d_dst. */
SLA_API sla_status sla_vec_scatter_add(int32_t dtype, int64_t n, const int32_t *d_idx, const void *d_src,
                                       void *d_dst, void *stream);

/* The list solve of sla_pcg_solve_batched (list handle, nrhs = 1; every system's vectors
 * must fit in shared memory -- SLA_ERR_UNSUPPORTED otherwise, since the workspace the
 * regular call would take is an allocation) for callers that cannot allocate device memory
 * while they solve --
 * code under a memory pool or budget that owns the device's memory, hosts that forbid
 * allocation after start-up, or code that must avoid the synchronisation an allocation or
 * free can bring.  This call allocates nothing: the per-system results pass through a
 * fixed array in the library's own device memory (1.5 MiB, held by every GPU that loads
 * the library until the process exits), and at most 65536 systems are accepted per call
 * (SLA_ERR_INVALID_ARG beyond that).  Every call looks up that array's device address in
 * the current context (cudaGetSymbolAddress, a host-side lookup), fills this call's slots
 * with status -1 and synchronises `stream` to read the results back into h_info, so the
 * call cannot be captured into a CUDA graph.  All calls on a device share the array: calls that overlap on
 * the GPU race on it.  The matrix and preconditioner handles
 * are created beforehand with the usual calls.  There is no counterpart on the pages this
 * library follows: it is an interface variant, not a different method. */
SLA_API sla_status sla_pcg_solve_batched_noalloc(const sla_csr *A, const sla_precond *M,
                                                 const void *d_B, void *d_X,
                                                 const sla_pcg_opts *opts, sla_pcg_info *h_info,
                                                 void *stream);

/* Per-kernel device time of one PCG iteration (metrics).  On the workspace of the
 * (A, M, nrhs, vector_f64) solver -- normally right after a solve, so it holds that solve's vectors --
 * launches the iteration's kernels `reps` times in loop order, each bracketed by CUDA
 * events on `stream`, with the scalar updates switched off, and writes the mean ms per
 * launch to h_ms[0..2]: [0] p-update + q = A p, [1] the x/r update (Jacobi: with z = D^-1 r;
 * SPAI: with y = G^T r), [2] z = G y + eps r (SPAI; 0 otherwise).  The workspace contents
 * are unspecified afterwards (the next solve re-initialises them).  Synchronises `stream`. */
SLA_API sla_status sla_pcg_kernel_times(const sla_csr *A, const sla_precond *M, int32_t nrhs,
                                        int32_t vector_f64, int32_t reps, double *h_ms, void *stream);

/* Device time, in ms, of the list kernel of the last list solve on list handle A (forward or
 * adjoint; CUDA events recorded on the solve's stream right before and after the kernel's
 * launch, so the time holds that one kernel and nothing the call does around it).
 * SLA_ERR_INVALID_ARG when A is not a list handle or no list solve has run on it since its
 * creation (the allocation-free list solve is not timed).  Waits for the end event. */
SLA_API sla_status sla_list_kernel_ms(const sla_csr *A, double *h_ms);

/* Device time per phase of the last persistent-engine solve of the (A, M, nrhs, vector_f64)
 * solver, measured inside the kernel by block 0 from one grid barrier to the next (so each
 * phase's time includes the barrier that ends it).  h_ms[0..3]: mean ms of a
 * [0] p-update + q = A p, [1] x/r update with y = G^T r (SPAI), [2] z = G y + eps r (SPAI),
 * [3] x/r update with z = D^-1 r (Jacobi or none); h_count[0..3]: phases of each kind run.
 * SLA_ERR_INVALID_ARG when that solver's last solve did not run on the persistent engine.
 * Synchronises `stream`. */
SLA_API sla_status sla_pcg_phase_times(const sla_csr *A, const sla_precond *M, int32_t nrhs,
                                       int32_t vector_f64, double *h_ms, int64_t *h_count,
                                       void *stream);

/* Device bytes the solver workspace takes for (A, M, nrhs, vector_f64); it depends on n and nnz only,
 * never on the iteration count ([TS] Complexity). */
SLA_API size_t sla_workspace_bytes(const sla_csr *A, const sla_precond *M, int32_t nrhs,
                                   int32_t vector_f64);

#ifdef __cplusplus
}
#endif
#endif /* SLA_H */
