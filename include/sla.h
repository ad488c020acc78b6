/*
 * sla.h -- C ABI of the B200 (sm_100a) library for differentiable sparse SPD
 * solves on CSR matrices: Jacobi-preconditioned conjugate gradient, its
 * implicit-function-theorem adjoint, and the sparse value gradient.
 *
 * The operations follow "torch-sla: Differentiable Sparse Linear Algebra with
 * Adjoint Solvers and Sparse Tensor Parallelism for PyTorch" (gist.science
 * summary page, technical summary):
 *   - "Methodology" 1 (unified backend abstraction): the autograd-aware
 *     `.solve` and `.matvec` calls, an iterative GPU solver, and the
 *     `SparseTensor` type that holds one matrix or a batch sharing one pattern;
 *   - "Methodology" 2 (adjoint differentiation framework, linear systems): the
 *     backward pass solves one adjoint system A^T lambda = dL/dx, and the
 *     gradient with respect to the matrix is -lambda_i * x_j on the sparsity
 *     pattern only (dL/db = lambda follows from the same implicit-function
 *     argument);
 *   - "Significance" (limitations): the PyTorch-native iterative backend uses
 *     a Jacobi preconditioner.
 *
 * Conventions shared by every call
 *   - Indices are int32: rowptr[n_rows + 1], colind[nnz], so nnz < 2^31.
 *     Column indices within a row are strictly increasing (validated by
 *     SLA_FLAG_VALIDATE or sla_csr_check).
 *   - Pointers named "device" must point to GPU global memory of the current
 *     device; the caller allocates and frees them.  The library never keeps a
 *     caller pointer beyond the call except rowptr/colind, which a handle
 *     borrows: they must stay valid and unchanged until sla_csr_destroy.
 *   - Batched arrays are batch-major and contiguous: values [B][nnz],
 *     vectors [B][n].  All B systems share the handle's pattern.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     only enqueues work on it and returns; results are valid once the stream
 *     reaches that point.  No call synchronises the host except
 *     sla_csr_create (pattern analysis) and the one-time lazy build of A^T's
 *     pattern (first transposed use of a non-symmetric handle).
 *   - Calls return an sla_status synchronously for argument errors and CUDA
 *     launch errors; sla_last_error_string() (per host thread) explains the
 *     last non-OK status.  Solve outcomes are per system and written to device
 *     memory (sla_cg_info) because they are only known on the GPU.
 *   - Workspace is caller-provided device memory of at least
 *     sla_workspace_bytes() bytes, 256-byte aligned.  Solves and SpMVs never
 *     allocate device memory.  Concurrent calls need distinct workspaces.
 *   - A handle fills a few caches on first use (A^T's pattern for a
 *     non-symmetric handle, the resident grid of the pipelined SpMV); calls on
 *     one handle from several host threads must be serialised by the caller.
 *   - Every device-side wait is bounded (sla_cg_opts.wait_timeout_ns); a wait
 *     that runs out makes the kernel return and the affected systems report
 *     SLA_TIMED_OUT.  No kernel traps.
 */
#ifndef SLA_H
#define SLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct sla_csr_s *sla_csr_t;

typedef enum { SLA_F64 = 0, SLA_F32 = 1 } sla_dtype;

/* Call-level status. */
typedef enum {
    SLA_OK = 0,
    SLA_ERR_INVALID = 1,      /* bad argument or invalid pattern */
    SLA_ERR_CUDA = 2,         /* a CUDA runtime call or launch failed */
    SLA_ERR_OOM = 3,          /* sla_csr_create could not allocate its metadata */
    SLA_ERR_TIMEOUT = 4,      /* reserved for host-side waits */
    SLA_ERR_UNSUPPORTED = 5   /* valid request this build cannot serve */
} sla_status;

/* Per-system solve outcome (device int32 in sla_cg_info.status). */
enum {
    SLA_CONVERGED = 0,        /* ||r_k|| <= max(rtol ||b||, atol), or r_k == 0 */
    SLA_NOT_CONVERGED = 1,    /* max_iter reached in tolerance mode */
    SLA_BREAKDOWN = 2,        /* p.Ap <= 0, or a diagonal entry <= 0 under Jacobi */
    SLA_NONFINITE = 3,        /* NaN/Inf in b, p.Ap or ||r||^2 */
    SLA_FIXED_DONE = 4,       /* exactly fixed_iters iterations ran */
    SLA_TIMED_OUT = 5         /* a device-side wait ran out; x is not valid */
};

/* sla_csr_create flags. */
enum {
    SLA_FLAG_VALIDATE = 1u,        /* check the pattern (sync); invalid -> SLA_ERR_INVALID */
    SLA_FLAG_SYMMETRIC = 2u,       /* caller asserts A^T == A for every value set */
    SLA_FLAG_BUILD_TRANSPOSE = 4u  /* build A^T's pattern now (needed for transposed ops
                                      on a non-symmetric handle; built lazily otherwise) */
};

/* Solver strategies (sla_cg_opts.strategy).  AUTO picks by size: one
 * thread-block cluster per system (matrix slice and vectors in the blocks'
 * shared memory, p shared over distributed shared memory) for a few systems
 * that fit a cluster; one thread block per system when a system's vectors fit
 * in shared memory; else one persistent cooperative grid with device-wide
 * barriers.  The others force a choice (benchmarks and tests). */
enum { SLA_STRATEGY_AUTO = 0, SLA_STRATEGY_GRID = 1, SLA_STRATEGY_BLOCK = 2,
       SLA_STRATEGY_CLUSTER = 3 };

typedef struct {
    double rtol;              /* relative residual target (tolerance mode) */
    double atol;              /* absolute residual floor; stop at max(rtol*||b||, atol) */
    int32_t max_iter;         /* cap in tolerance mode; <= 0 means min(10 n, 100000) */
    int32_t fixed_iters;      /* > 0: run exactly this many iterations, no tolerance test */
    int32_t precond;          /* 1: Jacobi M = diag(A); 0: none */
    int32_t x0_given;         /* 1: x holds the initial guess on entry; 0: start from 0 */
    int64_t wait_timeout_ns;  /* bound on each device-side wait; <= 0 means 5 s */
    int32_t strategy;         /* SLA_STRATEGY_* */
    int32_t reserved;         /* must be 0 */
} sla_cg_opts;

/* Per-system outputs, device pointers to [B] arrays ([n_items] for a list
 * handle, see sla_csr_list_create); any may be NULL. */
typedef struct {
    int32_t *iters;           /* completed iterations (alpha-updates) */
    double *relres;           /* recursive ||r_k|| / ||b|| at exit */
    int32_t *status;          /* SLA_CONVERGED ... SLA_TIMED_OUT */
} sla_cg_info;

/* Pattern statistics a handle computed at creation (host copy). */
typedef struct {
    int32_t n_rows, n_cols;
    int64_t nnz;
    int32_t batch;
    int32_t dtype;            /* sla_dtype */
    int32_t row_min, row_max; /* entries per row */
    double row_mean;
    int32_t lanes;            /* threads cooperating on one row in SpMV-like kernels */
    int32_t grid_blocks;      /* persistent-grid size on this device */
    int32_t block_fits;       /* 1 if one system fits the block-per-system solver */
    int32_t has_transpose;    /* 1 once A^T's pattern is built */
    int32_t grid_onchip;      /* 1 if the grid solver keeps x, r, M^-1 on chip (else in HBM);
                                 2 if, besides, a single system on the sliced layout runs
                                 the two-barrier form (directions formed while gathered);
                                 the environment variables SLA_GRID_ONCHIP=0 and
                                 SLA_GRID2=0, read at creation, turn these variants off */
    int32_t grid_tile_rows;   /* rows of one grid-solver tile (SLA_SELL_PACK=1, read at each
                                 solve, makes the sliced SpMV read value-and-column records,
                                 one load an entry; off by default, see the design notes) */
    int32_t sliced;           /* 1 if the grid solver uses the 8-row sliced layout (one
                                 extra value-gather kernel per solve); 2 if, besides,
                                 every slice is padded to the widest row (padding at most
                                 3 % of the entries; SLA_SELL_UNIFORM=0, read at creation,
                                 turns this off); 3 if the rows of each 32-row window are
                                 ordered by length before slicing (irregular rows, vectors
                                 in HBM; SLA_SELL_SORT=0 turns this off) */
    int32_t block_resident;   /* 1 if the block solver keeps values and pattern of a
                                 system in shared memory as well as its vectors */
    int32_t cluster_fits;     /* 1 if one system fits the cluster solver */
    int32_t n_items;          /* list handles: number of items (0 otherwise) */
    int32_t item_rows_max;    /* list handles: rows of the largest item */
    int32_t item_smem_rows;   /* list handles: items up to this size keep their vectors in
                                 shared memory (larger ones use the workspace) */
    int32_t sliced_col_bytes; /* bytes a column of the sliced layout takes in the solver's
                                 matrix stream: 2 when every |column - row| < 2^15 (16-bit
                                 offsets from the row; SLA_SELL_D16=0, read at creation,
                                 turns them off), else 4; 0 without the sliced layout */
    int32_t interleaved;      /* 1 if forward (and symmetric adjoint) grid solves of this
                                 batch of 2 or 4 systems run the interleaved solver: values
                                 [entry][system] and vectors [row][system] in the workspace,
                                 one column index and gather address for all systems.
                                 SLA_INTERLEAVE=0, read at creation, turns it off */
} sla_csr_props;

/* Operations for sla_workspace_bytes. */
enum { SLA_OP_SPMV = 0, SLA_OP_CG = 1, SLA_OP_ADJOINT = 2, SLA_OP_GRAD = 3 };

/*
 * Create a handle for a CSR pattern shared by `batch` value sets of `dtype`
 * ("Methodology" 1: SparseTensor with one shared pattern).
 * rowptr/colind: device, borrowed until destroy.  The handle allocates and owns
 * derived metadata only (diagonal positions; A^T's pattern when requested).
 * Synchronises `stream` once to read the pattern statistics (and the check
 * result with SLA_FLAG_VALIDATE).  Errors: SLA_ERR_INVALID (sizes, NULL,
 * invalid pattern with VALIDATE; the message names the first bad index),
 * SLA_ERR_OOM, SLA_ERR_CUDA.  *out is NULL on error.
 */
sla_status sla_csr_create(int32_t n_rows, int32_t n_cols, int64_t nnz,
                          const int32_t *rowptr, const int32_t *colind,
                          int32_t batch, sla_dtype dtype, uint32_t flags,
                          void *stream, sla_csr_t *out);

/* Release a handle and its metadata (waits for nothing; the caller must not
 * destroy a handle that queued work still uses).  NULL is a no-op. */
sla_status sla_csr_destroy(sla_csr_t h);

/* Host copy of the handle's statistics. */
sla_status sla_csr_get_props(sla_csr_t h, sla_csr_props *props);

/* Device pointers to A^T's pattern and the value permutation (A^T's entry s is
 * A's entry perm[s]); builds them on `stream` if not built yet.  Valid until
 * destroy.  For square symmetric handles the pattern equals A's. */
sla_status sla_csr_transpose_pattern(sla_csr_t h, const int32_t **rowptrT,
                                     const int32_t **colindT, const int32_t **perm,
                                     void *stream);

/* Workspace bytes that `op` needs on this handle (0 if none). */
size_t sla_workspace_bytes(sla_csr_t h, int32_t op);

/*
 * Batched SpMV ("Methodology" 1, `.matvec`):
 *   y_b = alpha * op(A_b) x_b + beta * y_b,  op = A (transpose == 0) or A^T.
 * vals: device [B][nnz]; x: device [B][n_cols] (A) or [B][n_rows] (A^T);
 * y: device [B][n_rows] or [B][n_cols].  beta == 0 never reads y.  x and y must
 * not overlap.  A^T on a non-symmetric handle uses A^T's pattern (built here on
 * first use, which allocates handle metadata once).
 */
sla_status sla_spmv(sla_csr_t h, const void *vals, const void *x, void *y,
                    int32_t transpose, double alpha, double beta, void *stream);

/*
 * Batched Jacobi-preconditioned CG solve of A_b x_b = b_b for every system b
 * (the iterative `.solve` of "Methodology" 1 with the Jacobi preconditioner
 * of "Significance").  Textbook Hestenes-Stiefel PCG; stopping on the
 * recursively updated residual; fixed mode runs exactly fixed_iters steps.
 * For dtype F32, vectors and row sums are fp32 and every dot product is
 * accumulated in fp64.  Each system stops on its own; the whole iteration
 * runs on the GPU with no host synchronisation.
 * vals [B][nnz], b [B][n], x [B][n] (in: initial guess if x0_given; out:
 * solution), all device.  ws: device, >= sla_workspace_bytes(h, SLA_OP_CG).
 * Requires n_rows == n_cols.
 */
sla_status sla_cg_solve(sla_csr_t h, const void *vals, const void *b, void *x,
                        const sla_cg_opts *opts, sla_cg_info info,
                        void *ws, size_t ws_bytes, void *stream);

/*
 * Adjoint solve A_b^T lambda_b = g_b ("Methodology" 2, linear systems: the
 * backward pass solves one adjoint system with right-hand side dL/dx).  With
 * SLA_FLAG_SYMMETRIC the forward pattern and values are used as they are;
 * otherwise A^T's values are gathered into the workspace first.
 * Same arguments and outcomes as sla_cg_solve (lambda plays x; dL/db = lambda).
 * ws >= sla_workspace_bytes(h, SLA_OP_ADJOINT).
 */
sla_status sla_cg_adjoint(sla_csr_t h, const void *vals, const void *g, void *lambda,
                          const sla_cg_opts *opts, sla_cg_info info,
                          void *ws, size_t ws_bytes, void *stream);

/*
 * Sparse value gradient ("Methodology" 2: dL/dA_ij = -lambda_i x_j on the
 * sparsity pattern only):  grad_b[t] = -lambda_b[i] * x_b[colind[t]] for entry
 * t of row i, or grad_b[t] += that value when accumulate != 0.
 * lambda [B][n_rows], x [B][n_cols], grad [B][nnz]; device.
 */
sla_status sla_grad_values(sla_csr_t h, const void *lambda, const void *x, void *grad,
                           int32_t accumulate, void *stream);

/*
 * Value gradient of the matrix-vector product ("Methodology" 1, `.matvec`, as an
 * autograd operation): for y_b = A_b x_b and an incoming gradient gy_b = dL/dy_b,
 * dL/dA_ij = gy_i * x_j on the stored entries only:  grad_b[t] = gy_b[i] *
 * x_b[colind[t]] for entry t of row i, or grad_b[t] += that value when
 * accumulate != 0.  gy [B][n_rows], x [B][n_cols], grad [B][nnz]; device.
 * Each entry is one rounded product (sla_grad_values with lambda = gy gives
 * its exact negation).
 */
sla_status sla_matvec_grad_values(sla_csr_t h, const void *gy, const void *x, void *grad,
                                  int32_t accumulate, void *stream);

/*
 * Transpose of a batched CSR matrix by a stable sort on the column index:
 * row c of A^T lists the entries of column c in increasing row order; values
 * are moved, never combined; perm[s] is the A-position of A^T's entry s.
 * Inputs device: rowptr[n_rows+1], colind[nnz], vals [B][nnz] (may be NULL to
 * skip values).  Outputs device: rowptrT[n_cols+1], colindT[nnz], valsT
 * [B][nnz] (ignored if vals is NULL), perm[nnz] (may be NULL only when vals
 * is NULL).  ws >= sla_transpose_workspace_bytes().  Bit-exact by
 * construction.  The pattern must be valid (see sla_csr_check).
 */
size_t sla_transpose_workspace_bytes(int32_t n_rows, int32_t n_cols, int64_t nnz);
sla_status sla_csr_transpose(int32_t n_rows, int32_t n_cols, int64_t nnz,
                             const int32_t *rowptr, const int32_t *colind,
                             int32_t batch, sla_dtype dtype, const void *vals,
                             int32_t *rowptrT, int32_t *colindT, void *valsT,
                             int32_t *perm, void *ws, size_t ws_bytes, void *stream);

/*
 * CSR from coordinate entries: entries ordered by (row, col) with a stable
 * sort; runs of equal (row, col) are summed left to right in input order.
 * Inputs device: row[nnz_in], col[nnz_in], val [B][nnz_in] (may be NULL).
 * Outputs device: rowptr[n_rows+1], colind[capacity nnz_in], val_out
 * [B][nnz_in] (row stride nnz_in; first *nnz_out entries of each row used),
 * slot[nnz_in] (output position of each input entry; may be NULL),
 * nnz_out (device int64[1]).  ws >= sla_coo_workspace_bytes().  Entries out of
 * range make the call write -1 to *nnz_out and leave the outputs undefined.
 */
size_t sla_coo_workspace_bytes(int32_t n_rows, int32_t n_cols, int64_t nnz_in);
sla_status sla_csr_from_coo(int32_t n_rows, int32_t n_cols, int64_t nnz_in,
                            const int32_t *row, const int32_t *col,
                            int32_t batch, sla_dtype dtype, const void *val,
                            int32_t *rowptr, int32_t *colind, void *val_out,
                            int32_t *slot, int64_t *nnz_out,
                            void *ws, size_t ws_bytes, void *stream);

/*
 * Pattern check on the GPU.  result: device int64[2] receives {code, where}:
 * 0 valid; 1 rowptr[0] != 0; 2 rowptr decreases at row `where`; 3 rowptr[n_rows]
 * != nnz; 4 column out of range at entry `where`; 5 columns not strictly
 * increasing at entry `where`; 6 (need_diag) row `where` has no diagonal.
 * When several problems exist, the lowest code wins and, within it, the lowest
 * index.  Enqueue-only.
 */
sla_status sla_csr_check(int32_t n_rows, int32_t n_cols, int64_t nnz,
                         const int32_t *rowptr, const int32_t *colind,
                         int32_t need_diag, int64_t *result, void *stream);

/*
 * Allocation-free variant of sla_cg_solve.  The pages have no counterpart: it
 * exists for callers that may not allocate device memory while they solve
 * (runtimes that reserve all device memory up front and hand it out
 * themselves, loops that cannot afford the device-wide synchronisation that
 * cudaMalloc/cudaFree may imply, plugins that must not call their host's
 * allocator).  It needs no handle and no workspace: it runs the persistent
 * grid solver with vectors in global memory, and its scratch (synchronisation
 * words, partial sums, diagonal positions, the r, p, q, M^-1 vectors) lives in
 * one static device array of 16 MiB that every GPU loading this library keeps
 * until the process exits.
 *   - Every call looks up the array's device address in the caller's current
 *     context (so a context switch or a device reset between calls is safe);
 *     the first call in a context also loads the library's device code into
 *     it, so make that first call before any stream capture.
 *   - Sizes whose scratch exceeds 16 MiB (about 4 + 4*sizeof(T) bytes per row
 *     and system, plus 32 bytes per tile) are rejected with SLA_ERR_INVALID
 *     and a message giving both sizes; it never allocates, not even then.
 *   - Every call on a device shares the array, which keeps what the last call
 *     left: the call clears what must start at zero, and calls whose kernels
 *     overlap on the GPU (other streams, other host threads) race on it.
 *   - The pattern is not validated (see sla_csr_check); rowptr/colind must be
 *     a valid square CSR pattern.
 * Arguments and outcomes are those of sla_cg_solve (rowptr[n+1], colind[nnz],
 * vals [B][nnz], b and x [B][n], all device; opts->strategy must not be
 * SLA_STRATEGY_BLOCK).
 */
sla_status sla_cg_solve_noalloc(int32_t n, int64_t nnz, const int32_t *rowptr,
                                const int32_t *colind, int32_t batch, sla_dtype dtype,
                                const void *vals, const void *b, void *x,
                                const sla_cg_opts *opts, sla_cg_info info, void *stream);

/*
 * A list of independent square systems, each with its own pattern (the
 * SparseTensorList of torch-sla, technical summary, "Methodology" 1: a batch
 * whose items have different patterns).  The caller stores the items as one
 * block-diagonal CSR: item s owns rows and columns [item_rows[s],
 * item_rows[s+1]) (device int32 [n_items + 1], read during the call only;
 * item_rows[0] = 0, non-decreasing, item_rows[n_items] = n_rows) and its
 * entries keep global column indices.  rowptr/colind are borrowed as for
 * sla_csr_create; flags as there (VALIDATE checks the CSR rules; the block
 * structure is always checked: an entry outside its item's block is
 * SLA_ERR_INVALID).  Synchronises the host.
 *
 * The handle has batch 1: values [nnz], vectors [n_rows].  sla_spmv and
 * sla_grad_values act on the whole block-diagonal matrix, which is each item's
 * own product.  sla_cg_solve / sla_cg_adjoint solve every item independently
 * (its own alpha, beta, stop test relative to its own ||b||) and write
 * sla_cg_info per item ([n_items]); strategy AUTO or BLOCK (each item runs in
 * one thread block, largest items first; items too large for shared memory
 * use the workspace vectors).
 */
sla_status sla_csr_list_create(int32_t n_items, const int32_t *item_rows, int32_t n_rows,
                               int64_t nnz, const int32_t *rowptr, const int32_t *colind,
                               sla_dtype dtype, uint32_t flags, void *stream, sla_csr_t *out);

/*
 * Edge-weighted graph Laplacian on a handle's pattern: the map from edge
 * conductivities to matrix values used by inverse coefficient learning
 * (torch-sla summary page, technical summary, "Experimental results",
 * end-to-end application: spatially varying conductivities of a Poisson
 * problem recovered through A.solve with a standard Adam loop).  The pages do
 * not spell the assembly out; this is the plain graph-Laplacian reading.  For
 * system b with weights w_b [E] and shift s_b:
 *   A_ij = A_ji = -w_e                  for edge e = (i, j), i != j;
 *   A_ii = (the weights of the edges at i, added one by one from 0 in
 *           ascending neighbour index) + s_b;
 *   every other stored entry = 0.
 * The gradient follows by the chain rule from G = dL/dvals (for a solve,
 * G_ij = -lambda_i x_j, "Methodology" 2):
 *   dL/dw_e = ((G_ii + G_jj) - G_ij) - G_ji,   dL/ds_b = sum_i G_ii.
 *
 * sla_edges_create maps undirected edges (device int32 ei[E], ej[E], read
 * only during the call) to their two pattern entries and keeps that map
 * (8 E + 4 nnz bytes of device memory, owned by the plan).  The handle must be
 * square and must outlive the plan.  It synchronises the host once.  Invalid
 * edges give SLA_ERR_INVALID; *check (host, may be NULL) receives
 * code << 40 | index of the failure with the smallest code, then the smallest
 * index (0 when valid):
 *   1 an endpoint outside [0, n)        (index: the edge)
 *   2 a self loop, i == j               (the edge)
 *   3 entry (i, j) or (j, i) not in the pattern   (the edge)
 *   4 an unordered pair that an earlier edge already names   (the later edge)
 *   5 a row without a diagonal entry    (the row)
 */
typedef struct sla_edges_s *sla_edges_t;
sla_status sla_edges_create(sla_csr_t h, int64_t n_edges, const int32_t *ei, const int32_t *ej,
                            int64_t *check, void *stream, sla_edges_t *out);
sla_status sla_edges_destroy(sla_edges_t e);

/* vals (device [B][nnz], the handle's dtype) = A(w, shift) for w (device
 * [B][E]) and shift (device [B], or NULL for 0).  Bit-exact: each entry is
 * one negation or the ordered sum above. */
sla_status sla_laplacian_assemble(sla_edges_t e, const void *w, const void *shift, void *vals,
                                  void *stream);

/* Workspace (256-byte aligned) of the two gradient calls below. */
size_t sla_edges_workspace_bytes(sla_edges_t e);

/* Flags of the two gradient calls below. */
enum {
    SLA_GRAD_ACCUMULATE = 1u,    /* add to dw / dshift instead of overwriting them */
    SLA_GRAD_SHIFT_SHARED = 2u   /* one shift serves every system: dshift is device [1]
                                    and receives dL/ds summed over all systems */
};

/* dw (device [B][E]) and dshift (device [B], or [1] with SLA_GRAD_SHIFT_SHARED;
 * may be NULL) from G (device [B][nnz]) by the chain rule above.  dw is
 * bit-exact (four entries added in the stated order); dshift is accumulated in
 * double over a fixed tree (over every system's diagonal with
 * SLA_GRAD_SHIFT_SHARED) and rounded once.  flags: SLA_GRAD_*. */
sla_status sla_laplacian_grad_values(sla_edges_t e, const void *G, void *dw, void *dshift,
                                     int32_t flags, void *ws, size_t ws_bytes, void *stream);

/* The same with G = -lambda x^T on the pattern (what sla_grad_values would
 * write), without forming G: each G entry is rounded exactly as
 * sla_grad_values rounds it, so dw equals sla_grad_values followed by
 * sla_laplacian_grad_values bit for bit.  lambda, x: device [B][n]. */
sla_status sla_laplacian_grad(sla_edges_t e, const void *lambda, const void *x, void *dw,
                              void *dshift, int32_t flags, void *ws, size_t ws_bytes,
                              void *stream);

/*
 * Bounds record of the bounds-checking build (libsla_debug_bounds.so, compiled
 * with SLA_DEBUG_BOUNDS=1).  There is no counterpart on the pages: this build
 * stands in for a memory checker.  Its kernels check every index they take from
 * the pattern (gathered columns, entry positions, diagonal positions, edge
 * slots) and every shared-memory or cluster-rank index derived from one before
 * using it; a bad index is recorded and replaced by 0, so the access stays in
 * bounds and no kernel traps.  This call waits for the device, then returns
 * the number of violations since the last reset (*violations), the smallest
 * code (1 column, 2 entry, 3 diagonal, 4 shared-memory or cluster index,
 * 5 edge; 0 if none) and that code's smallest index (-1 if none); with
 * reset != 0 it clears the record.  Any output pointer (host) may be NULL.
 * The regular library returns SLA_ERR_UNSUPPORTED.
 */
sla_status sla_debug_bounds_report(uint64_t *violations, int32_t *first_code, int64_t *first_index,
                                   int32_t reset);

/* Message for the last non-OK status on this host thread ("" if none). */
const char *sla_last_error_string(void);

/* Library version string. */
const char *sla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SLA_H */
