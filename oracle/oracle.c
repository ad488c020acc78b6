/*
 * CPU oracle for the differentiable sparse SPD solve (Jacobi-preconditioned CG
 * with the implicit-function-theorem adjoint) described in "torch-sla:
 * Differentiable Sparse Linear Algebra with Adjoint Solvers and Sparse Tensor
 * Parallelism for PyTorch" (technical summary, "Methodology" 1 and 2).
 *
 * TEST INFRASTRUCTURE ONLY.  This is the plain, slow, single-threaded
 * definition that the CUDA library is checked against.  Only the test suite,
 * the package smoke check and the benchmark's CPU-baseline leg may load it;
 * the library never does, and the two share no source.
 *
 * Build:  gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared oracle.c -lm
 * (contraction off: every product and sum is rounded on its own).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Per-solve outcome codes. */
enum { ORC_CONVERGED = 0, ORC_NOT_CONVERGED = 1, ORC_BREAKDOWN = 2,
       ORC_NONFINITE = 3, ORC_FIXED_DONE = 4 };

typedef struct {
    double rtol;            /* stop when ||r|| <= max(rtol*||b||, atol) */
    double atol;
    int32_t max_iter;       /* iteration cap in tolerance mode */
    int32_t fixed_iters;    /* > 0: run exactly this many iterations */
    int32_t precond;        /* 1: Jacobi M = diag(A); 0: none */
    int32_t x0_given;       /* 1: x holds the initial guess on entry */
    int32_t reverse_order;  /* 1: reverse every summation (rounding-spread probe) */
} orc_opts;

typedef struct {
    int32_t iters;
    int32_t status;
    double relres;          /* recursive ||r_k|| / ||b|| */
} orc_result;

/*
 * Transposed pattern by a stable counting sort on the column index: entries of
 * column c appear in A^T's row c in increasing original row order.  perm[s] is
 * the position in A of the entry stored at position s of A^T, so A^T's values
 * are vals[perm[s]]: moved, never combined.
 */
void orc_transpose_pattern(int32_t n_rows, int32_t n_cols, const int32_t *rowptr,
                           const int32_t *colind, int32_t *rowptrT, int32_t *colindT,
                           int64_t *perm)
{
    for (int32_t c = 0; c <= n_cols; ++c) rowptrT[c] = 0;
    for (int32_t t = 0; t < rowptr[n_rows]; ++t) rowptrT[colind[t] + 1] += 1;
    for (int32_t c = 0; c < n_cols; ++c) rowptrT[c + 1] += rowptrT[c];
    int32_t *next = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_cols > 0 ? n_cols : 1));
    for (int32_t c = 0; c < n_cols; ++c) next[c] = rowptrT[c];
    for (int32_t i = 0; i < n_rows; ++i)
        for (int32_t t = rowptr[i]; t < rowptr[i + 1]; ++t) {
            const int32_t s = next[colind[t]]++;
            colindT[s] = i;
            perm[s] = t;
        }
    free(next);
}

/*
 * Order of COO entries sorted by (row, col), stable: two stable counting sorts,
 * first by column, then by row (least significant key first).
 */
void orc_coo_order(int32_t n_rows, int32_t n_cols, int64_t nnz, const int32_t *row,
                   const int32_t *col, int64_t *order)
{
    int64_t *tmp = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nnz > 0 ? nnz : 1));
    int64_t nk = (n_rows > n_cols ? n_rows : n_cols) + 1;
    int64_t *cnt = (int64_t *)malloc(sizeof(int64_t) * (size_t)nk);
    /* pass 1: by column */
    for (int64_t k = 0; k < nk; ++k) cnt[k] = 0;
    for (int64_t e = 0; e < nnz; ++e) cnt[col[e] + 1] += 1;
    for (int64_t k = 1; k < nk; ++k) cnt[k] += cnt[k - 1];
    for (int64_t e = 0; e < nnz; ++e) tmp[cnt[col[e]]++] = e;
    /* pass 2: by row, stable over pass 1 */
    for (int64_t k = 0; k < nk; ++k) cnt[k] = 0;
    for (int64_t e = 0; e < nnz; ++e) cnt[row[e] + 1] += 1;
    for (int64_t k = 1; k < nk; ++k) cnt[k] += cnt[k - 1];
    for (int64_t s = 0; s < nnz; ++s) {
        const int64_t e = tmp[s];
        order[cnt[row[e]]++] = e;
    }
    free(tmp);
    free(cnt);
}

/*
 * Pattern checks of a CSR matrix.  Returns 0 when valid, else a code and the
 * first offending index in *where:
 *   1 rowptr[0] != 0            2 rowptr decreases at row *where
 *   3 rowptr[n_rows] != nnz     4 column out of [0, n_cols) at entry *where
 *   5 columns of a row not strictly increasing at entry *where
 *   6 (need_diag) row *where has no diagonal entry
 */
int32_t orc_csr_check(int32_t n_rows, int32_t n_cols, int64_t nnz, const int32_t *rowptr,
                      const int32_t *colind, int32_t need_diag, int64_t *where)
{
    *where = -1;
    if (rowptr[0] != 0) { *where = 0; return 1; }
    for (int32_t i = 0; i < n_rows; ++i)
        if (rowptr[i + 1] < rowptr[i]) { *where = i; return 2; }
    if ((int64_t)rowptr[n_rows] != nnz) { *where = n_rows; return 3; }
    for (int64_t t = 0; t < nnz; ++t)
        if (colind[t] < 0 || colind[t] >= n_cols) { *where = t; return 4; }
    for (int32_t i = 0; i < n_rows; ++i)
        for (int32_t t = rowptr[i] + 1; t < rowptr[i + 1]; ++t)
            if (colind[t] <= colind[t - 1]) { *where = t; return 5; }
    if (need_diag)
        for (int32_t i = 0; i < n_rows; ++i) {
            int32_t found = 0;
            for (int32_t t = rowptr[i]; t < rowptr[i + 1]; ++t)
                if (colind[t] == i) found = 1;
            if (!found) { *where = i; return 6; }
        }
    return 0;
}

/* Position of the diagonal entry of each row, -1 when the row has none. */
void orc_diag_positions(int32_t n_rows, const int32_t *rowptr, const int32_t *colind,
                        int32_t *diag_pos)
{
    for (int32_t i = 0; i < n_rows; ++i) {
        diag_pos[i] = -1;
        for (int32_t t = rowptr[i]; t < rowptr[i + 1]; ++t)
            if (colind[t] == i) diag_pos[i] = t;
    }
}

/*
 * Dense solve by Gaussian elimination with partial pivoting (row-major a[n][n],
 * overwritten; b overwritten by the solution).  Returns 0, or 1 if singular.
 * Used only to pin the iterative oracle on tiny systems.
 */
int32_t orc_dense_lu_solve(int32_t n, double *a, double *b)
{
    for (int32_t k = 0; k < n; ++k) {
        int32_t piv = k;
        for (int32_t i = k + 1; i < n; ++i)
            if (fabs(a[(size_t)i * n + k]) > fabs(a[(size_t)piv * n + k])) piv = i;
        if (a[(size_t)piv * n + k] == 0.0) return 1;
        if (piv != k) {
            for (int32_t j = 0; j < n; ++j) {
                double t = a[(size_t)k * n + j];
                a[(size_t)k * n + j] = a[(size_t)piv * n + j];
                a[(size_t)piv * n + j] = t;
            }
            double t = b[k]; b[k] = b[piv]; b[piv] = t;
        }
        for (int32_t i = k + 1; i < n; ++i) {
            const double l = a[(size_t)i * n + k] / a[(size_t)k * n + k];
            for (int32_t j = k; j < n; ++j) a[(size_t)i * n + j] -= l * a[(size_t)k * n + j];
            b[i] -= l * b[k];
        }
    }
    for (int32_t i = n - 1; i >= 0; --i) {
        double s = b[i];
        for (int32_t j = i + 1; j < n; ++j) s -= a[(size_t)i * n + j] * b[j];
        b[i] = s / a[(size_t)i * n + i];
    }
    return 0;
}

/*
 * Pattern positions of an undirected edge list, for the edge-weighted Laplacian
 * of inverse coefficient learning (torch-sla summary page, "Experimental
 * results", end-to-end application: spatially varying conductivities of a
 * Poisson problem recovered through A.solve by gradient descent).  Edge e joins
 * ei[e] and ej[e]; its two entries (i, j) and (j, i) are found by scanning rows
 * i and j.  owner[t] = the edge whose weight entry t carries, -1 for entries
 * that carry none (the diagonal and entries no edge names).  Every failure is
 * a pair (code, index); the smallest code, then the smallest index, is
 * returned with *where = that index (0 and -1 when the edges are valid):
 *   1 an endpoint outside [0, n)           (index: the edge)
 *   2 a self loop, i == j                  (the edge)
 *   3 entry (i, j) or (j, i) not stored    (the edge)
 *   4 an unordered pair an earlier edge already named  (the later edge)
 *   5 a row without a diagonal entry       (the row)
 */
int32_t orc_edge_slots(int32_t n, const int32_t *rowptr, const int32_t *colind,
                       int64_t n_edges, const int32_t *ei, const int32_t *ej,
                       int64_t *slot_ij, int64_t *slot_ji, int64_t *owner, int64_t *where)
{
    int32_t best = 0;
    int64_t best_at = -1;
#define ORC_FAIL(c, at) do { if (best == 0 || (c) < best || ((c) == best && (at) < best_at)) \
                                 { best = (c); best_at = (at); } } while (0)
    for (int64_t t = 0; t < (int64_t)rowptr[n]; ++t) owner[t] = -1;
    for (int64_t e = 0; e < n_edges; ++e) {
        const int32_t i = ei[e], j = ej[e];
        slot_ij[e] = slot_ji[e] = -1;
        if (i < 0 || i >= n || j < 0 || j >= n) { ORC_FAIL(1, e); continue; }
        if (i == j) { ORC_FAIL(2, e); continue; }
        for (int32_t t = rowptr[i]; t < rowptr[i + 1]; ++t)
            if (colind[t] == j) slot_ij[e] = t;
        for (int32_t t = rowptr[j]; t < rowptr[j + 1]; ++t)
            if (colind[t] == i) slot_ji[e] = t;
        if (slot_ij[e] < 0 || slot_ji[e] < 0) { ORC_FAIL(3, e); continue; }
        if (owner[slot_ij[e]] >= 0 || owner[slot_ji[e]] >= 0) { ORC_FAIL(4, e); continue; }
        owner[slot_ij[e]] = e;
        owner[slot_ji[e]] = e;
    }
    for (int32_t i = 0; i < n; ++i) {
        int32_t found = 0;
        for (int32_t t = rowptr[i]; t < rowptr[i + 1]; ++t)
            if (colind[t] == i) found = 1;
        if (!found) ORC_FAIL(5, i);
    }
#undef ORC_FAIL
    *where = best_at;
    return best;
}

#define T double
#define SUFFIX f64
#include "oracle_body.h"
#undef T
#undef SUFFIX

#define T float
#define SUFFIX f32
#include "oracle_body.h"
#undef T
#undef SUFFIX
