/*
 * Type-generic body of the CPU oracle; included by oracle.c once with T = double
 * (suffix f64) and once with T = float (suffix f32).  TEST INFRASTRUCTURE ONLY.
 *
 * Precision policy for T = float (the pages fix none; plainest reading): matrix
 * values, vectors and matrix-row sums are float; every dot product and norm is
 * accumulated in double; the scalars alpha, beta, rho are double and are rounded
 * to float only where they multiply a float vector.  For T = double everything
 * is double.  Arithmetic is plain C with floating-point contraction disabled at
 * compile time, so every product and sum is rounded separately.
 *
 * The OpenMP pragmas are inert in the oracle's own build (compiled without
 * -fopenmp).  The benchmark's all-cores CPU baseline compiles this same source
 * with -fopenmp: rows and vector entries are then split over threads, which
 * changes nothing in their arithmetic, and dot products are summed per thread
 * and then combined, which changes only the order of their additions.
 */

#define CAT_(a, b) a##_##b
#define CAT(a, b) CAT_(a, b)
#define FN(name) CAT(name, SUFFIX)

/*
 * Sparse matrix-vector product y = A x, the ".matvec" operation of torch-sla
 * (technical summary, "Methodology" 1, unified backend abstraction).  Row i's
 * entries are summed in stored (CSR) order, or in reverse order when
 * reverse != 0 (used only to measure the oracle's own rounding spread).
 */
void FN(orc_spmv)(int32_t n_rows, const int32_t *rowptr, const int32_t *colind,
                  const T *vals, const T *x, T *y, int32_t reverse)
{
    #pragma omp parallel for schedule(static)
    for (int32_t i = 0; i < n_rows; ++i) {
        T s = (T)0;
        if (!reverse) {
            for (int32_t t = rowptr[i]; t < rowptr[i + 1]; ++t)
                s = s + vals[t] * x[colind[t]];
        } else {
            for (int32_t t = rowptr[i + 1] - 1; t >= rowptr[i]; --t)
                s = s + vals[t] * x[colind[t]];
        }
        y[i] = s;
    }
}

static double FN(dot)(int32_t n, const T *a, const T *b, int32_t reverse)
{
    double s = 0.0;
    if (!reverse) {
        #pragma omp parallel for schedule(static) reduction(+:s)
        for (int32_t i = 0; i < n; ++i) s = s + (double)a[i] * (double)b[i];
    } else {
        for (int32_t i = n - 1; i >= 0; --i) s = s + (double)a[i] * (double)b[i];
    }
    return s;
}

/*
 * Jacobi-preconditioned conjugate gradient for a sparse SPD system A x = b, the
 * iterative solve of torch-sla's PyTorch-native GPU backend (technical summary,
 * "Methodology" 1; Jacobi preconditioning named under "Significance",
 * limitations).  The pages print no algorithm, so this is the textbook
 * Hestenes-Stiefel preconditioned CG with M = diag(A):
 *
 *   x = x0 (0 unless given);  r = b - A x;  z = M^-1 r;  p = z;  rho = r.z
 *   repeat:  q = A p;  sigma = p.q;  alpha = rho / sigma
 *            x += alpha p;  r -= alpha q;  k += 1
 *            stop when ||r|| <= max(rtol ||b||, atol)  (tolerance mode)
 *            z = M^-1 r;  rho' = r.z;  beta = rho' / rho;  p = z + beta p
 *
 * Stopping uses the recursively updated residual.  In fixed mode
 * (fixed_iters > 0) exactly fixed_iters steps run unless r becomes exactly zero
 * or the step breaks down.  sigma <= 0 is a breakdown (A not positive definite
 * along p); a non-finite sigma or ||r||^2 ends the solve as non-finite.
 */
int32_t FN(orc_pcg)(int32_t n, const int32_t *rowptr, const int32_t *colind,
                    const T *vals, const T *b, T *x, const orc_opts *opt,
                    orc_result *res)
{
    const int32_t rev = opt->reverse_order;
    const int32_t fixed = opt->fixed_iters > 0;
    const int32_t limit = fixed ? opt->fixed_iters : opt->max_iter;
    T *r = (T *)malloc(sizeof(T) * (size_t)(n > 0 ? n : 1));
    T *p = (T *)malloc(sizeof(T) * (size_t)(n > 0 ? n : 1));
    T *q = (T *)malloc(sizeof(T) * (size_t)(n > 0 ? n : 1));
    T *dinv = (T *)malloc(sizeof(T) * (size_t)(n > 0 ? n : 1));
    if (!r || !p || !q || !dinv) { free(r); free(p); free(q); free(dinv); return -1; }

    res->iters = 0;
    res->relres = 0.0;
    res->status = ORC_CONVERGED;

    /* M = diag(A): dinv_i = 1 / A_ii, or 1 without preconditioning. */
    int32_t bad_diag = 0;
    #pragma omp parallel for schedule(static) reduction(|:bad_diag)
    for (int32_t i = 0; i < n; ++i) {
        T d = (T)0;
        for (int32_t t = rowptr[i]; t < rowptr[i + 1]; ++t)
            if (colind[t] == i) d = vals[t];
        if (opt->precond) {
            if (!(d > (T)0)) bad_diag = 1;
            dinv[i] = (T)1 / d;
        } else {
            dinv[i] = (T)1;
        }
    }

    const double nb = sqrt(FN(dot)(n, b, b, rev));
    if (!opt->x0_given)
        for (int32_t i = 0; i < n; ++i) x[i] = (T)0;
    if (nb == 0.0) {
        for (int32_t i = 0; i < n; ++i) x[i] = (T)0;
        free(r); free(p); free(q); free(dinv);
        return 0;
    }
    if (!isfinite(nb)) {
        res->status = ORC_NONFINITE;
        free(r); free(p); free(q); free(dinv);
        return 0;
    }
    if (opt->x0_given) {
        FN(orc_spmv)(n, rowptr, colind, vals, x, q, rev);
        #pragma omp parallel for schedule(static)
        for (int32_t i = 0; i < n; ++i) r[i] = b[i] - q[i];
    } else {
        #pragma omp parallel for schedule(static)
        for (int32_t i = 0; i < n; ++i) r[i] = b[i];
    }
    if (opt->precond && bad_diag) {
        /* M = diag(A) is not positive definite: A cannot be SPD. */
        res->status = ORC_BREAKDOWN;
        res->relres = sqrt(FN(dot)(n, r, r, rev)) / nb;
        free(r); free(p); free(q); free(dinv);
        return 0;
    }
    #pragma omp parallel for schedule(static)
    for (int32_t i = 0; i < n; ++i) p[i] = dinv[i] * r[i];
    double rho = FN(dot)(n, r, p, rev);
    double rr = FN(dot)(n, r, r, rev);
    const double tol = fmax(opt->rtol * nb, opt->atol);

    int32_t k = 0;
    int32_t status = fixed ? ORC_FIXED_DONE : ORC_NOT_CONVERGED;
    if (!fixed && sqrt(rr) <= tol) status = ORC_CONVERGED;
    else if (rr == 0.0) status = ORC_CONVERGED;
    else {
        while (k < limit) {
            FN(orc_spmv)(n, rowptr, colind, vals, p, q, rev);
            const double sigma = FN(dot)(n, p, q, rev);
            if (!isfinite(sigma)) { status = ORC_NONFINITE; break; }
            if (!(sigma > 0.0)) { status = ORC_BREAKDOWN; break; }
            const double alpha = rho / sigma;
            const T a = (T)alpha;
            #pragma omp parallel for schedule(static)
            for (int32_t i = 0; i < n; ++i) x[i] = x[i] + a * p[i];
            #pragma omp parallel for schedule(static)
            for (int32_t i = 0; i < n; ++i) r[i] = r[i] - a * q[i];
            k = k + 1;
            rr = FN(dot)(n, r, r, rev);
            if (!isfinite(rr)) { status = ORC_NONFINITE; break; }
            if (!fixed && sqrt(rr) <= tol) { status = ORC_CONVERGED; break; }
            if (rr == 0.0) { status = ORC_CONVERGED; break; }
            if (k == limit) break;
            #pragma omp parallel for schedule(static)
            for (int32_t i = 0; i < n; ++i) q[i] = dinv[i] * r[i];   /* q holds z */
            const double rho_new = FN(dot)(n, r, q, rev);
            const double beta = rho_new / rho;
            const T bt = (T)beta;
            #pragma omp parallel for schedule(static)
            for (int32_t i = 0; i < n; ++i) p[i] = q[i] + bt * p[i];
            rho = rho_new;
        }
    }
    res->iters = k;
    res->status = status;
    res->relres = sqrt(rr) / nb;
    free(r); free(p); free(q); free(dinv);
    return 0;
}

/*
 * Gradient of L with respect to the stored values, from the linear adjoint rule
 * of torch-sla (technical summary, "Methodology" 2, linear systems): with
 * A^T lambda = dL/dx solved, dL/dA_ij = -lambda_i x_j, on the sparsity pattern
 * only.  grad[t] = -(lambda[i] * x[colind[t]]) for entry t of row i; when
 * accumulate != 0 it is added to grad[t] instead of stored.
 */
void FN(orc_grad_values)(int32_t n_rows, const int32_t *rowptr, const int32_t *colind,
                         const T *lambda, const T *x, T *grad, int32_t accumulate)
{
    #pragma omp parallel for schedule(static)
    for (int32_t i = 0; i < n_rows; ++i)
        for (int32_t t = rowptr[i]; t < rowptr[i + 1]; ++t) {
            const T g = -(lambda[i] * x[colind[t]]);
            grad[t] = accumulate ? grad[t] + g : g;
        }
}

/*
 * Adjoint solve A^T lambda = g of the linear adjoint rule (technical summary,
 * "Methodology" 2).  The transpose is built explicitly, by the oracle's own
 * stable transpose, even when A is symmetric; then the same PCG runs on it.
 */
int32_t FN(orc_cg_adjoint)(int32_t n, const int32_t *rowptr, const int32_t *colind,
                           const T *vals, const T *g, T *lambda, const orc_opts *opt,
                           orc_result *res)
{
    const int32_t nnz = rowptr[n];
    int32_t *rpT = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n + 1));
    int32_t *ciT = (int32_t *)malloc(sizeof(int32_t) * (size_t)(nnz > 0 ? nnz : 1));
    int64_t *perm = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nnz > 0 ? nnz : 1));
    T *vT = (T *)malloc(sizeof(T) * (size_t)(nnz > 0 ? nnz : 1));
    if (!rpT || !ciT || !perm || !vT) { free(rpT); free(ciT); free(perm); free(vT); return -1; }
    orc_transpose_pattern(n, n, rowptr, colind, rpT, ciT, perm);
    #pragma omp parallel for schedule(static)
    for (int32_t t = 0; t < nnz; ++t) vT[t] = vals[perm[t]];
    const int32_t rc = FN(orc_pcg)(n, rpT, ciT, vT, g, lambda, opt, res);
    free(rpT); free(ciT); free(perm); free(vT);
    return rc;
}

/*
 * Edge-weighted graph Laplacian plus a diagonal shift, written into the values
 * of a given pattern (the conductivity-to-matrix map of inverse coefficient
 * learning, torch-sla summary page, "Experimental results", end-to-end
 * application; the pages leave the assembly open, so this is the plain
 * graph-Laplacian reading):
 *   A_ij = A_ji = -w_e for every edge e = (i, j);
 *   A_ii = (the weights of the edges at i, added one by one from 0 in
 *           ascending neighbour index) + shift;
 *   every other stored entry 0.
 * owner[] is orc_edge_slots' (rows hold strictly increasing columns, so a row
 * walk in stored order visits the neighbours in ascending index).
 */
void FN(orc_laplacian_assemble)(int32_t n, const int32_t *rowptr, const int32_t *colind,
                                const int64_t *owner, const T *w, T shift, T *vals)
{
    for (int32_t i = 0; i < n; ++i) {
        T d = (T)0;
        int64_t dpos = -1;
        for (int32_t t = rowptr[i]; t < rowptr[i + 1]; ++t) {
            if (colind[t] == i) {
                dpos = t;
            } else if (owner[t] >= 0) {
                vals[t] = -w[owner[t]];
                d = d + w[owner[t]];
            } else {
                vals[t] = (T)0;
            }
        }
        if (dpos >= 0) vals[dpos] = d + shift;
    }
}

/*
 * Chain rule through orc_laplacian_assemble: with G = dL/dvals,
 *   dL/dw_e = G_ii + G_jj - G_ij - G_ji   (added left to right),
 *   dL/dshift = sum_i G_ii                (accumulated in double, rounded to T).
 * With accumulate != 0 both are added to dw / *dshift instead of stored.
 */
void FN(orc_laplacian_grad_values)(int32_t n, const int32_t *rowptr, const int32_t *colind,
                                   int64_t n_edges, const int32_t *ei, const int32_t *ej,
                                   const int64_t *slot_ij, const int64_t *slot_ji,
                                   const T *G, T *dw, T *dshift, int32_t accumulate)
{
    int32_t *dpos = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
    if (!dpos) return;
    orc_diag_positions(n, rowptr, colind, dpos);
    for (int64_t e = 0; e < n_edges; ++e) {
        const T v = ((G[dpos[ei[e]]] + G[dpos[ej[e]]]) - G[slot_ij[e]]) - G[slot_ji[e]];
        dw[e] = accumulate ? dw[e] + v : v;
    }
    double s = 0.0;
    for (int32_t i = 0; i < n; ++i) s = s + (double)G[dpos[i]];
    *dshift = accumulate ? *dshift + (T)s : (T)s;
    free(dpos);
}


/*
 * CSR from coordinate (COO) entries: entries are ordered by (row, col) with a
 * stable sort, so equal (row, col) entries keep their input order, and each run
 * of duplicates is summed left to right in that order.  Writes rowptr[n_rows+1],
 * colind/val_out (capacity nnz_in) and returns the number of stored entries.
 * slot[e] receives the output position of input entry e.
 */
int64_t FN(orc_coo_to_csr)(int32_t n_rows, int32_t n_cols, int64_t nnz_in,
                           const int32_t *row, const int32_t *col, const T *val,
                           int32_t *rowptr, int32_t *colind, T *val_out, int64_t *slot)
{
    int64_t *order = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nnz_in > 0 ? nnz_in : 1));
    if (!order) return -1;
    orc_coo_order(n_rows, n_cols, nnz_in, row, col, order);
    for (int32_t i = 0; i <= n_rows; ++i) rowptr[i] = 0;
    int64_t m = 0;
    for (int64_t s = 0; s < nnz_in; ++s) {
        const int64_t e = order[s];
        if (s > 0 && row[e] == row[order[s - 1]] && col[e] == col[order[s - 1]]) {
            val_out[m - 1] = val_out[m - 1] + val[e];
        } else {
            colind[m] = col[e];
            val_out[m] = val[e];
            rowptr[row[e] + 1] += 1;
            m = m + 1;
        }
        slot[e] = m - 1;
    }
    for (int32_t i = 0; i < n_rows; ++i) rowptr[i + 1] += rowptr[i];
    free(order);
    return m;
}

#undef FN
#undef CAT
#undef CAT_
