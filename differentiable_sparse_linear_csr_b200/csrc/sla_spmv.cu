// Batched CSR SpMV (the `.matvec` call) and the sparse value gradient
// dL/dA_ij = -lambda_i x_j on the stored entries, both row-parallel with
// LANES threads per row chosen from the pattern's mean row length.
//   torch-sla summary page, technical summary: "Methodology" 1 (`.matvec`)
//   and "Methodology" 2 (linear systems: gradient on the sparsity pattern).
#include "sla_rows.cuh"

namespace sla {

template <typename T, int LANES, bool PERM>
__global__ void __launch_bounds__(kRowBlock)
spmv_kernel(int n_rows, int64_t nnz, int64_t x_stride, int B, const int32_t *__restrict__ rowptr,
            const int32_t *__restrict__ colind, const int32_t *__restrict__ perm,
            const T *__restrict__ vals, const T *__restrict__ x, T *__restrict__ y, T alpha,
            T beta) {
    constexpr int RPB = kRowBlock / LANES;
    const int i = blockIdx.x * RPB + threadIdx.x / LANES;
    const int lane = threadIdx.x % LANES;
    if (i >= n_rows) return;  // a sub-warp shares i, so it leaves together
    for (int sys = blockIdx.y; sys < B; sys += gridDim.y) {
        const T *vb = vals + (int64_t)sys * nnz;
        const T *xb = x + (int64_t)sys * x_stride;
        T *yb = y + (int64_t)sys * n_rows;
        T s;
        if constexpr (PERM)
            s = row_dot_perm<T, LANES>(rowptr, colind, perm, vb, xb, i, lane);
        else
            s = row_dot<T, LANES>(rowptr, colind, vb, xb, i, lane);
        if (lane == 0) yb[i] = (beta == T(0)) ? alpha * s : alpha * s + beta * yb[i];
    }
}

// grad[t] = -(lambda[i] * x[colind[t]]) for entry t of row i (+= if accumulate).
template <typename T, int LANES>
__global__ void __launch_bounds__(kRowBlock)
grad_values_kernel(int n_rows, int n_cols, int64_t nnz, int B, const int32_t *__restrict__ rowptr,
                   const int32_t *__restrict__ colind, const T *__restrict__ lam,
                   const T *__restrict__ x, T *__restrict__ grad, int accumulate) {
    constexpr int RPB = kRowBlock / LANES;
    const int i = blockIdx.x * RPB + threadIdx.x / LANES;
    const int lane = threadIdx.x % LANES;
    if (i >= n_rows) return;
    const int t0 = __ldg(rowptr + i), t1 = __ldg(rowptr + i + 1);
    for (int sys = blockIdx.y; sys < B; sys += gridDim.y) {
        const T li = __ldg(lam + (int64_t)sys * n_rows + i);
        const T *xb = x + (int64_t)sys * n_cols;
        T *gb = grad + (int64_t)sys * nnz;
        for (int t = t0 + lane; t < t1; t += LANES) {
            const T g = -(li * __ldg(xb + __ldg(colind + t)));
            gb[t] = accumulate ? gb[t] + g : g;
        }
    }
}

static dim3 row_grid(int rows, int lanes, int B) {
    const int rpb = kRowBlock / lanes;
    return dim3((unsigned)((rows + rpb - 1) / rpb), (unsigned)(B < 65535 ? B : 65535));
}

}  // namespace sla

using namespace sla;

extern "C" sla_status sla_spmv(sla_csr_t hh, const void *vals, const void *x, void *y,
                               int32_t transpose, double alpha, double beta, void *stream) {
    clear_error();
    Csr *h = reinterpret_cast<Csr *>(hh);
    SLA_REQUIRE(h != nullptr, "sla_spmv: NULL handle");
    const bool tr = transpose != 0;
    const int rows = tr ? h->n_cols : h->n_rows;
    const int xlen = tr ? h->n_rows : h->n_cols;
    if (rows == 0) return SLA_OK;
    SLA_REQUIRE(y != nullptr, "sla_spmv: NULL y");
    SLA_REQUIRE(h->nnz == 0 || (vals != nullptr && x != nullptr), "sla_spmv: NULL vals or x");
    cudaStream_t s = as_stream(stream);
    const bool use_perm = tr && !((h->flags & SLA_FLAG_SYMMETRIC) && h->n_rows == h->n_cols);
    if (use_perm) {
        sla_status st = ensure_transpose(h, s);
        if (st != SLA_OK) return st;
    }
    const int32_t *rp = use_perm ? h->rowptrT : h->rowptr;
    const int32_t *ci = use_perm ? h->colindT : h->colind;
    const int lanes = use_perm ? lanes_for_mean(rows ? (double)h->nnz / rows : 0.0) : h->lanes;
    const dim3 grid = row_grid(rows, lanes, h->batch);
    return with_lanes(lanes, [&](auto L) -> sla_status {
        constexpr int LN = decltype(L)::value;
        if (h->dtype == SLA_F64) {
            if (use_perm)
                spmv_kernel<double, LN, true><<<grid, kRowBlock, 0, s>>>(
                    rows, h->nnz, xlen, h->batch, rp, ci, h->permT, (const double *)vals,
                    (const double *)x, (double *)y, alpha, beta);
            else
                spmv_kernel<double, LN, false><<<grid, kRowBlock, 0, s>>>(
                    rows, h->nnz, xlen, h->batch, rp, ci, nullptr, (const double *)vals,
                    (const double *)x, (double *)y, alpha, beta);
        } else {
            if (use_perm)
                spmv_kernel<float, LN, true><<<grid, kRowBlock, 0, s>>>(
                    rows, h->nnz, xlen, h->batch, rp, ci, h->permT, (const float *)vals,
                    (const float *)x, (float *)y, (float)alpha, (float)beta);
            else
                spmv_kernel<float, LN, false><<<grid, kRowBlock, 0, s>>>(
                    rows, h->nnz, xlen, h->batch, rp, ci, nullptr, (const float *)vals,
                    (const float *)x, (float *)y, (float)alpha, (float)beta);
        }
        SLA_CHECK_LAUNCH();
        return SLA_OK;
    });
}

extern "C" sla_status sla_grad_values(sla_csr_t hh, const void *lambda, const void *x,
                                      void *grad, int32_t accumulate, void *stream) {
    clear_error();
    Csr *h = reinterpret_cast<Csr *>(hh);
    SLA_REQUIRE(h != nullptr, "sla_grad_values: NULL handle");
    if (h->n_rows == 0 || h->nnz == 0) return SLA_OK;
    SLA_REQUIRE(lambda && x && grad, "sla_grad_values: NULL lambda, x or grad");
    cudaStream_t s = as_stream(stream);
    const dim3 grid = row_grid(h->n_rows, h->lanes, h->batch);
    return with_lanes(h->lanes, [&](auto L) -> sla_status {
        constexpr int LN = decltype(L)::value;
        if (h->dtype == SLA_F64)
            grad_values_kernel<double, LN><<<grid, kRowBlock, 0, s>>>(
                h->n_rows, h->n_cols, h->nnz, h->batch, h->rowptr, h->colind,
                (const double *)lambda, (const double *)x, (double *)grad, accumulate);
        else
            grad_values_kernel<float, LN><<<grid, kRowBlock, 0, s>>>(
                h->n_rows, h->n_cols, h->nnz, h->batch, h->rowptr, h->colind,
                (const float *)lambda, (const float *)x, (float *)grad, accumulate);
        SLA_CHECK_LAUNCH();
        return SLA_OK;
    });
}
