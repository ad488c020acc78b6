// Batched CSR SpMV (the `.matvec` call) and the sparse value gradients on the
// stored entries: dL/dA_ij = -lambda_i x_j after a solve, and dL/dA_ij =
// gy_i x_j for y = A x.
//   torch-sla summary page, technical summary: "Methodology" 1 (`.matvec`)
//   and "Methodology" 2 (linear systems: gradient on the sparsity pattern).
//
// Short rows (one thread a row): a block takes 256 consecutive rows, whose
// entries are one contiguous range of the CSR arrays.  The block copies that
// range's column indices (and, per system, values) into shared memory with
// coalesced loads, so every global read of the pattern and the values and
// every gradient store is a whole-sector access; the per-row work then reads
// shared memory and gathers x.  A row keeps its stored-order sum (the same
// rounding as a thread walking the row in global memory).  Chunks whose range
// exceeds the shared-memory capacity fall back to that direct walk.
// Long rows (LANES > 1 threads a row) are walked by sub-warps, which already
// read consecutive entries.
#include "sla_rows.cuh"

namespace sla {

constexpr int kChunkRows = 256;          // rows (and threads) of one staged block

// Entries a staged block holds: room for rows 4 entries longer than the mean,
// at most 4096; a chunk with more entries walks its rows in global memory.
static int chunk_cap(double row_mean) {
    const double c = kChunkRows * (row_mean + 4.0);
    return c >= 4096.0 ? 4096 : ((int)c + 31) / 32 * 32;
}

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
            s = row_dot_perm<T, LANES>(rowptr, colind, perm, vb, xb, i, lane, (int)x_stride, nnz);
        else
            s = row_dot<T, LANES>(rowptr, colind, vb, xb, i, lane, (int)x_stride, nnz);
        if (lane == 0) yb[i] = (beta == T(0)) ? alpha * s : alpha * s + beta * yb[i];
    }
}

// y = alpha A x + beta y for one-thread rows, the chunk's pattern and values
// staged in shared memory (see the file comment).
template <typename T>
__global__ void __launch_bounds__(kChunkRows)
spmv_staged_kernel(int n_rows, int64_t nnz, int64_t x_stride, int B, const int32_t *__restrict__ rowptr,
                   const int32_t *__restrict__ colind, const T *__restrict__ vals,
                   const T *__restrict__ x, T *__restrict__ y, T alpha, T beta, int cap) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *s_vals = reinterpret_cast<T *>(smem_raw);                 // [cap]
    int32_t *s_cols = reinterpret_cast<int32_t *>(s_vals + cap);  // [cap]
    const int tid = threadIdx.x;
    const int r0 = blockIdx.x * kChunkRows, r1 = min(n_rows, r0 + kChunkRows);
    const int i = r0 + tid;
    const int e0 = __ldg(rowptr + r0), e1 = __ldg(rowptr + r1);
    const int t0 = i < r1 ? __ldg(rowptr + i) : 0, t1 = i < r1 ? __ldg(rowptr + i + 1) : 0;
    const bool staged = e1 - e0 <= cap;
    if (staged) {
#pragma unroll 4
        for (int t = e0 + tid; t < e1; t += kChunkRows)
            s_cols[t - e0] = __ldg(colind + SLA_IDX(t, nnz, kBndEntry));
    }
    for (int sys = blockIdx.y; sys < B; sys += gridDim.y) {
        const T *vb = vals + (int64_t)sys * nnz;
        const T *xb = x + (int64_t)sys * x_stride;
        T s = T(0);
        if (staged) {
#pragma unroll 4
            for (int t = e0 + tid; t < e1; t += kChunkRows) s_vals[t - e0] = __ldg(vb + SLA_IDX(t, nnz, kBndEntry));
            __syncthreads();
#pragma unroll 4
            for (int t = t0; t < t1; ++t)
                s += s_vals[t - e0] * __ldg(xb + SLA_IDX(s_cols[t - e0], x_stride, kBndColumn));
            __syncthreads();
        } else {
            for (int t = t0; t < t1; ++t) {
                const int tt = SLA_IDX(t, nnz, kBndEntry);
                s += __ldg(vb + tt) * __ldg(xb + SLA_IDX(__ldg(colind + tt), x_stride, kBndColumn));
            }
        }
        if (i < r1) {
            T *yb = y + (int64_t)sys * n_rows;
            yb[i] = (beta == T(0)) ? alpha * s : alpha * s + beta * yb[i];
        }
    }
}

// grad[t] = -(lambda[i] * x[colind[t]]) for entry t of row i, or +(u[i] x[...])
// when NEG is false (+= if accumulate); LANES threads a row.
template <typename T, int LANES, bool NEG>
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
            const int tt = SLA_IDX(t, nnz, kBndEntry);
            const T p = li * __ldg(xb + SLA_IDX(__ldg(colind + tt), n_cols, kBndColumn));
            const T g = NEG ? -p : p;
            gb[tt] = accumulate ? gb[tt] + g : g;
        }
    }
}

// The same for one-thread rows, entry-parallel over the chunk: each thread
// first marks the chunk slots of its row with the row's position, then the
// block walks the slots in order, so column reads and gradient stores are
// coalesced.  Each entry is the same single product as above.
template <typename T, bool NEG>
__global__ void __launch_bounds__(kChunkRows)
grad_staged_kernel(int n_rows, int n_cols, int64_t nnz, int B, const int32_t *__restrict__ rowptr,
                   const int32_t *__restrict__ colind, const T *__restrict__ lam,
                   const T *__restrict__ x, T *__restrict__ grad, int accumulate, int cap) {
    extern __shared__ uint8_t s_row[];   // [cap]: position of each slot's row in the chunk
    const int tid = threadIdx.x;
    const int r0 = blockIdx.x * kChunkRows, r1 = min(n_rows, r0 + kChunkRows);
    const int i = r0 + tid;
    const int e0 = __ldg(rowptr + r0), e1 = __ldg(rowptr + r1);
    const int t0 = i < r1 ? __ldg(rowptr + i) : 0, t1 = i < r1 ? __ldg(rowptr + i + 1) : 0;
    const bool staged = e1 - e0 <= cap;
    if (staged) {
        for (int t = t0; t < t1; ++t) s_row[t - e0] = (uint8_t)tid;
        __syncthreads();
    }
    for (int sys = blockIdx.y; sys < B; sys += gridDim.y) {
        const T *lb = lam + (int64_t)sys * n_rows + r0;
        const T *xb = x + (int64_t)sys * n_cols;
        T *gb = grad + (int64_t)sys * nnz;
        if (staged) {
#pragma unroll 4
            for (int t = e0 + tid; t < e1; t += kChunkRows) {
                const int tt = SLA_IDX(t, nnz, kBndEntry);
                const T p = __ldg(lb + s_row[t - e0]) * __ldg(xb + SLA_IDX(__ldg(colind + tt), n_cols, kBndColumn));
                const T g = NEG ? -p : p;
                gb[tt] = accumulate ? gb[tt] + g : g;
            }
        } else if (i < r1) {
            const T li = __ldg(lb + tid);
            for (int t = t0; t < t1; ++t) {
                const int tt = SLA_IDX(t, nnz, kBndEntry);
                const T p = li * __ldg(xb + SLA_IDX(__ldg(colind + tt), n_cols, kBndColumn));
                const T g = NEG ? -p : p;
                gb[tt] = accumulate ? gb[tt] + g : g;
            }
        }
    }
}

static dim3 row_grid(int rows, int lanes, int B) {
    const int rpb = kRowBlock / lanes;
    return dim3((unsigned)((rows + rpb - 1) / rpb), (unsigned)(B < 65535 ? B : 65535));
}

static dim3 chunk_grid(int rows, int B) {
    return dim3((unsigned)((rows + kChunkRows - 1) / kChunkRows), (unsigned)(B < 65535 ? B : 65535));
}

template <bool NEG>
static sla_status grad_entry(const char *name, sla_csr_t hh, const void *u, const void *x, void *grad,
                             int32_t accumulate, void *stream) {
    clear_error();
    Csr *h = reinterpret_cast<Csr *>(hh);
    SLA_REQUIRE(h != nullptr, "%s: NULL handle", name);
    if (h->n_rows == 0 || h->nnz == 0) return SLA_OK;
    SLA_REQUIRE(u && x && grad, "%s: NULL vector or grad", name);
    cudaStream_t s = as_stream(stream);
    if (h->lanes == 1) {
        const dim3 grid = chunk_grid(h->n_rows, h->batch);
        const int cap = chunk_cap(h->row_mean);
        if (h->dtype == SLA_F64)
            grad_staged_kernel<double, NEG><<<grid, kChunkRows, cap, s>>>(
                h->n_rows, h->n_cols, h->nnz, h->batch, h->rowptr, h->colind, (const double *)u,
                (const double *)x, (double *)grad, accumulate, cap);
        else
            grad_staged_kernel<float, NEG><<<grid, kChunkRows, cap, s>>>(
                h->n_rows, h->n_cols, h->nnz, h->batch, h->rowptr, h->colind, (const float *)u,
                (const float *)x, (float *)grad, accumulate, cap);
        SLA_CHECK_LAUNCH();
        return SLA_OK;
    }
    const dim3 grid = row_grid(h->n_rows, h->lanes, h->batch);
    return with_lanes(h->lanes, [&](auto L) -> sla_status {
        constexpr int LN = decltype(L)::value;
        if (h->dtype == SLA_F64)
            grad_values_kernel<double, LN, NEG><<<grid, kRowBlock, 0, s>>>(
                h->n_rows, h->n_cols, h->nnz, h->batch, h->rowptr, h->colind,
                (const double *)u, (const double *)x, (double *)grad, accumulate);
        else
            grad_values_kernel<float, LN, NEG><<<grid, kRowBlock, 0, s>>>(
                h->n_rows, h->n_cols, h->nnz, h->batch, h->rowptr, h->colind,
                (const float *)u, (const float *)x, (float *)grad, accumulate);
        SLA_CHECK_LAUNCH();
        return SLA_OK;
    });
}

}  // namespace sla

using namespace sla;

extern "C" sla_status sla_spmv(sla_csr_t hh, const void *vals, const void *x, void *y,
                               int32_t transpose, double alpha, double beta, void *stream) {
    SLA_RANGE("sla_spmv");
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
    if (!use_perm && lanes == 1) {
        const dim3 grid = chunk_grid(rows, h->batch);
        const int cap = chunk_cap(h->row_mean);
        const size_t smem = (size_t)cap * (dtype_size(h->dtype) + sizeof(int32_t));
        if (h->dtype == SLA_F64)
            spmv_staged_kernel<double><<<grid, kChunkRows, smem, s>>>(
                rows, h->nnz, xlen, h->batch, rp, ci, (const double *)vals, (const double *)x,
                (double *)y, alpha, beta, cap);
        else
            spmv_staged_kernel<float><<<grid, kChunkRows, smem, s>>>(
                rows, h->nnz, xlen, h->batch, rp, ci, (const float *)vals, (const float *)x,
                (float *)y, (float)alpha, (float)beta, cap);
        SLA_CHECK_LAUNCH();
        return SLA_OK;
    }
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
    SLA_RANGE("sla_grad_values");
    return grad_entry<true>("sla_grad_values", hh, lambda, x, grad, accumulate, stream);
}

extern "C" sla_status sla_matvec_grad_values(sla_csr_t hh, const void *gy, const void *x,
                                             void *grad, int32_t accumulate, void *stream) {
    SLA_RANGE("sla_matvec_grad_values");
    return grad_entry<false>("sla_matvec_grad_values", hh, gy, x, grad, accumulate, stream);
}
