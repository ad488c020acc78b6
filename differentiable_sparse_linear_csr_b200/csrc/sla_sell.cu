// Sliced layout of a short-row CSR pattern for the solver's SpMV.
//
// Rows are grouped in slices of kSellRows (8) consecutive rows; a slice stores
// entry k of its 8 rows next to each other, padded to the slice's longest row.
// Eight consecutive threads (one row each) then read 8 consecutive values and
// column indices per step -- whole 32-byte sectors for both fp64 values and
// int32 columns -- with no row-pointer chain, so a thread can keep loads of
// several rows in flight.  Padding entries point at the row itself with value
// 0, which leaves the row sum unchanged: rows are still summed in stored order.
// The values are laid out per solve (one gather pass) into the workspace.
#include "sla_common.cuh"

namespace sla {

__global__ void sell_width_kernel(int n, const int32_t *__restrict__ rowptr, unsigned *__restrict__ cnt) {
    const int64_t sl = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t nsl = ((int64_t)n + kSellRows - 1) / kSellRows;
    if (sl > nsl) return;
    if (sl == nsl) { cnt[sl] = 0; return; }
    int w = 0;
    for (int l = 0; l < kSellRows; ++l) {
        const int64_t i = sl * kSellRows + l;
        if (i < n) w = max(w, rowptr[i + 1] - rowptr[i]);
    }
    cnt[sl] = (unsigned)(w * kSellRows);
}

__global__ void sell_fill_kernel(int n, const int32_t *__restrict__ rowptr,
                                 const int32_t *__restrict__ colind, const int32_t *__restrict__ sptr,
                                 int32_t *__restrict__ cols, int32_t *__restrict__ map) {
    const int64_t sl = blockIdx.x * (int64_t)(blockDim.x / kSellRows) + threadIdx.x / kSellRows;
    const int l = threadIdx.x % kSellRows;
    const int64_t nsl = ((int64_t)n + kSellRows - 1) / kSellRows;
    if (sl >= nsl) return;
    const int64_t i = sl * kSellRows + l;
    const int base = sptr[sl], w = (sptr[sl + 1] - base) / kSellRows;
    const int t0 = i < n ? rowptr[i] : 0, len = i < n ? rowptr[i + 1] - t0 : 0;
    const int own = i < n ? (int)i : 0;
    for (int k = 0; k < w; ++k) {
        const int slot = base + k * kSellRows + l;
        if (k < len) {
            cols[slot] = colind[t0 + k];
            map[slot] = t0 + k;
        } else {
            cols[slot] = own;
            map[slot] = -1;
        }
    }
}

template <typename T>
__global__ void sell_values_kernel(int64_t sell_nnz, int64_t nnz, int B, const int32_t *__restrict__ map,
                                   const T *__restrict__ vals, T *__restrict__ out) {
    const int64_t slot = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (slot >= sell_nnz) return;
    const int t = map[slot];
    for (int b = 0; b < B; ++b)
        out[(int64_t)b * sell_nnz + slot] = t >= 0 ? vals[(int64_t)b * nnz + t] : T(0);
}

sla_status build_sell(Csr *h, cudaStream_t s) {
    const int n = h->n_rows;
    const int64_t nsl = ((int64_t)n + kSellRows - 1) / kSellRows;
    unsigned *cnt = nullptr;
    void *ws = nullptr;
    SLA_CHECK_CUDA(cudaMalloc(&h->sell_ptr, (size_t)(nsl + 1) * sizeof(int32_t)));
    SLA_CHECK_CUDA(cudaMalloc(&cnt, (size_t)(nsl + 1) * sizeof(unsigned)));
    SLA_CHECK_CUDA(cudaMalloc(&ws, scan_ws_bytes(nsl + 1)));
    sell_width_kernel<<<(unsigned)((nsl + 1 + 255) / 256), 256, 0, s>>>(n, h->rowptr, cnt);
    SLA_CHECK_LAUNCH();
    sla_status st = exclusive_scan(cnt, reinterpret_cast<unsigned *>(h->sell_ptr), nsl + 1, ws, s);
    unsigned total = 0;
    if (st == SLA_OK &&
        (cudaMemcpyAsync(&total, h->sell_ptr + nsl, sizeof total, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
         cudaStreamSynchronize(s) != cudaSuccess))
        st = SLA_ERR_CUDA;
    cudaFree(cnt);
    cudaFree(ws);
    if (st != SLA_OK) {
        set_error("build_sell: %s", cudaGetErrorString(cudaGetLastError()));
        return st;
    }
    if (total > 0x7fffffffu) {   // padded layout would overflow int32 offsets: keep CSR only
        cudaFree(h->sell_ptr);
        h->sell_ptr = nullptr;
        return SLA_OK;
    }
    h->sell_nnz = total;
    const size_t z = (size_t)(total > 0 ? total : 1);
    SLA_CHECK_CUDA(cudaMalloc(&h->sell_cols, z * sizeof(int32_t)));
    SLA_CHECK_CUDA(cudaMalloc(&h->sell_map, z * sizeof(int32_t)));
    constexpr int kThreads = 256;
    const unsigned grid = (unsigned)((nsl + kThreads / kSellRows - 1) / (kThreads / kSellRows));
    sell_fill_kernel<<<grid, kThreads, 0, s>>>(n, h->rowptr, h->colind, h->sell_ptr, h->sell_cols,
                                               h->sell_map);
    SLA_CHECK_LAUNCH();
    h->has_sell = true;
    return SLA_OK;
}

sla_status sell_values(const Csr *h, const void *vals, void *vals_sell, cudaStream_t s) {
    if (h->sell_nnz == 0) return SLA_OK;
    const unsigned grid = (unsigned)((h->sell_nnz + 255) / 256);
    if (h->dtype == SLA_F64)
        sell_values_kernel<double><<<grid, 256, 0, s>>>(h->sell_nnz, h->nnz, h->batch, h->sell_map,
                                                        (const double *)vals, (double *)vals_sell);
    else
        sell_values_kernel<float><<<grid, 256, 0, s>>>(h->sell_nnz, h->nnz, h->batch, h->sell_map,
                                                       (const float *)vals, (float *)vals_sell);
    SLA_CHECK_LAUNCH();
    return SLA_OK;
}

}  // namespace sla
