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
//
// Two refinements, chosen at creation:
//  - uniform width: when padding every slice to the widest row costs at most
//    3 % of the entries (stencil and grid patterns), all slices get that width
//    and the kernels compute a slice's first slot instead of reading it;
//  - sorted windows (the SELL-C-sigma idea of Kreutzer, Hager, Wellein, Fehske
//    and Bishop, 2014, with sigma = 32): for irregular row lengths, the rows of
//    each aligned 32-row window are ordered by decreasing length (ties by row)
//    before they are cut into slices, so rows of similar length share a slice
//    and the padding shrinks (a 10-entry-mean kNN graph: 19 % -> 6 %).  A
//    window is one warp's rows in the solver, so each warp still handles the
//    same rows; sell_perm maps a position to its row.  Each row's entries keep
//    their stored order, so its sum is unchanged;
//  - compact columns: when every |column - row| < 2^15 (stencils, grids,
//    bandwidth-reduced orderings), the columns are also kept as 16-bit offsets
//    from their row (sell_d16), which the solver reads instead: 2 bytes an
//    entry instead of 4 in the matrix stream.
#include <climits>
#include <cstdlib>

#include "sla_common.cuh"

namespace sla {

// perm[pos] for the rows of each aligned 32-row window, longest first (ties by
// row): one warp per window, each lane ranks its row against the other 31.
__global__ void sell_sort_kernel(int n, const int32_t *__restrict__ rowptr, int32_t *__restrict__ perm) {
    const int64_t win = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) / kSellSortWindow;
    const int lane = threadIdx.x % kSellSortWindow;
    const int64_t i = win * kSellSortWindow + lane;
    const int len = i < n ? rowptr[i + 1] - rowptr[i] : -1;
    int rank = 0;
    for (int j = 0; j < kSellSortWindow; ++j) {
        const int lj = __shfl_sync(0xffffffffu, len, j);
        rank += (lj > len) || (lj == len && j < lane);
    }
    if (i < n) perm[win * kSellSortWindow + rank] = (int32_t)i;
}

// Slots of each slice: 8 times the longest of its rows (the rows at its
// positions when perm is given).
__global__ void sell_width_kernel(int n, const int32_t *__restrict__ rowptr, const int32_t *__restrict__ perm,
                                  unsigned *__restrict__ cnt) {
    const int64_t sl = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t nsl = ((int64_t)n + kSellRows - 1) / kSellRows;
    if (sl > nsl) return;
    if (sl == nsl) { cnt[sl] = 0; return; }
    int w = 0;
    for (int l = 0; l < kSellRows; ++l) {
        const int64_t i = sl * kSellRows + l;
        if (i < n) {
            const int r = perm ? perm[i] : (int)i;
            w = max(w, rowptr[r + 1] - rowptr[r]);
        }
    }
    cnt[sl] = (unsigned)(w * kSellRows);
}

// Columns, slot-to-entry map and 16-bit column offsets (clamped; *dmax
// receives the largest |column - row| so the caller can tell whether they hold).
__global__ void sell_fill_kernel(int n, const int32_t *__restrict__ rowptr,
                                 const int32_t *__restrict__ colind, const int32_t *__restrict__ sptr,
                                 const int32_t *__restrict__ perm, int32_t *__restrict__ cols,
                                 int32_t *__restrict__ map, int16_t *__restrict__ d16, int *__restrict__ dmax) {
    const int64_t sl = blockIdx.x * (int64_t)(blockDim.x / kSellRows) + threadIdx.x / kSellRows;
    const int l = threadIdx.x % kSellRows;
    const int64_t nsl = ((int64_t)n + kSellRows - 1) / kSellRows;
    int far = 0;
    if (sl < nsl) {
        const int64_t i = sl * kSellRows + l;
        const int base = sptr[sl], w = (sptr[sl + 1] - base) / kSellRows;
        const int row = i < n ? (perm ? perm[i] : (int)i) : 0;
        const int t0 = i < n ? rowptr[row] : 0, len = i < n ? rowptr[row + 1] - t0 : 0;
        for (int k = 0; k < w; ++k) {
            const int slot = base + k * kSellRows + l;
            const int c = k < len ? colind[t0 + k] : row;
            cols[slot] = c;
            map[slot] = k < len ? t0 + k : -1;
            const long long d = (long long)c - row;
            const long long ad = d < 0 ? -d : d;
            far = (int)max((long long)far, ad < INT_MAX ? ad : (long long)INT_MAX);
            d16[slot] = (int16_t)(d < -32768 ? -32768 : (d > 32767 ? 32767 : d));
        }
    }
    for (int o = 16; o > 0; o >>= 1) far = max(far, __shfl_xor_sync(0xffffffffu, far, o));
    if ((threadIdx.x & 31) == 0) atomicMax(dmax, far);
}

// Keeps the 16-bit column offsets when every |column - row| fits (stencils and
// bandwidth-reduced orderings): 2 bytes an entry instead of 4 in the matrix
// stream.  SLA_SELL_D16=0 turns them off.
static sla_status finish_d16(Csr *h, int *dmax_dev, cudaStream_t s) {
    int dmax = INT_MAX;
    SLA_CHECK_CUDA(cudaMemcpyAsync(&dmax, dmax_dev, sizeof dmax, cudaMemcpyDeviceToHost, s));
    SLA_CHECK_CUDA(cudaStreamSynchronize(s));
    cudaFree(dmax_dev);
    const char *e = getenv("SLA_SELL_D16");
    if (dmax > 32767 || (e && e[0] == '0')) {
        cudaFree(h->sell_d16);
        h->sell_d16 = nullptr;
    }
    return SLA_OK;
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

// Every slice padded to the widest row: slice s starts at slot s * 8 * w.
__global__ void sell_uniform_ptr_kernel(int64_t nsl, int w, int32_t *__restrict__ sptr) {
    const int64_t sl = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (sl <= nsl) sptr[sl] = (int32_t)(sl * kSellRows * w);
}

sla_status build_sell(Csr *h, bool sort_ok, cudaStream_t s) {
    const int n = h->n_rows;
    const int64_t nsl = ((int64_t)n + kSellRows - 1) / kSellRows;
    SLA_CHECK_CUDA(cudaMalloc(&h->sell_ptr, (size_t)(nsl + 1) * sizeof(int32_t)));
    // Uniform width when padding every slice to the widest row costs at most 3 %
    // of the entries (stencil and grid patterns): the kernels then compute a
    // slice's first slot instead of reading it.  SLA_SELL_UNIFORM=0 turns it off.
    const int64_t uslots = nsl * kSellRows * (int64_t)h->row_max;
    const char *ue = getenv("SLA_SELL_UNIFORM");
    if (h->row_max > 0 && uslots <= 0x7fffffffLL && (double)(uslots - h->nnz) <= 0.03 * (double)h->nnz &&
        !(ue && ue[0] == '0')) {
        sell_uniform_ptr_kernel<<<(unsigned)((nsl + 1 + 255) / 256), 256, 0, s>>>(nsl, h->row_max, h->sell_ptr);
        SLA_CHECK_LAUNCH();
        h->sell_w = h->row_max;
        h->sell_nnz = uslots;
        SLA_CHECK_CUDA(cudaMalloc(&h->sell_cols, (size_t)uslots * sizeof(int32_t)));
        SLA_CHECK_CUDA(cudaMalloc(&h->sell_map, (size_t)uslots * sizeof(int32_t)));
        SLA_CHECK_CUDA(cudaMalloc(&h->sell_d16, (size_t)uslots * sizeof(int16_t)));
        int *dmax = nullptr;
        SLA_CHECK_CUDA(cudaMalloc(&dmax, sizeof(int)));
        SLA_CHECK_CUDA(cudaMemsetAsync(dmax, 0, sizeof(int), s));
        constexpr int kThreads = 256;
        const unsigned grid = (unsigned)((nsl + kThreads / kSellRows - 1) / (kThreads / kSellRows));
        sell_fill_kernel<<<grid, kThreads, 0, s>>>(n, h->rowptr, h->colind, h->sell_ptr, nullptr,
                                                   h->sell_cols, h->sell_map, h->sell_d16, dmax);
        SLA_CHECK_LAUNCH();
        h->has_sell = true;
        return finish_d16(h, dmax, s);
    }
    // Irregular rows: sort each 32-row window by length when the solver keeps q
    // in HBM by row index (SLA_SELL_SORT=0 turns it off).
    const char *se = getenv("SLA_SELL_SORT");
    if (sort_ok && h->row_min != h->row_max && !(se && se[0] == '0')) {
        SLA_CHECK_CUDA(cudaMalloc(&h->sell_perm, (size_t)n * sizeof(int32_t)));
        const int64_t threads = ((int64_t)n + kSellSortWindow - 1) / kSellSortWindow * kSellSortWindow;
        sell_sort_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(n, h->rowptr, h->sell_perm);
        SLA_CHECK_LAUNCH();
    }
    unsigned *cnt = nullptr;
    void *ws = nullptr;
    SLA_CHECK_CUDA(cudaMalloc(&cnt, (size_t)(nsl + 1) * sizeof(unsigned)));
    SLA_CHECK_CUDA(cudaMalloc(&ws, scan_ws_bytes(nsl + 1)));
    sell_width_kernel<<<(unsigned)((nsl + 1 + 255) / 256), 256, 0, s>>>(n, h->rowptr, h->sell_perm, cnt);
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
        cudaFree(h->sell_perm);
        h->sell_ptr = h->sell_perm = nullptr;
        return SLA_OK;
    }
    h->sell_nnz = total;
    const size_t z = (size_t)(total > 0 ? total : 1);
    SLA_CHECK_CUDA(cudaMalloc(&h->sell_cols, z * sizeof(int32_t)));
    SLA_CHECK_CUDA(cudaMalloc(&h->sell_map, z * sizeof(int32_t)));
    SLA_CHECK_CUDA(cudaMalloc(&h->sell_d16, z * sizeof(int16_t)));
    int *dmax = nullptr;
    SLA_CHECK_CUDA(cudaMalloc(&dmax, sizeof(int)));
    SLA_CHECK_CUDA(cudaMemsetAsync(dmax, 0, sizeof(int), s));
    constexpr int kThreads = 256;
    const unsigned grid = (unsigned)((nsl + kThreads / kSellRows - 1) / (kThreads / kSellRows));
    sell_fill_kernel<<<grid, kThreads, 0, s>>>(n, h->rowptr, h->colind, h->sell_ptr, h->sell_perm,
                                               h->sell_cols, h->sell_map, h->sell_d16, dmax);
    SLA_CHECK_LAUNCH();
    h->has_sell = true;
    return finish_d16(h, dmax, s);
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
