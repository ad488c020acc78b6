// Integer pattern work, bit-exact by construction: a device exclusive scan, a
// stable least-significant-digit radix sort (8-bit digits), and on top of them
// the CSR transpose (stable by column, values moved never combined) and the
// COO -> CSR build (stable by (row, col), duplicates summed in input order).
// The transposed pattern serves the adjoint solve A^T lambda = dL/dx of the
// torch-sla summary page (technical summary, "Methodology" 2) on handles whose
// storage is not symmetric.
#include "sla_common.cuh"

namespace sla {

// ----------------------------------------------------------------- scan ----
constexpr int kScanThreads = 1024, kScanItems = 4;
constexpr int64_t kScanTile = (int64_t)kScanThreads * kScanItems;

// Exclusive scan of one tile per block; the tile total goes to sums[block].
// Each thread reads its own items before writing them, so in == out is allowed.
__global__ void __launch_bounds__(kScanThreads)
scan_tile_kernel(const unsigned *in, unsigned *out, unsigned *sums, int64_t n) {
    __shared__ unsigned wtot[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t base = blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanItems;
    unsigned v[kScanItems];
    unsigned tsum = 0;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        v[k] = (base + k < n) ? in[base + k] : 0u;
        tsum += v[k];
    }
    unsigned incl = tsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        unsigned w = wtot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned t = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += t;
        }
        wtot[lane] = w;
    }
    __syncthreads();
    unsigned run = incl - tsum + (warp > 0 ? wtot[warp - 1] : 0u);
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        if (base + k < n) out[base + k] = run;
        run += v[k];
    }
    if (threadIdx.x == kScanThreads - 1) sums[blockIdx.x] = wtot[31];
}

__global__ void scan_add_kernel(unsigned *out, const unsigned *offs, int64_t n) {
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i < n) out[i] += offs[i / kScanTile];
}

size_t scan_ws_bytes(int64_t n) {
    size_t b = 256;
    while (n > kScanTile) {
        n = (n + kScanTile - 1) / kScanTile;
        b += 2 * align_up((size_t)n * sizeof(unsigned));
    }
    return b + 2 * 256;
}

sla_status exclusive_scan(const unsigned *in, unsigned *out, int64_t n, void *ws,
                                 cudaStream_t s) {
    if (n <= 0) return SLA_OK;
    const int64_t nb = (n + kScanTile - 1) / kScanTile;
    Carver c(ws);
    unsigned *sums = c.take<unsigned>(nb);
    unsigned *sums_x = c.take<unsigned>(nb);
    scan_tile_kernel<<<(unsigned)nb, kScanThreads, 0, s>>>(in, out, sums, n);
    SLA_CHECK_LAUNCH();
    if (nb > 1) {
        sla_status st = exclusive_scan(sums, sums_x, nb, static_cast<char *>(ws) + c.off, s);
        if (st != SLA_OK) return st;
        scan_add_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(out, sums_x, n);
        SLA_CHECK_LAUNCH();
    }
    return SLA_OK;
}

// ------------------------------------------------------------ radix sort ----
constexpr int kSortThreads = 256, kSortRounds = 16, kSortWarps = kSortThreads / 32;
constexpr int64_t kSortTile = (int64_t)kSortThreads * kSortRounds;

__global__ void __launch_bounds__(kSortThreads)
radix_hist_kernel(const unsigned *__restrict__ keys, int64_t n, int shift,
                  unsigned *__restrict__ hist, int ntiles) {
    __shared__ unsigned cnt[256];
    cnt[threadIdx.x] = 0;
    __syncthreads();
    const int64_t base = blockIdx.x * kSortTile;
    for (int r = 0; r < kSortRounds; ++r) {
        const int64_t idx = base + (int64_t)r * kSortThreads + threadIdx.x;
        if (idx < n) atomicAdd(&cnt[(keys[idx] >> shift) & 255u], 1u);
    }
    __syncthreads();
    hist[(int64_t)threadIdx.x * ntiles + blockIdx.x] = cnt[threadIdx.x];
}

// Stable scatter of one tile: items are taken in index order (round, warp,
// lane), and an item's slot is its digit's running offset plus the number of
// equal digits before it in that order.
__global__ void __launch_bounds__(kSortThreads)
radix_scatter_kernel(const unsigned *__restrict__ kin, const int32_t *__restrict__ vin,
                     unsigned *__restrict__ kout, int32_t *__restrict__ vout, int64_t n,
                     int shift, const unsigned *__restrict__ offs, int ntiles) {
    __shared__ unsigned running[256];
    __shared__ unsigned wcnt[kSortWarps][256];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    unsigned lt;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt));
    running[tid] = offs[(int64_t)tid * ntiles + blockIdx.x];
    const int64_t base = blockIdx.x * kSortTile;
    for (int r = 0; r < kSortRounds; ++r) {
#pragma unroll
        for (int w = 0; w < kSortWarps; ++w) wcnt[w][tid] = 0;
        __syncthreads();
        const int64_t idx = base + (int64_t)r * kSortThreads + tid;
        const bool valid = idx < n;
        const unsigned k = valid ? kin[idx] : 0u;
        const int32_t v = valid ? vin[idx] : 0;
        const unsigned d = valid ? ((k >> shift) & 255u) : 256u;
        const unsigned peers = __match_any_sync(0xffffffffu, d);
        const unsigned rank = __popc(peers & lt);
        if (valid && lane == __ffs(peers) - 1) wcnt[warp][d] = __popc(peers);
        __syncthreads();
        unsigned run = running[tid];
#pragma unroll
        for (int w = 0; w < kSortWarps; ++w) {
            const unsigned cc = wcnt[w][tid];
            wcnt[w][tid] = run;
            run += cc;
        }
        running[tid] = run;
        __syncthreads();
        if (valid) {
            const unsigned pos = wcnt[warp][d] + rank;
            kout[pos] = k;
            vout[pos] = v;
        }
        __syncthreads();
    }
}

static int key_bits(int64_t max_key) {
    int b = 0;
    while (max_key > 0) { ++b; max_key >>= 1; }
    return b;
}

static size_t radix_ws_bytes(int64_t n) {
    const int64_t ntiles = (n + kSortTile - 1) / kSortTile;
    return 2 * align_up((size_t)(256 * ntiles) * sizeof(unsigned)) + scan_ws_bytes(256 * ntiles);
}

// Sorts (k[0], v[0]) by key bits [0, bits) using (k[1], v[1]) as the other
// buffer; returns in *which the index of the buffer that holds the result.
static sla_status radix_sort(unsigned *k[2], int32_t *v[2], int64_t n, int bits, void *ws,
                             cudaStream_t s, int *which) {
    *which = 0;
    if (n <= 1 || bits <= 0) return SLA_OK;
    const int64_t ntiles = (n + kSortTile - 1) / kSortTile;
    Carver c(ws);
    unsigned *hist = c.take<unsigned>(256 * ntiles);
    unsigned *offs = c.take<unsigned>(256 * ntiles);
    void *scan_ws = static_cast<char *>(ws) + c.off;
    int cur = 0;
    for (int shift = 0; shift < bits; shift += 8) {
        radix_hist_kernel<<<(unsigned)ntiles, kSortThreads, 0, s>>>(k[cur], n, shift, hist,
                                                                  (int)ntiles);
        SLA_CHECK_LAUNCH();
        sla_status st = exclusive_scan(hist, offs, 256 * ntiles, scan_ws, s);
        if (st != SLA_OK) return st;
        radix_scatter_kernel<<<(unsigned)ntiles, kSortThreads, 0, s>>>(
            k[cur], v[cur], k[1 - cur], v[1 - cur], n, shift, offs, (int)ntiles);
        SLA_CHECK_LAUNCH();
        cur = 1 - cur;
    }
    *which = cur;
    return SLA_OK;
}

// ------------------------------------------------------------ transpose ----
__global__ void expand_rows_kernel(int n_rows, int64_t nnz, const int32_t *__restrict__ rowptr,
                                   int32_t *__restrict__ rowidx) {
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= n_rows) return;
    const int t0 = max(rowptr[i], 0), t1 = min((int64_t)rowptr[i + 1], nnz);
    for (int t = t0; t < t1; ++t) rowidx[t] = (int32_t)i;
}

__global__ void keys_iota_kernel(int64_t n, const int32_t *__restrict__ key, unsigned *kout,
                                 int32_t *vout) {
    const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (t >= n) return;
    kout[t] = (unsigned)key[t];
    vout[t] = (int32_t)t;
}

__global__ void count_kernel(int64_t n, int nkeys, const int32_t *__restrict__ key, unsigned *cnt) {
    const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (t < n && key[t] >= 0 && key[t] < nkeys) atomicAdd(cnt + key[t], 1u);
}

__global__ void transpose_finish_kernel(int64_t n, const int32_t *__restrict__ order,
                                        const int32_t *__restrict__ rowidx,
                                        int32_t *__restrict__ colindT, int32_t *__restrict__ perm) {
    const int64_t s = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (s >= n) return;
    const int32_t t = order[s];
    colindT[s] = rowidx[t];
    if (perm) perm[s] = t;
}

template <typename T>
__global__ void gather_values_kernel(int64_t nnz, int B, const int32_t *__restrict__ perm,
                                     const T *__restrict__ vals, T *__restrict__ out) {
    const int64_t s = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (s >= nnz) return;
    const int32_t t = perm[s];
    for (int b = 0; b < B; ++b) out[(int64_t)b * nnz + s] = vals[(int64_t)b * nnz + t];
}

static inline unsigned nblk(int64_t n, int t = 256) { return (unsigned)((n + t - 1) / t); }

size_t transpose_ws_bytes(int32_t n_rows, int32_t n_cols, int64_t nnz) {
    (void)n_rows;
    const size_t z = (size_t)(nnz > 0 ? nnz : 1);
    return 5 * align_up(z * 4) + 2 * align_up(((size_t)n_cols + 1) * 4) +
           radix_ws_bytes(nnz) + scan_ws_bytes((int64_t)n_cols + 1) + 4 * 256;
}

sla_status transpose_pattern(int32_t n_rows, int32_t n_cols, int64_t nnz,
                             const int32_t *rowptr, const int32_t *colind, int32_t *rowptrT,
                             int32_t *colindT, int32_t *perm, void *ws, cudaStream_t s) {
    Carver c(ws);
    const size_t z = (size_t)(nnz > 0 ? nnz : 1);
    unsigned *k[2] = {c.take<unsigned>(z), c.take<unsigned>(z)};
    int32_t *v[2] = {c.take<int32_t>(z), c.take<int32_t>(z)};
    int32_t *rowidx = c.take<int32_t>(z);
    unsigned *cnt = c.take<unsigned>((size_t)n_cols + 1);
    void *rest = static_cast<char *>(ws) + c.off;
    SLA_CHECK_CUDA(cudaMemsetAsync(cnt, 0, ((size_t)n_cols + 1) * sizeof(unsigned), s));
    if (nnz > 0) {
        expand_rows_kernel<<<nblk(n_rows), 256, 0, s>>>(n_rows, nnz, rowptr, rowidx);
        keys_iota_kernel<<<nblk(nnz), 256, 0, s>>>(nnz, colind, k[0], v[0]);
        count_kernel<<<nblk(nnz), 256, 0, s>>>(nnz, n_cols, colind, cnt);
        SLA_CHECK_LAUNCH();
        int which = 0;
        sla_status st = radix_sort(k, v, nnz, key_bits((int64_t)n_cols - 1), rest, s, &which);
        if (st != SLA_OK) return st;
        transpose_finish_kernel<<<nblk(nnz), 256, 0, s>>>(nnz, v[which], rowidx, colindT, perm);
        SLA_CHECK_LAUNCH();
    }
    return exclusive_scan(cnt, reinterpret_cast<unsigned *>(rowptrT), (int64_t)n_cols + 1, rest, s);
}

// ------------------------------------------------------------ COO -> CSR ----
__global__ void coo_range_kernel(int64_t n, int n_rows, int n_cols, const int32_t *__restrict__ row,
                                 const int32_t *__restrict__ col, unsigned *bad) {
    const int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (e >= n) return;
    if (row[e] < 0 || row[e] >= n_rows || col[e] < 0 || col[e] >= n_cols) atomicExch(bad, 1u);
}

__global__ void gather_keys_kernel(int64_t n, const int32_t *__restrict__ src,
                                   const int32_t *__restrict__ idx, unsigned *__restrict__ kout) {
    const int64_t s = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (s < n) kout[s] = (unsigned)src[idx[s]];
}

__global__ void coo_heads_kernel(int64_t n, const unsigned *__restrict__ rows_sorted,
                                 const int32_t *__restrict__ order, const int32_t *__restrict__ col,
                                 unsigned *__restrict__ head) {
    const int64_t s = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (s > n) return;
    if (s == n) { head[s] = 0; return; }
    head[s] = (s == 0 || rows_sorted[s] != rows_sorted[s - 1] ||
               col[order[s]] != col[order[s - 1]]) ? 1u : 0u;
}

__global__ void coo_place_kernel(int64_t n, int n_rows, const unsigned *__restrict__ bad,
                                 const unsigned *__restrict__ rows_sorted,
                                 const int32_t *__restrict__ order, const int32_t *__restrict__ col,
                                 const unsigned *__restrict__ head, const unsigned *__restrict__ pos,
                                 int32_t *__restrict__ colind, int32_t *__restrict__ slot,
                                 unsigned *__restrict__ rowcnt) {
    const int64_t s = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (s >= n || *bad) return;
    const unsigned out = pos[s] + head[s] - 1u;
    if (head[s]) {
        colind[out] = col[order[s]];
        atomicAdd(rowcnt + rows_sorted[s], 1u);
    }
    if (slot) slot[order[s]] = (int32_t)out;
}

// One thread per output entry: the run of equal (row, col) is summed left to
// right in sorted order, which the stable sort made the input order.
template <typename T>
__global__ void coo_values_kernel(int64_t n, int B, const unsigned *__restrict__ bad,
                                  const int32_t *__restrict__ order, const unsigned *__restrict__ head,
                                  const unsigned *__restrict__ pos, const T *__restrict__ val,
                                  T *__restrict__ val_out) {
    const int64_t s = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (s >= n || *bad || !head[s]) return;
    const unsigned out = pos[s];
    for (int b = 0; b < B; ++b) {
        const T *vb = val + (int64_t)b * n;
        T sum = vb[order[s]];
        for (int64_t u = s + 1; u < n && !head[u]; ++u) sum = sum + vb[order[u]];
        val_out[(int64_t)b * n + out] = sum;
    }
}

__global__ void coo_finish_kernel(int64_t n, const unsigned *bad, const unsigned *pos,
                                  int64_t *nnz_out) {
    *nnz_out = *bad ? -1 : (int64_t)pos[n];
}

sla_status transpose_values(const Csr *h, const void *vals, void *valsT, cudaStream_t s) {
    if (h->nnz == 0) return SLA_OK;
    if (h->dtype == SLA_F64)
        gather_values_kernel<double><<<nblk(h->nnz), 256, 0, s>>>(
            h->nnz, h->batch, h->permT, (const double *)vals, (double *)valsT);
    else
        gather_values_kernel<float><<<nblk(h->nnz), 256, 0, s>>>(
            h->nnz, h->batch, h->permT, (const float *)vals, (float *)valsT);
    SLA_CHECK_LAUNCH();
    return SLA_OK;
}

static size_t coo_ws(int32_t n_rows, int32_t n_cols, int64_t nnz_in) {
    (void)n_cols;
    const size_t z = (size_t)(nnz_in > 0 ? nnz_in : 1);
    return 4 * align_up(z * 4) + 2 * align_up((z + 1) * 4) + align_up(((size_t)n_rows + 1) * 4) +
           256 + radix_ws_bytes(nnz_in) + scan_ws_bytes((int64_t)nnz_in + 1) +
           scan_ws_bytes((int64_t)n_rows + 1) + 4 * 256;
}

}  // namespace sla

using namespace sla;

extern "C" size_t sla_transpose_workspace_bytes(int32_t n_rows, int32_t n_cols, int64_t nnz) {
    if (n_rows < 0 || n_cols < 0 || nnz < 0) return 0;
    return transpose_ws_bytes(n_rows, n_cols, nnz);
}

extern "C" sla_status sla_csr_transpose(int32_t n_rows, int32_t n_cols, int64_t nnz,
                                        const int32_t *rowptr, const int32_t *colind,
                                        int32_t batch, sla_dtype dtype, const void *vals,
                                        int32_t *rowptrT, int32_t *colindT, void *valsT,
                                        int32_t *perm, void *ws, size_t ws_bytes, void *stream) {
    SLA_RANGE("sla_csr_transpose");
    clear_error();
    SLA_REQUIRE(n_rows >= 0 && n_cols >= 0 && nnz >= 0 && nnz <= 0x7fffffff,
                "sla_csr_transpose: bad sizes");
    SLA_REQUIRE(batch >= 1 && (dtype == SLA_F64 || dtype == SLA_F32), "sla_csr_transpose: bad batch/dtype");
    SLA_REQUIRE(rowptr && rowptrT && (nnz == 0 || (colind && colindT)), "sla_csr_transpose: NULL pointer");
    SLA_REQUIRE(ws && ws_bytes >= transpose_ws_bytes(n_rows, n_cols, nnz),
                "sla_csr_transpose: workspace too small (%zu < %zu)", ws_bytes,
                transpose_ws_bytes(n_rows, n_cols, nnz));
    SLA_REQUIRE(!vals || (valsT && perm), "sla_csr_transpose: vals need valsT and perm");
    cudaStream_t s = as_stream(stream);
    sla_status st = transpose_pattern(n_rows, n_cols, nnz, rowptr, colind, rowptrT, colindT,
                                      perm, ws, s);
    if (st != SLA_OK || !vals || nnz == 0) return st;
    const int32_t *p = perm;
    if (dtype == SLA_F64)
        gather_values_kernel<double><<<nblk(nnz), 256, 0, s>>>(nnz, batch, p, (const double *)vals,
                                                              (double *)valsT);
    else
        gather_values_kernel<float><<<nblk(nnz), 256, 0, s>>>(nnz, batch, p, (const float *)vals,
                                                             (float *)valsT);
    SLA_CHECK_LAUNCH();
    return SLA_OK;
}

extern "C" size_t sla_coo_workspace_bytes(int32_t n_rows, int32_t n_cols, int64_t nnz_in) {
    if (n_rows < 0 || n_cols < 0 || nnz_in < 0) return 0;
    return coo_ws(n_rows, n_cols, nnz_in);
}

extern "C" sla_status sla_csr_from_coo(int32_t n_rows, int32_t n_cols, int64_t nnz_in,
                                       const int32_t *row, const int32_t *col, int32_t batch,
                                       sla_dtype dtype, const void *val, int32_t *rowptr,
                                       int32_t *colind, void *val_out, int32_t *slot,
                                       int64_t *nnz_out, void *ws, size_t ws_bytes, void *stream) {
    SLA_RANGE("sla_csr_from_coo");
    clear_error();
    SLA_REQUIRE(n_rows >= 0 && n_cols >= 0 && nnz_in >= 0 && nnz_in < 0x7fffffff,
                "sla_csr_from_coo: bad sizes");
    SLA_REQUIRE(batch >= 1 && (dtype == SLA_F64 || dtype == SLA_F32), "sla_csr_from_coo: bad batch/dtype");
    SLA_REQUIRE(rowptr && nnz_out && (nnz_in == 0 || (row && col && colind)),
                "sla_csr_from_coo: NULL pointer");
    SLA_REQUIRE(!val || val_out, "sla_csr_from_coo: val given without val_out");
    SLA_REQUIRE(ws && ws_bytes >= coo_ws(n_rows, n_cols, nnz_in),
                "sla_csr_from_coo: workspace too small (%zu < %zu)", ws_bytes,
                coo_ws(n_rows, n_cols, nnz_in));
    cudaStream_t s = as_stream(stream);
    const int64_t n = nnz_in;
    const size_t z = (size_t)(n > 0 ? n : 1);
    Carver c(ws);
    unsigned *k[2] = {c.take<unsigned>(z), c.take<unsigned>(z)};
    int32_t *v[2] = {c.take<int32_t>(z), c.take<int32_t>(z)};
    unsigned *head = c.take<unsigned>(z + 1);
    unsigned *pos = c.take<unsigned>(z + 1);
    unsigned *rowcnt = c.take<unsigned>((size_t)n_rows + 1);
    unsigned *bad = c.take<unsigned>(4);
    void *rest = static_cast<char *>(ws) + c.off;
    SLA_CHECK_CUDA(cudaMemsetAsync(bad, 0, sizeof(unsigned), s));
    SLA_CHECK_CUDA(cudaMemsetAsync(rowcnt, 0, ((size_t)n_rows + 1) * sizeof(unsigned), s));
    if (n > 0) {
        coo_range_kernel<<<nblk(n), 256, 0, s>>>(n, n_rows, n_cols, row, col, bad);
        keys_iota_kernel<<<nblk(n), 256, 0, s>>>(n, col, k[0], v[0]);
        SLA_CHECK_LAUNCH();
        int which = 0;
        sla_status st = radix_sort(k, v, n, key_bits((int64_t)n_cols - 1), rest, s, &which);
        if (st != SLA_OK) return st;
        // second key: the row of each entry in column order, sorted stably
        unsigned *k2[2] = {k[1 - which], k[which]};
        int32_t *v2[2] = {v[which], v[1 - which]};
        gather_keys_kernel<<<nblk(n), 256, 0, s>>>(n, row, v2[0], k2[0]);
        SLA_CHECK_LAUNCH();
        int which2 = 0;
        st = radix_sort(k2, v2, n, key_bits((int64_t)n_rows - 1), rest, s, &which2);
        if (st != SLA_OK) return st;
        const unsigned *rows_sorted = k2[which2];
        const int32_t *order = v2[which2];
        coo_heads_kernel<<<nblk(n + 1), 256, 0, s>>>(n, rows_sorted, order, col, head);
        SLA_CHECK_LAUNCH();
        st = exclusive_scan(head, pos, n + 1, rest, s);
        if (st != SLA_OK) return st;
        coo_place_kernel<<<nblk(n), 256, 0, s>>>(n, n_rows, bad, rows_sorted, order, col, head,
                                                 pos, colind, slot, rowcnt);
        SLA_CHECK_LAUNCH();
        if (val) {
            if (dtype == SLA_F64)
                coo_values_kernel<double><<<nblk(n), 256, 0, s>>>(n, batch, bad, order, head, pos,
                                                                 (const double *)val, (double *)val_out);
            else
                coo_values_kernel<float><<<nblk(n), 256, 0, s>>>(n, batch, bad, order, head, pos,
                                                                (const float *)val, (float *)val_out);
            SLA_CHECK_LAUNCH();
        }
    } else {
        SLA_CHECK_CUDA(cudaMemsetAsync(pos, 0, sizeof(unsigned), s));
    }
    sla_status st = exclusive_scan(rowcnt, reinterpret_cast<unsigned *>(rowptr), (int64_t)n_rows + 1,
                                   rest, s);
    if (st != SLA_OK) return st;
    coo_finish_kernel<<<1, 1, 0, s>>>(n, bad, pos, nnz_out);
    SLA_CHECK_LAUNCH();
    return SLA_OK;
}
