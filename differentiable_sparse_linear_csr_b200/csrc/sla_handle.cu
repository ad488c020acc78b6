// CSR handle: pattern validation, pattern statistics, diagonal positions and
// (on request) A^T's pattern.  A handle is the shared-pattern `SparseTensor`
// of the torch-sla summary page (technical summary, "Methodology" 1: one
// matrix, or a batch of value sets sharing one pattern); a list handle holds
// items with their own patterns, stored block-diagonally (`SparseTensorList`).
#include <climits>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <vector>

#include "sla_common.cuh"

namespace sla {

static thread_local std::string g_error;

void set_error(const char *fmt, ...) {
    char buf[1024];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_error = buf;
}

void clear_error() { g_error.clear(); }

int lanes_for_mean(double m) {
    if (m < 12.0) return 1;
    if (m < 24.0) return 2;
    if (m < 48.0) return 4;
    if (m < 96.0) return 8;
    if (m < 192.0) return 16;
    return 32;
}

// --------------------------------------------------------------- checks ----
// Findings are packed as (code << 40) | where and combined with atomicMin, so
// the lowest code wins and, within a code, the lowest index.
__device__ __forceinline__ void report(unsigned long long *best, int code, long long where) {
    atomicMin(best, ((unsigned long long)code << 40) | (unsigned long long)where);
}

__global__ void check_init_kernel(unsigned long long *best) { *best = ~0ull; }

__global__ void check_rows_kernel(int n_rows, int64_t nnz, const int32_t *__restrict__ rowptr,
                                  unsigned long long *best) {
    const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (i == 0 && rowptr[0] != 0) report(best, 1, 0);
    if (i < n_rows && rowptr[i + 1] < rowptr[i]) report(best, 2, i);
    if (i == 0 && (int64_t)rowptr[n_rows] != nnz) report(best, 3, n_rows);
}

// Entry checks run only when the row pointers are sound (codes 1-3 absent),
// so every entry range read below lies inside [0, nnz).
__global__ void check_entries_kernel(int n_rows, int n_cols, int64_t nnz,
                                     const int32_t *__restrict__ rowptr,
                                     const int32_t *__restrict__ colind, int need_diag,
                                     unsigned long long *best) {
    if ((*(volatile unsigned long long *)best >> 40) <= 3) return;
    const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (i >= n_rows) return;
    const int t0 = rowptr[i], t1 = rowptr[i + 1];
    bool diag = false;
    for (int t = t0; t < t1; ++t) {
        const int c = colind[t];
        if (c < 0 || c >= n_cols) report(best, 4, t);
        else if (t > t0 && c <= colind[t - 1]) report(best, 5, t);
        if (c == i) diag = true;
    }
    if (need_diag && !diag) report(best, 6, i);
}

__global__ void check_finish_kernel(const unsigned long long *best, int64_t *result) {
    const unsigned long long b = *best;
    if (b == ~0ull) {
        result[0] = 0;
        result[1] = -1;
    } else {
        result[0] = (int64_t)(b >> 40);
        result[1] = (int64_t)(b & ((1ull << 40) - 1));
    }
}

static sla_status enqueue_check(int32_t n_rows, int32_t n_cols, int64_t nnz,
                                const int32_t *rowptr, const int32_t *colind, int need_diag,
                                unsigned long long *best, int64_t *result, cudaStream_t s) {
    check_init_kernel<<<1, 1, 0, s>>>(best);
    const int nb = (n_rows + 1 + 255) / 256;
    check_rows_kernel<<<nb, 256, 0, s>>>(n_rows, nnz, rowptr, best);
    if (n_rows > 0)
        check_entries_kernel<<<(n_rows + 255) / 256, 256, 0, s>>>(n_rows, n_cols, nnz, rowptr,
                                                                  colind, need_diag, best);
    check_finish_kernel<<<1, 1, 0, s>>>(best, result);
    SLA_CHECK_LAUNCH();
    return SLA_OK;
}

// ----------------------------------------------------------- statistics ----
__global__ void diagpos_kernel(int n, const int32_t *__restrict__ rowptr,
                               const int32_t *__restrict__ colind, int32_t *__restrict__ diagpos) {
    const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (i >= n) return;
    int d = -1;
    for (int t = rowptr[i]; t < rowptr[i + 1]; ++t)
        if (colind[t] == i) d = t;
    diagpos[i] = d;
}

__global__ void row_stats_kernel(int n, const int32_t *__restrict__ rowptr, int *minmax) {
    const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    int len_min = INT_MAX, len_max = 0;
    if (i < n) len_min = len_max = rowptr[i + 1] - rowptr[i];
    for (int o = 16; o > 0; o >>= 1) {
        len_min = min(len_min, __shfl_xor_sync(0xffffffffu, len_min, o));
        len_max = max(len_max, __shfl_xor_sync(0xffffffffu, len_max, o));
    }
    if ((threadIdx.x & 31) == 0) {
        atomicMin(minmax, len_min);
        atomicMax(minmax + 1, len_max);
    }
}

__global__ void row_stats_init_kernel(int *minmax) {
    minmax[0] = INT_MAX;
    minmax[1] = 0;
}

sla_status diag_positions(int32_t n, const int32_t *rowptr, const int32_t *colind,
                          int32_t *diagpos, cudaStream_t s) {
    if (n == 0) return SLA_OK;
    diagpos_kernel<<<(n + 255) / 256, 256, 0, s>>>(n, rowptr, colind, diagpos);
    SLA_CHECK_LAUNCH();
    return SLA_OK;
}

sla_status ensure_transpose(Csr *h, cudaStream_t s) {
    if (h->has_transpose) return SLA_OK;
    const size_t n1 = (size_t)h->n_cols + 1, z = (size_t)(h->nnz > 0 ? h->nnz : 1);
    SLA_CHECK_CUDA(cudaMalloc(&h->rowptrT, n1 * sizeof(int32_t)));
    SLA_CHECK_CUDA(cudaMalloc(&h->colindT, z * sizeof(int32_t)));
    SLA_CHECK_CUDA(cudaMalloc(&h->permT, z * sizeof(int32_t)));
    if (h->n_rows == h->n_cols)
        SLA_CHECK_CUDA(cudaMalloc(&h->diagposT, (size_t)(h->n_cols > 0 ? h->n_cols : 1) * sizeof(int32_t)));
    const size_t wsb = transpose_ws_bytes(h->n_rows, h->n_cols, h->nnz);
    void *ws = nullptr;
    SLA_CHECK_CUDA(cudaMalloc(&ws, wsb > 0 ? wsb : 1));
    sla_status st = transpose_pattern(h->n_rows, h->n_cols, h->nnz, h->rowptr, h->colind,
                                      h->rowptrT, h->colindT, h->permT, ws, s);
    if (st == SLA_OK && h->diagposT)
        st = diag_positions(h->n_cols, h->rowptrT, h->colindT, h->diagposT, s);
    // the temporary must outlive the queued kernels
    cudaStreamSynchronize(s);
    cudaFree(ws);
    if (st != SLA_OK) return st;
    h->has_transpose = true;
    return SLA_OK;
}

// Persistent-grid and block-solver layout for the handle (in sla_cg.cu).
sla_status cg_configure(Csr *h);
// Segment-solver layout of a list handle (in sla_cg.cu).
sla_status cg_configure_list(Csr *h);

// Every entry of a list handle's row lies in its item's diagonal block:
// row i of item s (seg[s] <= i < seg[s+1]) may only hold columns in the same
// range.  The first offending entry is reported as code 7.
__global__ void list_check_kernel(int n_rows, const int32_t *rowptr, const int32_t *colind,
                                  int n_items, const int32_t *seg, unsigned long long *best) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_rows) return;
    int lo = 0, hi = n_items - 1;           // the item s with seg[s] <= i < seg[s+1]
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (seg[mid] <= i) lo = mid;
        else hi = mid - 1;
    }
    const int c0 = seg[lo], c1 = seg[lo + 1];
    for (int t = rowptr[i]; t < rowptr[i + 1]; ++t) {
        const int c = colind[t];
        if (c < c0 || c >= c1) {
            atomicMin(best, (7ull << 40) | (unsigned long long)t);
            return;
        }
    }
}

}  // namespace sla

using namespace sla;

extern "C" const char *sla_last_error_string(void) { return g_error.c_str(); }

extern "C" const char *sla_version(void) {
    return SLA_DEBUG_BOUNDS ? "sla 0.2.0 (sm_100a, bounds-checking build)" : "sla 0.2.0 (sm_100a)";
}

#if SLA_DEBUG_BOUNDS
namespace sla {
// Readers of every translation unit's bounds record, registered at load time.
static std::vector<DbgReader> &dbg_readers() {
    static std::vector<DbgReader> r;
    return r;
}
int dbg_register(DbgReader f) {
    dbg_readers().push_back(f);
    return (int)dbg_readers().size();
}
}  // namespace sla
#endif

extern "C" sla_status sla_debug_bounds_report(uint64_t *violations, int32_t *first_code,
                                              int64_t *first_index, int32_t reset) {
    clear_error();
#if SLA_DEBUG_BOUNDS
    unsigned long long count = 0, first = ~0ull;
    for (DbgReader f : dbg_readers()) {
        unsigned long long c = 0, fi = ~0ull;
        SLA_CHECK_CUDA(f(&c, &fi, reset != 0));
        count += c;
        if (fi < first) first = fi;
    }
    if (violations) *violations = count;
    if (first_code) *first_code = count ? (int32_t)(first >> 56) : 0;
    if (first_index) *first_index = count ? (int64_t)(first & ((1ull << 56) - 1)) : -1;
    return SLA_OK;
#else
    (void)reset;
    if (violations) *violations = 0;
    if (first_code) *first_code = 0;
    if (first_index) *first_index = -1;
    set_error("sla_debug_bounds_report: this library was built without SLA_DEBUG_BOUNDS "
              "(load libsla_debug_bounds.so)");
    return SLA_ERR_UNSUPPORTED;
#endif
}

extern "C" sla_status sla_csr_check(int32_t n_rows, int32_t n_cols, int64_t nnz,
                                    const int32_t *rowptr, const int32_t *colind,
                                    int32_t need_diag, int64_t *result, void *stream) {
    SLA_RANGE("sla_csr_check");
    clear_error();
    SLA_REQUIRE(n_rows >= 0 && n_cols >= 0 && nnz >= 0 && nnz <= INT_MAX,
                "sla_csr_check: bad sizes n_rows=%d n_cols=%d nnz=%lld", n_rows, n_cols,
                (long long)nnz);
    SLA_REQUIRE(rowptr && result && (nnz == 0 || colind), "sla_csr_check: NULL pointer");
    unsigned long long *best = reinterpret_cast<unsigned long long *>(result);
    // result[0..1] doubles as the scratch word: the finish kernel rewrites it.
    return enqueue_check(n_rows, n_cols, nnz, rowptr, colind, need_diag, best, result,
                         as_stream(stream));
}

namespace {
sla_status create_handle(int32_t n_rows, int32_t n_cols, int64_t nnz, const int32_t *rowptr,
                         const int32_t *colind, int32_t batch, sla_dtype dtype, uint32_t flags,
                         void *stream, sla_csr_t *out, bool list);
}

extern "C" sla_status sla_csr_create(int32_t n_rows, int32_t n_cols, int64_t nnz,
                                     const int32_t *rowptr, const int32_t *colind,
                                     int32_t batch, sla_dtype dtype, uint32_t flags,
                                     void *stream, sla_csr_t *out) {
    SLA_RANGE("sla_csr_create");
    clear_error();
    return create_handle(n_rows, n_cols, nnz, rowptr, colind, batch, dtype, flags, stream, out, false);
}

extern "C" sla_status sla_csr_list_create(int32_t n_items, const int32_t *item_rows, int32_t n_rows,
                                          int64_t nnz, const int32_t *rowptr, const int32_t *colind,
                                          sla_dtype dtype, uint32_t flags, void *stream,
                                          sla_csr_t *out) {
    SLA_RANGE("sla_csr_list_create");
    clear_error();
    SLA_REQUIRE(out != nullptr, "sla_csr_list_create: NULL out");
    *out = nullptr;
    SLA_REQUIRE(n_items >= 1, "sla_csr_list_create: n_items must be >= 1 (got %d)", n_items);
    SLA_REQUIRE(item_rows != nullptr, "sla_csr_list_create: NULL item_rows");
    SLA_REQUIRE(n_rows >= 0, "sla_csr_list_create: negative size");
    std::vector<int32_t> seg((size_t)n_items + 1);
    cudaStream_t s = as_stream(stream);
    if (cudaMemcpyAsync(seg.data(), item_rows, seg.size() * sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        set_error("sla_csr_list_create: cannot read item_rows");
        return SLA_ERR_CUDA;
    }
    SLA_REQUIRE(seg[0] == 0 && seg[n_items] == n_rows,
                "sla_csr_list_create: item_rows must run from 0 to n_rows (%d .. %d, n_rows %d)", seg[0],
                seg[n_items], n_rows);
    int32_t seg_max = 0;
    for (int32_t i = 0; i < n_items; ++i) {
        SLA_REQUIRE(seg[i + 1] >= seg[i], "sla_csr_list_create: item_rows decreases at item %d", i);
        seg_max = std::max(seg_max, seg[i + 1] - seg[i]);
    }
    sla_csr_t hh = nullptr;
    sla_status st = create_handle(n_rows, n_rows, nnz, rowptr, colind, 1, dtype, flags, stream, &hh, true);
    if (st != SLA_OK) return st;
    Csr *h = reinterpret_cast<Csr *>(hh);
    auto fail = [&](sla_status e) {
        sla_csr_destroy(hh);
        return e;
    };
    std::vector<int32_t> order(n_items);
    for (int32_t i = 0; i < n_items; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(),
                     [&](int32_t a, int32_t b) { return seg[a + 1] - seg[a] > seg[b + 1] - seg[b]; });
    unsigned long long *best = nullptr;
    if (cudaMalloc(&h->seg, seg.size() * sizeof(int32_t)) != cudaSuccess ||
        cudaMalloc(&h->seg_order, order.size() * sizeof(int32_t)) != cudaSuccess ||
        cudaMalloc(&best, sizeof(unsigned long long)) != cudaSuccess) {
        cudaFree(best);
        set_error("sla_csr_list_create: out of device memory");
        return fail(SLA_ERR_OOM);
    }
    unsigned long long code = ~0ull;
    if (cudaMemcpyAsync(h->seg, seg.data(), seg.size() * sizeof(int32_t), cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(h->seg_order, order.data(), order.size() * sizeof(int32_t), cudaMemcpyHostToDevice, s) !=
            cudaSuccess ||
        cudaMemsetAsync(best, 0xff, sizeof(unsigned long long), s) != cudaSuccess) {
        cudaFree(best);
        set_error("sla_csr_list_create: copy failed");
        return fail(SLA_ERR_CUDA);
    }
    if (n_rows > 0)
        list_check_kernel<<<(n_rows + 255) / 256, 256, 0, s>>>(n_rows, rowptr, colind, n_items, h->seg, best);
    const bool ok = cudaGetLastError() == cudaSuccess &&
                    cudaMemcpyAsync(&code, best, sizeof(code), cudaMemcpyDeviceToHost, s) == cudaSuccess &&
                    cudaStreamSynchronize(s) == cudaSuccess;
    cudaFree(best);
    if (!ok) {
        set_error("sla_csr_list_create: block check failed");
        return fail(SLA_ERR_CUDA);
    }
    if (code != ~0ull) {
        set_error("sla_csr_list_create: entry %lld lies outside its item's diagonal block",
                  (long long)(code & ((1ull << 40) - 1)));
        return fail(SLA_ERR_INVALID);
    }
    h->n_items = n_items;
    h->seg_max = seg_max;
    st = cg_configure_list(h);
    if (st != SLA_OK) return fail(st);
    *out = hh;
    return SLA_OK;
}

namespace {
sla_status create_handle(int32_t n_rows, int32_t n_cols, int64_t nnz, const int32_t *rowptr,
                         const int32_t *colind, int32_t batch, sla_dtype dtype, uint32_t flags,
                         void *stream, sla_csr_t *out, bool list) {
    SLA_REQUIRE(out != nullptr, "sla_csr_create: NULL out");
    *out = nullptr;
    SLA_REQUIRE(n_rows >= 0 && n_cols >= 0, "sla_csr_create: negative size");
    SLA_REQUIRE(nnz >= 0 && nnz <= INT_MAX, "sla_csr_create: nnz=%lld outside [0, 2^31)",
                (long long)nnz);
    SLA_REQUIRE(batch >= 1, "sla_csr_create: batch must be >= 1 (got %d)", batch);
    SLA_REQUIRE(dtype == SLA_F64 || dtype == SLA_F32, "sla_csr_create: bad dtype %d", (int)dtype);
    SLA_REQUIRE(rowptr != nullptr, "sla_csr_create: NULL rowptr");
    SLA_REQUIRE(nnz == 0 || colind != nullptr, "sla_csr_create: NULL colind");
    SLA_REQUIRE((flags & ~7u) == 0, "sla_csr_create: unknown flags 0x%x", flags);
    SLA_REQUIRE(!(flags & SLA_FLAG_SYMMETRIC) || n_rows == n_cols,
                "sla_csr_create: SYMMETRIC needs a square pattern");
    cudaStream_t s = as_stream(stream);

    Csr *h = new Csr();
    h->n_rows = n_rows;
    h->n_cols = n_cols;
    h->nnz = nnz;
    h->batch = batch;
    h->dtype = dtype;
    h->flags = flags;
    h->rowptr = rowptr;
    h->colind = colind;
    auto fail = [&](sla_status st) {
        sla_csr_destroy(reinterpret_cast<sla_csr_t>(h));
        return st;
    };
    if (cudaGetDevice(&h->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess) {
        set_error("sla_csr_create: no usable CUDA device");
        return fail(SLA_ERR_CUDA);
    }
    int64_t *scratch = nullptr;   // [0..1] check result, [2..3] row min/max
    if (cudaMalloc(&scratch, 4 * sizeof(int64_t)) != cudaSuccess) {
        set_error("sla_csr_create: cannot allocate scratch");
        return fail(SLA_ERR_OOM);
    }
    int64_t host[4] = {0, -1, 0, 0};
    sla_status st = SLA_OK;
    if (flags & SLA_FLAG_VALIDATE)
        st = enqueue_check(n_rows, n_cols, nnz, rowptr, colind, 0,
                           reinterpret_cast<unsigned long long *>(scratch), scratch, s);
    int *mm = reinterpret_cast<int *>(scratch + 2);
    if (st == SLA_OK && n_rows > 0) {
        row_stats_init_kernel<<<1, 1, 0, s>>>(mm);
        row_stats_kernel<<<(n_rows + 255) / 256, 256, 0, s>>>(n_rows, rowptr, mm);
        if (cudaGetLastError() != cudaSuccess) st = SLA_ERR_CUDA;
    }
    if (st == SLA_OK &&
        (cudaMemcpyAsync(host, scratch, sizeof host, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
         cudaStreamSynchronize(s) != cudaSuccess)) {
        set_error("sla_csr_create: %s", cudaGetErrorString(cudaGetLastError()));
        st = SLA_ERR_CUDA;
    }
    cudaFree(scratch);
    if (st != SLA_OK) return fail(st);
    if ((flags & SLA_FLAG_VALIDATE) && host[0] != 0) {
        static const char *what[] = {"", "rowptr[0] != 0", "rowptr decreases at row",
                                     "rowptr[n_rows] != nnz", "column out of range at entry",
                                     "columns not strictly increasing at entry",
                                     "missing diagonal at row"};
        set_error("sla_csr_create: invalid CSR pattern: %s %lld",
                  what[host[0] >= 1 && host[0] <= 6 ? host[0] : 0], (long long)host[1]);
        return fail(SLA_ERR_INVALID);
    }
    if (n_rows > 0) {
        int mmh[2];
        std::memcpy(mmh, &host[2], sizeof mmh);
        h->row_min = mmh[0];
        h->row_max = mmh[1];
        h->row_mean = (double)nnz / n_rows;
    }
    h->lanes = lanes_for_mean(h->row_mean);
    if (n_rows == n_cols && n_rows > 0) {
        if (cudaMalloc(&h->diagpos, (size_t)n_rows * sizeof(int32_t)) != cudaSuccess) {
            set_error("sla_csr_create: cannot allocate diagonal positions");
            return fail(SLA_ERR_OOM);
        }
        st = diag_positions(n_rows, rowptr, colind, h->diagpos, s);
        if (st != SLA_OK) return fail(st);
    }
    if (n_rows == n_cols && !list) {
        st = cg_configure(h);
        if (st == SLA_OK) st = cg_tile_deps(h, s);
        if (st != SLA_OK) return fail(st);
        const char *sv = getenv("SLA_SELL");
        if (h->lanes == 1 && n_rows > 0 && !(sv && sv[0] == '0')) {
            // rows sorted within windows only for the solver variant that keeps q in
            // HBM by row, with windows inside tiles (not the interleaved batch solver)
            const bool sort_ok = !h->onchip && h->il_blocks == 0 && h->tile_rows % kSellSortWindow == 0;
            st = build_sell(h, sort_ok, s);
            if (st != SLA_OK) return fail(st);
        }
    }
    if ((flags & SLA_FLAG_BUILD_TRANSPOSE) && !(flags & SLA_FLAG_SYMMETRIC)) {
        st = ensure_transpose(h, s);
        if (st != SLA_OK) return fail(st);
    }
    *out = reinterpret_cast<sla_csr_t>(h);
    return SLA_OK;
}
}  // namespace

extern "C" sla_status sla_csr_destroy(sla_csr_t hh) {
    Csr *h = reinterpret_cast<Csr *>(hh);
    if (!h) return SLA_OK;
    cudaFree(h->diagpos);
    cudaFree(h->rowptrT);
    cudaFree(h->colindT);
    cudaFree(h->permT);
    cudaFree(h->diagposT);
    cudaFree(h->sell_ptr);
    cudaFree(h->sell_cols);
    cudaFree(h->sell_map);
    cudaFree(h->sell_perm);
    cudaFree(h->sell_d16);
    cudaFree(h->dep_lo);
    cudaFree(h->dep_hi);
    cudaFree(h->seg);
    cudaFree(h->seg_order);
    delete h;
    return SLA_OK;
}

extern "C" sla_status sla_csr_get_props(sla_csr_t hh, sla_csr_props *p) {
    clear_error();
    Csr *h = reinterpret_cast<Csr *>(hh);
    SLA_REQUIRE(h && p, "sla_csr_get_props: NULL argument");
    p->n_rows = h->n_rows;
    p->n_cols = h->n_cols;
    p->nnz = h->nnz;
    p->batch = h->batch;
    p->dtype = (int32_t)h->dtype;
    p->row_min = h->row_min;
    p->row_max = h->row_max;
    p->row_mean = h->row_mean;
    p->lanes = h->lanes;
    p->grid_blocks = h->grid_blocks;
    p->block_fits = h->block_fits ? 1 : 0;
    p->has_transpose = h->has_transpose ? 1 : 0;
    p->grid_onchip = h->onchip ? (h->grid2 && h->has_sell ? 2 : 1) : 0;
    p->grid_tile_rows = h->tile_rows;
    p->sliced = h->has_sell ? (h->sell_w > 0 ? 2 : (h->sell_perm ? 3 : 1)) : 0;
    p->sliced_col_bytes = h->has_sell ? (h->sell_d16 ? 2 : 4) : 0;
    p->block_resident = h->block_mres ? 1 : 0;
    p->cluster_fits = h->cluster_fits ? 1 : 0;
    p->n_items = h->n_items;
    p->item_rows_max = h->seg_max;
    p->item_smem_rows = h->seg_smem_rows;
    p->interleaved = h->il_blocks > 0 && h->has_sell && !h->onchip ? 1 : 0;
    return SLA_OK;
}

extern "C" sla_status sla_csr_transpose_pattern(sla_csr_t hh, const int32_t **rowptrT,
                                                const int32_t **colindT, const int32_t **perm,
                                                void *stream) {
    SLA_RANGE("sla_csr_transpose_pattern");
    clear_error();
    Csr *h = reinterpret_cast<Csr *>(hh);
    SLA_REQUIRE(h && rowptrT && colindT && perm, "sla_csr_transpose_pattern: NULL argument");
    sla_status st = ensure_transpose(h, as_stream(stream));
    if (st != SLA_OK) return st;
    *rowptrT = h->rowptrT;
    *colindT = h->colindT;
    *perm = h->permT;
    return SLA_OK;
}
