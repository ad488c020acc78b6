// Shared internals of the sm_100a library behind include/sla.h: error
// reporting, the CSR handle, and device helpers (deterministic reductions and
// a bounded device-wide barrier for persistent cooperative kernels).
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include <cstdarg>
#include <cstdio>
#include <string>
#include <type_traits>

#include "../../include/sla.h"

namespace sla {

// ---------------------------------------------------------------- errors ----
void set_error(const char *fmt, ...);
void clear_error();

#define SLA_CHECK_CUDA(call)                                                   \
    do {                                                                       \
        cudaError_t e_ = (call);                                               \
        if (e_ != cudaSuccess) {                                               \
            ::sla::set_error("%s failed: %s (%s:%d)", #call,                   \
                             cudaGetErrorString(e_), __FILE__, __LINE__);      \
            return SLA_ERR_CUDA;                                               \
        }                                                                      \
    } while (0)

#define SLA_CHECK_LAUNCH()                                                     \
    do {                                                                       \
        cudaError_t e_ = cudaGetLastError();                                   \
        if (e_ != cudaSuccess) {                                               \
            ::sla::set_error("kernel launch failed: %s (%s:%d)",               \
                             cudaGetErrorString(e_), __FILE__, __LINE__);      \
            return SLA_ERR_CUDA;                                               \
        }                                                                      \
    } while (0)

#define SLA_REQUIRE(cond, ...)                                                 \
    do {                                                                       \
        if (!(cond)) {                                                         \
            ::sla::set_error(__VA_ARGS__);                                     \
            return SLA_ERR_INVALID;                                            \
        }                                                                      \
    } while (0)

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// Names a C entry point in profiler timelines (an NVTX range around the call,
// which encloses the kernels it enqueues); without a profiler attached the
// push and pop do nothing.
struct Range {
    explicit Range(const char *name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
    Range(const Range &) = delete;
    Range &operator=(const Range &) = delete;
};
#define SLA_RANGE(name) ::sla::Range sla_range_(name)

inline size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }

// Sequential carving of a caller workspace into 256-byte aligned pieces.
struct Carver {
    char *base;
    size_t off = 0;
    explicit Carver(void *p) : base(static_cast<char *>(p)) {}
    template <typename U>
    U *take(size_t count) {
        U *p = reinterpret_cast<U *>(base ? base + off : nullptr);
        off = align_up(off + count * sizeof(U));
        return p;
    }
};

// Rows handled by one thread block in row-parallel kernels.
constexpr int kRowBlock = 256;
// Threads of the persistent-grid and block-per-system CG kernels.
constexpr int kCgThreads = 512;

// ---------------------------------------------------------------- handle ----
struct Csr {
    int32_t n_rows = 0, n_cols = 0;
    int64_t nnz = 0;
    int32_t batch = 1;
    sla_dtype dtype = SLA_F64;
    uint32_t flags = 0;
    int device = 0;
    int num_sms = 0;
    const int32_t *rowptr = nullptr;   // borrowed
    const int32_t *colind = nullptr;   // borrowed
    int32_t *diagpos = nullptr;        // owned [n_rows]: position of A_ii, -1 if absent
    // A^T's pattern (owned; built on request)
    int32_t *rowptrT = nullptr, *colindT = nullptr, *permT = nullptr, *diagposT = nullptr;
    bool has_transpose = false;
    // statistics
    int32_t row_min = 0, row_max = 0;
    double row_mean = 0.0;
    int32_t lanes = 1;
    // persistent-grid CG layout
    int32_t grid_blocks = 0;           // cooperative grid size for this dtype
    int32_t tile_rows = 0;             // rows of one tile (tiles never straddle systems)
    int32_t ntiles = 0;                // tiles per system
    bool block_fits = false;           // one system fits the block-per-system solver
    bool onchip = false;               // grid solver keeps x, r, M^-1 in shared memory
    int32_t onchip_rpt = 0;            // rows a thread in the on-chip grid solver
    bool grid2 = false;                // single system, on chip, sliced: two barriers an iteration
    int32_t grid_threads = 0;          // threads of a grid-solver block
    size_t grid_smem = 0;              // dynamic shared memory of a grid-solver block
    size_t block_smem = 0;             // its dynamic shared memory per block
    bool block_mres = false;           // block solver keeps the whole system in shared memory
    bool cluster_fits = false;         // one system fits the cluster solver
    int32_t cluster_rows = 0;          // rows of one cluster block
    int32_t cluster_nnz = 0;           // most entries any cluster block holds
    size_t cluster_smem = 0;           // its dynamic shared memory
    int32_t *dep_lo = nullptr, *dep_hi = nullptr;  // owned [ntiles]: tiles a tile's gathers reach
    int32_t block_grid = 0;            // blocks of the block solver (each loops over systems)
    int32_t il_blocks = 0;             // batches of 2 or 4 in HBM: interleaved solver grid (0: none)
    // A list of independent systems (block-diagonal pattern; see sla_csr_list_create):
    // item s owns rows and columns [seg[s], seg[s+1]).
    int32_t n_items = 0;
    int32_t *seg = nullptr;            // owned [n_items + 1]
    int32_t *seg_order = nullptr;      // owned [n_items]: items by decreasing size
    int32_t seg_max = 0;               // rows of the largest item
    int32_t seg_smem_rows = 0;         // items up to this size keep their vectors in shared memory
    int32_t seg_grid = 0;              // blocks of the segment solver
    size_t seg_smem = 0;               // its dynamic shared memory per block
    // Sliced layout of the pattern for the solver's short-row SpMV (see sla_sell.cu):
    // slices of kSellRows consecutive rows, entry k of the slice's rows stored
    // together (padded to the slice's longest row).
    bool has_sell = false;
    int64_t sell_nnz = 0;              // stored entries including padding
    int32_t sell_w = 0;                // > 0: every slice padded to this width (no offsets needed)
    int32_t *sell_perm = nullptr;      // owned [n_rows] or null: row at each position (rows of each
                                       // 32-row window ordered by decreasing length)
    int16_t *sell_d16 = nullptr;       // owned [sell_nnz] or null: columns as offsets from their row
    int32_t *sell_ptr = nullptr;       // owned [n_slices + 1]: first entry of each slice
    int32_t *sell_cols = nullptr;      // owned [sell_nnz]: column (own row for padding)
    int32_t *sell_map = nullptr;       // owned [sell_nnz]: CSR position, -1 for padding
    // Grid of the pipelined one-thread-row SpMV (blocks resident at once; 0
    // until first used).
    int32_t pipe_grid_spmv = 0;
};

inline size_t dtype_size(sla_dtype dt) { return dt == SLA_F64 ? 8 : 4; }

// Picks the threads-per-row of row-parallel kernels from the mean row length.
int lanes_for_mean(double mean_row);

// Builds A^T's pattern into the handle (allocates once).
sla_status ensure_transpose(Csr *h, cudaStream_t s);

// Stable radix-sort based transpose of a pattern; used by the public call and
// the handle.  `ws` must hold transpose_ws_bytes().
size_t transpose_ws_bytes(int32_t n_rows, int32_t n_cols, int64_t nnz);
sla_status transpose_pattern(int32_t n_rows, int32_t n_cols, int64_t nnz,
                             const int32_t *rowptr, const int32_t *colind,
                             int32_t *rowptrT, int32_t *colindT, int32_t *perm,
                             void *ws, cudaStream_t s);

// valsT[b][s] = vals[b][permT[s]] for every system (needs the handle's A^T).
sla_status transpose_values(const Csr *h, const void *vals, void *valsT, cudaStream_t s);

// Device exclusive scan of unsigned counts (n entries; ws >= scan_ws_bytes(n)).
size_t scan_ws_bytes(int64_t n);
sla_status exclusive_scan(const unsigned *in, unsigned *out, int64_t n, void *ws, cudaStream_t s);

// Sliced layout (built at handle creation for short-row square patterns).
constexpr int kSellRows = 8;
constexpr int kSellSortWindow = 32;   // rows sorted by length together (one warp's rows)
// sort_ok: the solver that uses this layout keeps q by row index (vectors in
// HBM), so rows may be permuted within windows.
sla_status build_sell(Csr *h, bool sort_ok, cudaStream_t s);
sla_status cg_tile_deps(Csr *h, cudaStream_t s);   // in sla_cg.cu
// vals_sell[b][slot] = vals[b][sell_map[slot]] (0 for padding), every system.
sla_status sell_values(const Csr *h, const void *vals, void *vals_sell, cudaStream_t s);

// Diagonal positions of a square pattern (kernel; enqueue only).
sla_status diag_positions(int32_t n, const int32_t *rowptr, const int32_t *colind,
                          int32_t *diagpos, cudaStream_t s);

// ------------------------------------------------------- device helpers ----
__device__ __forceinline__ unsigned long long global_timer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Deterministic block sum of one double per thread; every thread of the block
// must call it.  The result is returned to all threads.  `red` holds >= 33
// doubles of shared memory.
template <int NT>
__device__ __forceinline__ double block_sum(double v, double *red) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        double s = lane < NW ? red[lane] : 0.0;
        s = warp_sum(s);
        if (lane == 0) red[32] = s;
    }
    __syncthreads();
    const double r = red[32];
    __syncthreads();
    return r;
}

// Two sums in one pass (same order as two block_sum calls).
template <int NT>
__device__ __forceinline__ void block_sum2(double &a, double &b, double *red) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    a = warp_sum(a);
    b = warp_sum(b);
    if (lane == 0) { red[warp] = a; red[32 + warp] = b; }
    __syncthreads();
    if (warp == 0) {
        double s = lane < NW ? red[lane] : 0.0;
        double t = lane < NW ? red[32 + lane] : 0.0;
        s = warp_sum(s);
        t = warp_sum(t);
        if (lane == 0) { red[64] = s; red[65] = t; }
    }
    __syncthreads();
    a = red[64];
    b = red[65];
    __syncthreads();
}

// Device-wide barrier for a cooperative (co-resident) grid.  sync[0] counts
// arrivals, sync[1] is the generation, sync[2] the error flag.  Each wait is
// bounded by timeout_ns of %globaltimer; a block that gives up sets the error
// flag, and blocks that see the flag give up too.  Returns false when the
// caller must leave the kernel.  Every thread of the block must call it.
__device__ __forceinline__ bool grid_barrier(unsigned *sync, unsigned nblocks,
                                             long long timeout_ns, int *flag_smem) {
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned *count = sync, *gen = sync + 1, *err = sync + 2;
        const unsigned g = ld_acquire_u32(gen);
        int ok = 1;
        __threadfence();
        const unsigned prev = atomicAdd(count, 1u);
        if (prev == nblocks - 1) {
            atomicExch(count, 0u);
            __threadfence();
            atomicAdd(gen, 1u);
        } else {
            const unsigned long long t0 = global_timer_ns();
            unsigned spins = 0;
            while (ld_acquire_u32(gen) == g) {
                if ((spins++ & 7u) == 0) {   // first poll, then every 8th
                    if (ld_acquire_u32(err) != 0) { ok = 0; break; }
                    if ((long long)(global_timer_ns() - t0) > timeout_ns) {
                        atomicExch(err, 1u);
                        ok = 0;
                        break;
                    }
                }
            }
        }
        if (ok && ld_acquire_u32(err) != 0) ok = 0;
        __threadfence();
        *flag_smem = ok;
    }
    __syncthreads();
    return *flag_smem != 0;
}

// ------------------------------------------------- bounds-checking build ----
// With SLA_DEBUG_BOUNDS=1 (the library's debug_bounds variant) every index the
// kernels take from the pattern (a column gathered from a vector, a CSR or
// sliced-layout entry, a diagonal position, an edge's entry) and every
// shared-memory or cluster-rank index derived from it is checked against its
// range before use.  A bad index is recorded (a count, and the smallest
// (code, index) pair) and replaced by 0, so the access stays in bounds and
// nothing traps; sla_debug_bounds_report reads the record.  Without the flag
// SLA_IDX is the index itself and no code is added.
enum {
    kBndColumn = 1,   // gathered column >= vector length
    kBndEntry = 2,    // entry position outside the value / column arrays
    kBndDiag = 3,     // diagonal position outside the entries
    kBndLocal = 4,    // shared-memory index or cluster rank out of range
    kBndEdge = 5      // edge endpoint or edge-to-entry slot out of range
};

#ifndef SLA_DEBUG_BOUNDS
#define SLA_DEBUG_BOUNDS 0
#endif

#if SLA_DEBUG_BOUNDS
// One record per translation unit (device variables of a file without
// relocatable device code are the file's own); each registers its reader.
namespace {
__device__ unsigned long long dbg_count = 0;
__device__ unsigned long long dbg_first = ~0ull;
}  // namespace

__device__ __forceinline__ long long dbg_index(long long i, long long n, int code) {
    if ((unsigned long long)i < (unsigned long long)n) return i;
    atomicAdd(&dbg_count, 1ull);
    atomicMin(&dbg_first, ((unsigned long long)code << 56) | ((unsigned long long)i & ((1ull << 56) - 1)));
    return 0;
}
#define SLA_IDX(i, n, code) \
    ((std::decay_t<decltype(i)>)::sla::dbg_index((long long)(i), (long long)(n), (code)))

using DbgReader = cudaError_t (*)(unsigned long long *count, unsigned long long *first, bool reset);
int dbg_register(DbgReader f);   // sla_handle.cu
namespace {
cudaError_t dbg_read(unsigned long long *count, unsigned long long *first, bool reset) {
    cudaError_t e = cudaMemcpyFromSymbol(count, dbg_count, sizeof(unsigned long long));
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(first, dbg_first, sizeof(unsigned long long));
    if (e == cudaSuccess && reset) {
        const unsigned long long zero = 0, none = ~0ull;
        e = cudaMemcpyToSymbol(dbg_count, &zero, sizeof zero);
        if (e == cudaSuccess) e = cudaMemcpyToSymbol(dbg_first, &none, sizeof none);
    }
    return e;
}
[[maybe_unused]] const int dbg_registered = dbg_register(&dbg_read);
}  // namespace
#else
#define SLA_IDX(i, n, code) (i)
#endif

}  // namespace sla
