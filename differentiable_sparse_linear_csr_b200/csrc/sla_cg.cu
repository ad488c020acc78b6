// Jacobi-preconditioned conjugate gradient, batched over systems that share
// one CSR pattern, with the whole iteration resident on the GPU.
//
// Method: torch-sla summary page, technical summary -- "Methodology" 1 (the
// iterative `.solve` of the PyTorch-native GPU backend; `SparseTensor` batches
// sharing a pattern), "Significance" (that backend's Jacobi preconditioner),
// "Methodology" 2 (the adjoint solve A^T lambda = dL/dx).  The pages give no
// algorithm listing; this is textbook Hestenes-Stiefel PCG:
//   r = b - A x, z = M^-1 r, p = z, rho = r.z
//   loop: q = A p; alpha = rho / p.q; x += alpha p; r -= alpha q;
//         stop on ||r|| <= max(rtol ||b||, atol) (or after exactly k steps);
//         z = M^-1 r; beta = r.z / rho; p = z + beta p
// Dot products accumulate in fp64 for both value types.
//
// Kernels, all with the iteration loop on the device and every wait bounded:
//  * cg_grid_kernel -- one persistent cooperative grid (all blocks resident)
//    for systems too large for one block.  Rows are split into fixed tiles; a
//    block owns the same tiles in every phase.  Device-wide barriers separate
//    SpMV+p.q, the r update with r.z and r.r (x += alpha p runs while the
//    following barrier completes), and the direction update; for one system
//    with banded tile dependencies, p-ready tile flags replace the third.
//    Vectors stay on chip (shared memory and registers) when a block's tile
//    fits, else in HBM.  Every block reduces the per-tile partials of a system
//    itself, in one fixed order, so all blocks take identical decisions
//    without extra communication; results are bit-reproducible run to run.
//  * cg_grid2_kernel -- the same for one system on chip with two barriers an
//    iteration: directions are formed while gathered in the next SpMV.
//  * cg_grid_il_kernel -- batches of 2 or 4 systems in HBM with values and
//    vectors interleaved by system, one column index for all of them.
//  * cg_block_kernel -- one thread block per system with x, r, p, q, M^-1 in
//    shared memory (small systems, large batches): no device-wide barrier.
//  * cg_cluster_kernel -- one 8-block thread-block cluster per small system,
//    the matrix slice and vectors in each block's shared memory, p over DSMEM.
//  * cg_segment_kernel -- lists of systems with their own patterns, one item
//    a block, largest first.
#include <cmath>
#include <cstdlib>
#include <cooperative_groups.h>

#include <algorithm>
#include <climits>
#include <vector>

#include "sla_rows.cuh"

namespace sla {

constexpr int kActive = -1;
constexpr long long kDefaultTimeoutNs = 5000000000LL;

template <typename T>
struct CgArgs {
    int n, B;
    int64_t nnz;
    const int32_t *rowptr, *colind, *diagpos;
    const T *vals;     // [B][nnz]
    const T *b;        // [B][n]
    T *x;              // [B][n]
    T *r, *p, *q, *d;  // [B][n] (grid kernel only)
    double *part;      // [4][B * ntiles] per-tile partial sums
    double *sysd;      // [4][B]: rho (two slots), ||b||, last ||r||^2
    int *state;        // [B]: kActive or the final status
    unsigned *sync;    // count, generation, error, systems still active
    int32_t *out_iters;
    double *out_relres;
    int32_t *out_status;
    double rtol, atol;
    int limit, fixed, precond, x0_given;
    long long timeout_ns;
    int tile_rows, ntiles;
    const int32_t *dep_lo, *dep_hi;        // tiles whose p a tile gathers (null: use a barrier)
    unsigned *pflag;                        // [ntiles] iteration whose p a tile has written
    const int32_t *sell_ptr, *sell_cols;   // sliced layout of the pattern (SELL kernels)
    const T *sell_vals;                     // [B][sell_nnz] values in that layout
    const SellRec<T> *sell_rec;             // or [B][sell_nnz] value-and-column records
    int64_t sell_nnz;
    int sell_w;         // > 0: every slice of the sliced layout is sell_w entries wide
    int sell_pipe;      // on-chip SpMV of widths 5 and 7: next row's columns loaded ahead
    const int32_t *sell_perm;   // or null: the row at each position of the sliced layout
    const int16_t *sell_d16;    // or null: the sliced layout's columns as offsets from their row
};

// ------------------------------------------------------------ helpers ----
constexpr int kMaxLocalTiles = 128;   // tiles one block of the grid kernel may own

template <typename T>
__device__ __forceinline__ void finalize(const CgArgs<T> &a, int s, int status, int iters,
                                         double relres, bool count_down) {
    a.state[s] = status;
    if (a.out_status) a.out_status[s] = status;
    if (a.out_iters) a.out_iters[s] = iters;
    if (a.out_relres) a.out_relres[s] = relres;
    if (count_down) atomicSub(a.sync + 3, 1u);
}

// Deterministic block sum of NV doubles per thread (fixed xor tree in each warp,
// then warp totals in warp order); every thread gets the sums.  red >= 33*NV.
template <int NT, int NV>
__device__ __forceinline__ void block_sums(double (&v)[NV], double *red) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        v[k] = warp_sum(v[k]);
        if (lane == 0) red[k * 33 + warp] = v[k];
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            double s = lane < NW ? red[k * 33 + lane] : 0.0;
            s = warp_sum(s);
            if (lane == 0) red[k * 33 + 32] = s;
        }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < NV; ++k) v[k] = red[k * 33 + 32];
    __syncthreads();
}

// Sum over a system's tile partials.  Thread t takes partials t, t+NT, ... in
// order and the block tree combines them, so every block computes the same
// value; all partials are fetched in one round of parallel loads.
template <int NT, int NV>
__device__ __forceinline__ void system_sums(const double *const (&arr)[NV], int ntiles,
                                            double (&out)[NV], double *red) {
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        double acc = 0.0;
        for (int j = threadIdx.x; j < ntiles; j += NT) acc += __ldcg(arr[k] + j);
        out[k] = acc;
    }
    block_sums<NT, NV>(out, red);
}

// system_sums for an array of partial pointers built at run time.
template <int NT, int NV>
__device__ __forceinline__ void system_sums_dyn(const double *const *arr, int ntiles, double (&out)[NV],
                                                double *red) {
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        double acc = 0.0;
        for (int j = threadIdx.x; j < ntiles; j += NT) acc += __ldcg(arr[k] + j);
        out[k] = acc;
    }
    block_sums<NT, NV>(out, red);
}

__device__ __forceinline__ void red_release_gpu_u32(unsigned *p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// grid_sync in two halves, for work that needs neither the barrier's partials
// nor other blocks' writes: grid_arrive announces the block (after a block
// barrier) and grid_wait completes the barrier.  Every block calls both, in
// this order, with nothing between them that other blocks wait for.
__device__ __forceinline__ void grid_arrive(unsigned *sync, unsigned &target) {
    __syncthreads();
    target += gridDim.x;
    if (threadIdx.x == 0) red_release_gpu_u32(sync, 1u);
}

__device__ __forceinline__ bool grid_wait(unsigned *sync, unsigned target, long long timeout_ns, int *flag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned *count = sync, *err = sync + 2;
        int ok = 1;
        const unsigned long long t0 = global_timer_ns();
        unsigned spins = 0;
        while ((int)(ld_acquire_u32(count) - target) < 0) {
            if ((spins++ & 7u) == 0) {
                if (ld_acquire_u32(err) != 0) { ok = 0; break; }
                if ((long long)(global_timer_ns() - t0) > timeout_ns) {
                    atomicExch(err, 1u);
                    ok = 0;
                    break;
                }
            }
        }
        if (ok && ld_acquire_u32(err) != 0) ok = 0;
        *flag = ok;
    }
    __syncthreads();
    return *flag != 0;
}

// Device-wide barrier on a monotonically increasing arrival counter: the k-th
// barrier of the launch completes when the counter reaches k * gridDim.x, a
// target every block knows, so arrival is a single fire-and-forget add and the
// wait is one polling load.  sync[0] counts, sync[2] is the error flag.  Each
// wait is bounded by timeout_ns of %globaltimer (checked on the first poll and
// every 8th after); a block that gives up raises the flag and blocks that see
// it give up too.  If `watch` is given, thread 0 also reads it after the
// barrier and *watched holds the value for the whole block.
__device__ __forceinline__ bool grid_sync(unsigned *sync, unsigned &target, long long timeout_ns,
                                          int *flag, const unsigned *watch = nullptr,
                                          unsigned *watched = nullptr) {
    __syncthreads();
    target += gridDim.x;
    if (threadIdx.x == 0) {
        unsigned *count = sync, *err = sync + 2;
        int ok = 1;
        // The arrival is a release at gpu scope: it orders every write of the
        // block (ordered before it by the block barrier above) before the
        // count; the polls below are acquires, so no separate fences are needed.
        red_release_gpu_u32(count, 1u);
        const unsigned long long t0 = global_timer_ns();
        unsigned spins = 0;
        while ((int)(ld_acquire_u32(count) - target) < 0) {
            if ((spins++ & 7u) == 0) {
                if (ld_acquire_u32(err) != 0) { ok = 0; break; }
                if ((long long)(global_timer_ns() - t0) > timeout_ns) {
                    atomicExch(err, 1u);
                    ok = 0;
                    break;
                }
            }
        }
        if (ok && ld_acquire_u32(err) != 0) ok = 0;
        if (watch) *watched = ld_acquire_u32(watch);
        *flag = ok;
    }
    __syncthreads();
    return *flag != 0;
}

__device__ __forceinline__ void st_release_u32(unsigned *p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Wait until tiles lo..hi (at most 32) have published p of iteration k: warp 0
// polls them in parallel with acquire loads, bounded like grid_sync.  Every
// thread of the block must call it; false means leave the kernel.
__device__ __forceinline__ bool wait_tiles(const unsigned *pflag, int lo, int hi, unsigned k,
                                           unsigned *sync, long long timeout_ns, int *flag) {
    if (threadIdx.x < 32) {
        const int t = lo + (int)threadIdx.x;
        int ok = 1;
        const unsigned long long t0 = global_timer_ns();
        unsigned spins = 0;
        while (true) {
            const bool ready = t > hi || ld_acquire_u32(pflag + t) >= k;
            if (__all_sync(0xffffffffu, ready)) break;
            if ((spins++ & 7u) == 0) {
                int bad = 0;
                if (threadIdx.x == 0)
                    bad = ld_acquire_u32(sync + 2) != 0 ||
                          (long long)(global_timer_ns() - t0) > timeout_ns;
                if (__shfl_sync(0xffffffffu, bad, 0)) {
                    if (threadIdx.x == 0) atomicExch(sync + 2, 1u);
                    ok = 0;
                    break;
                }
            }
        }
        if (threadIdx.x == 0) *flag = ok;
    }
    __syncthreads();
    return *flag != 0;
}

template <typename T>
__device__ void give_up(const CgArgs<T> &a) {
    // A wait ran out: every system this block owns reports it.
    if (threadIdx.x != 0) return;
    for (int tile = blockIdx.x; tile < a.B * a.ntiles; tile += gridDim.x)
        if (tile % a.ntiles == 0) {
            const int s = tile / a.ntiles;
            if (a.out_status) a.out_status[s] = SLA_TIMED_OUT;
            a.state[s] = SLA_TIMED_OUT;
        }
}

// ------------------------------------------------------- grid kernel ----
// q = A p over rows [r0, r1) of the sliced layout with vectors in HBM, one row
// a thread; the matrix streams past L1 (no-allocate loads).  Returns the
// thread's partial p.q.
template <int NT, typename T>
__device__ __forceinline__ double sell_tile_hbm(const CgArgs<T> &a, const T *svals, const T *pg, T *qg,
                                                int r0, int r1) {
    double acc = 0.0;
    for (int i = r0 + threadIdx.x; i < r1; i += NT) {
        const int row = a.sell_perm ? SLA_IDX(__ldg(a.sell_perm + i), a.n, kBndLocal) : i;
        const T qi = a.sell_d16
                         ? sell_row<1, true>(a.sell_ptr, a.sell_cols, a.sell_d16, svals, pg, i, row, a.n,
                                             a.sell_nnz, a.sell_w)
                         : sell_row<1, false>(a.sell_ptr, a.sell_cols, a.sell_d16, svals, pg, i, row, a.n,
                                              a.sell_nnz, a.sell_w);
        qg[row] = qi;
        acc += (double)pg[row] * (double)qi;
    }
    return acc;
}

// sell_tile_hbm for slices all W wide with 16-bit columns: the next row's
// position and column offsets load while the current row gathers.
template <int W, int NT, typename T>
__device__ __forceinline__ double sell_tile_hbm_w(const CgArgs<T> &a, const T *svals, const T *pg, T *qg,
                                                  int r0, int r1) {
    double acc = 0.0;
    int i = r0 + threadIdx.x;
    if (i >= r1) return acc;
    int rown = a.sell_perm ? SLA_IDX(__ldg(a.sell_perm + i), a.n, kBndLocal) : i;
    int dn[W];
    sell_d16_fetch<W, 1>(a.sell_d16, i, a.sell_nnz, dn);
    for (; i < r1; i += NT) {
        const int row = rown;
        int d[W];
#pragma unroll
        for (int k = 0; k < W; ++k) d[k] = dn[k];
        if (i + NT < r1) {
            rown = a.sell_perm ? SLA_IDX(__ldg(a.sell_perm + i + NT), a.n, kBndLocal) : i + NT;
            sell_d16_fetch<W, 1>(a.sell_d16, i + NT, a.sell_nnz, dn);
        }
        const T qi = sell_row_w<W, 1>(svals, pg, d, i, row, a.n, a.sell_nnz);
        qg[row] = qi;
        acc += (double)pg[row] * (double)qi;
    }
    return acc;
}

// Phase A of the on-chip solver for a tile whose sliced rows are all W wide
// with 16-bit columns: q of the thread's rows into qreg, returning its part
// of p.q; the next row's column offsets load while the current row gathers.
template <int W, int RPT, int NT, typename T>
__device__ __forceinline__ double onchip_rows_w(const CgArgs<T> &a, const T *svals, const T *pg, int r0,
                                                int r1, T (&qreg)[RPT]) {
    const int tid = threadIdx.x;
    double acc = 0.0;
    int dn[W];
    if (r0 + tid < r1) sell_d16_fetch<W>(a.sell_d16, r0 + tid, a.sell_nnz, dn);
#pragma unroll
    for (int j = 0; j < RPT; ++j) {
        const int i = r0 + tid + j * NT;
        int d[W];
#pragma unroll
        for (int k = 0; k < W; ++k) d[k] = dn[k];
        if (j + 1 < RPT && i + NT < r1) sell_d16_fetch<W>(a.sell_d16, i + NT, a.sell_nnz, dn);
        if (i < r1) {
            const T qi = sell_row_w<W>(svals, pg, d, i, i, a.n, a.sell_nnz);
            qreg[j] = qi;
            acc += (double)pg[i] * (double)qi;
        }
    }
    return acc;
}

// Every block owns the tiles blockIdx.x + lt * gridDim.x (lt = 0, 1, ...) for
// the whole solve and takes the decisions (breakdown, stop, alpha, beta) for
// them itself from the shared partials; ONCHIP keeps x, r and M^-1 of its one
// tile in shared memory and q in registers (RPT rows a thread), so only A and
// p travel through L2/HBM each iteration.
template <typename T, int LANES, bool ONCHIP, int RPT, int NT, bool SELL>
__global__ void __launch_bounds__(NT, ONCHIP ? 1 : 2)
cg_grid_kernel(CgArgs<T> a) {
    constexpr int LT = ONCHIP ? 1 : kMaxLocalTiles;   // tiles one block may own
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ double red[4 * 33];
    __shared__ double l_rho[LT], l_nb[LT], l_rr[LT], l_alpha[LT];
    __shared__ int l_state[LT];
    __shared__ int flag;
    __shared__ unsigned active;
    constexpr int NSUB = NT / LANES;
    const int tid = threadIdx.x, sub = tid / LANES, lane = tid % LANES;
    const int ntot = a.B * a.ntiles;
    const int G = gridDim.x;
    const int nlt = blockIdx.x < ntot ? (ntot - blockIdx.x + G - 1) / G : 0;
    // With one system spread over every block, each block sees every decision;
    // otherwise the count of active systems decides when the loop ends.
    const bool local_end = (a.B == 1 && a.ntiles >= G);
    // p-ready flags replace the barrier after the direction update when each
    // tile's gathers reach only a few tiles (one system spread over all blocks).
    const bool tile_flags = local_end && a.dep_lo != nullptr;
    double *P0 = a.part, *P1 = P0 + ntot, *P2 = P1 + ntot, *P3 = P2 + ntot;
    const int n = a.n;
    unsigned target = 0;
    T qreg[ONCHIP ? RPT : 1];
    // ONCHIP fp32: the tile's p, read once for x += alpha p and kept in
    // registers for the direction update (q's registers are free again by
    // then); fp64 keeps re-reading it (two more registers a row spill there)
    constexpr bool KEEP_P = ONCHIP && sizeof(T) == 4;
    T preg[KEEP_P ? RPT : 1];
    T *xs_ = reinterpret_cast<T *>(smem_raw);     // ONCHIP: [tile_rows] each
    T *rs_ = xs_ + (ONCHIP ? a.tile_rows : 0);
    T *ds_ = rs_ + (ONCHIP ? a.tile_rows : 0);

    if (blockIdx.x == 0 && tid == 0) a.sync[3] = (unsigned)a.B;

    // ---- init: r = b - A x0 (or b), z = M^-1 r, p = z; partials of b.b, r.z, r.r
    for (int lt = 0; lt < nlt; ++lt) {
        const int tile = blockIdx.x + lt * G;
        const int s = tile / a.ntiles, tt = tile % a.ntiles;
        const int r0 = tt * a.tile_rows, r1 = min(n, r0 + a.tile_rows);
        const T *vs = a.vals + (int64_t)s * a.nnz;
        const T *bs = a.b + (int64_t)s * n;
        T *xg = a.x + (int64_t)s * n, *pg = a.p + (int64_t)s * n, *qg = a.q + (int64_t)s * n;
        if (a.x0_given) {
            for (int i = r0 + sub; i < r1; i += NSUB) {
                const T v = row_dot<T, LANES>(a.rowptr, a.colind, vs, xg, i, lane, n, a.nnz);
                if (lane == 0) qg[i] = v;
            }
            __syncthreads();
        }
        double acc[4] = {0.0, 0.0, 0.0, 0.0};   // b.b, r.z, r.r, bad diagonals
        for (int i = r0 + tid; i < r1; i += NT) {
            const T bi = bs[i];
            const T xi = a.x0_given ? xg[i] : T(0);
            const T ri = a.x0_given ? bi - qg[i] : bi;
            T di = T(1);
            if (a.precond) {
                const int dp = __ldg(a.diagpos + i);
                const T dv = dp >= 0 ? __ldg(vs + SLA_IDX(dp, a.nnz, kBndDiag)) : T(0);
                if (!(dv > T(0))) acc[3] += 1.0;
                di = T(1) / dv;
            }
            const T zi = di * ri;
            pg[i] = zi;
            if constexpr (ONCHIP) {
                xs_[i - r0] = xi;
                rs_[i - r0] = ri;
                ds_[i - r0] = di;
            } else {
                if (!a.x0_given) xg[i] = T(0);
                a.r[(int64_t)s * n + i] = ri;
                a.d[(int64_t)s * n + i] = di;
            }
            acc[0] += (double)bi * (double)bi;
            acc[1] += (double)ri * (double)zi;
            acc[2] += (double)ri * (double)ri;
        }
        block_sums<NT, 4>(acc, red);
        if (tid == 0) {
            P0[tile] = acc[0];
            P1[tile] = acc[1];
            P2[tile] = acc[2];
            P3[tile] = acc[3];
        }
    }
    if (!grid_sync(a.sync, target, a.timeout_ns, &flag)) { give_up(a); return; }

    // ---- initial decisions, taken identically by every block holding a tile
    for (int lt = 0; lt < nlt; ++lt) {
        const int tile = blockIdx.x + lt * G;
        const int s = tile / a.ntiles, tt = tile % a.ntiles;
        const int off = s * a.ntiles;
        const double *const arr[4] = {P0 + off, P1 + off, P2 + off, P3 + off};
        double sum[4];
        system_sums<NT, 4>(arr, a.ntiles, sum, red);
        const double bb = sum[0], rho0 = sum[1], rr = sum[2], bad = sum[3];
        const double nb = sqrt(bb);
        const double tol = fmax(a.rtol * nb, a.atol);
        int st = kActive;
        double relres = 0.0;
        if (nb == 0.0) st = SLA_CONVERGED;
        else if (!isfinite(nb)) st = SLA_NONFINITE;
        else if (a.precond && bad > 0.0) { st = SLA_BREAKDOWN; relres = sqrt(rr) / nb; }
        else if (!a.fixed && sqrt(rr) <= tol) { st = SLA_CONVERGED; relres = sqrt(rr) / nb; }
        else if (rr == 0.0) st = SLA_CONVERGED;
        if (nb == 0.0) {
            const int r0 = tt * a.tile_rows, r1 = min(n, r0 + a.tile_rows);
            for (int i = r0 + tid; i < r1; i += NT) {
                if constexpr (ONCHIP) xs_[i - r0] = T(0);
                else a.x[(int64_t)s * n + i] = T(0);
            }
        }
        if (tid == 0) {
            l_state[lt] = st;
            l_rho[lt] = rho0;
            l_nb[lt] = nb;
            l_rr[lt] = rr;
            if (tt == 0) {
                if (st == kActive) a.state[s] = kActive;
                else finalize(a, s, st, 0, relres, true);
            }
        }
    }
    __syncthreads();
    bool more;
    if (local_end) {
        more = nlt > 0 && l_state[0] == kActive;
    } else {
        if (!grid_sync(a.sync, target, a.timeout_ns, &flag, a.sync + 3, &active)) { give_up(a); return; }
        more = active != 0;
    }

    int k = 0;
    while (more) {
        // ---- phase A: q = A p and the partials of p.q
        for (int lt = 0; lt < nlt; ++lt) {
            if (l_state[lt] != kActive) continue;
            const int tile = blockIdx.x + lt * G;
            const int s = tile / a.ntiles, tt = tile % a.ntiles;
            if (tile_flags && k > 0 &&
                !wait_tiles(a.pflag, __ldg(a.dep_lo + tt), __ldg(a.dep_hi + tt), (unsigned)k,
                            a.sync, a.timeout_ns, &flag)) {
                give_up(a);
                return;
            }
            const int r0 = tt * a.tile_rows, r1 = min(n, r0 + a.tile_rows);
            const T *vs = a.vals + (int64_t)s * a.nnz;
            const T *pg = a.p + (int64_t)s * n;
            double acc[1] = {0.0};
            if constexpr (ONCHIP && SELL) {
                if (a.sell_rec) {
                    const SellRec<T> *rec = a.sell_rec + (int64_t)s * a.sell_nnz;
#pragma unroll
                    for (int j = 0; j < RPT; ++j) {
                        const int i = r0 + tid + j * NT;
                        if (i < r1) {
                            const T qi = sell_row_rec<false>(a.sell_ptr, rec, pg, i, n, a.sell_nnz);
                            qreg[j] = qi;
                            acc[0] += (double)pg[i] * (double)qi;
                        }
                    }
                } else if (a.sell_d16 && a.sell_w == 5 && a.sell_pipe) {
                    acc[0] = onchip_rows_w<5, RPT, NT>(a, a.sell_vals + (int64_t)s * a.sell_nnz, pg, r0, r1, qreg);
                } else if (sizeof(T) == 4 && a.sell_d16 && a.sell_w == 7 && a.sell_pipe) {
                    acc[0] = onchip_rows_w<7, RPT, NT>(a, a.sell_vals + (int64_t)s * a.sell_nnz, pg, r0, r1, qreg);
                } else {
                    const T *svals = a.sell_vals + (int64_t)s * a.sell_nnz;
#pragma unroll
                    for (int j = 0; j < RPT; ++j) {
                        const int i = r0 + tid + j * NT;
                        if (i < r1) {
                            const T qi = a.sell_d16
                                ? sell_row<0, true>(a.sell_ptr, a.sell_cols, a.sell_d16, svals, pg, i, i, n,
                                                    a.sell_nnz, a.sell_w)
                                : sell_row<0, false>(a.sell_ptr, a.sell_cols, a.sell_d16, svals, pg, i, i, n,
                                                     a.sell_nnz, a.sell_w);
                            qreg[j] = qi;
                            acc[0] += (double)pg[i] * (double)qi;
                        }
                    }
                }
            } else if constexpr (ONCHIP) {
#pragma unroll
                for (int j = 0; j < RPT; ++j) {
                    const int i = r0 + tid + j * NT;
                    if (i < r1) {
                        const T qi = row_dot<T, 1>(a.rowptr, a.colind, vs, pg, i, 0, n, a.nnz);
                        qreg[j] = qi;
                        acc[0] += (double)pg[i] * (double)qi;
                    }
                }
            } else if constexpr (SELL) {
                T *qg = a.q + (int64_t)s * n;
                if (a.sell_rec) {
                    const SellRec<T> *rec = a.sell_rec + (int64_t)s * a.sell_nnz;
                    for (int i = r0 + tid; i < r1; i += NT) {
                        const T qi = sell_row_rec<true>(a.sell_ptr, rec, pg, i, n, a.sell_nnz);
                        const int row = a.sell_perm ? SLA_IDX(__ldg(a.sell_perm + i), n, kBndLocal) : i;
                        qg[row] = qi;
                        acc[0] += (double)pg[row] * (double)qi;
                    }
                } else {
                    const T *svals = a.sell_vals + (int64_t)s * a.sell_nnz;
                    if (a.sell_d16 && a.sell_w == 7 && a.sell_pipe)
                        acc[0] = sell_tile_hbm_w<7, NT>(a, svals, pg, qg, r0, r1);
                    else if (a.sell_d16 && a.sell_w == 5 && a.sell_pipe)
                        acc[0] = sell_tile_hbm_w<5, NT>(a, svals, pg, qg, r0, r1);
                    else
                        acc[0] = sell_tile_hbm<NT>(a, svals, pg, qg, r0, r1);
                }
            } else {
                T *qg = a.q + (int64_t)s * n;
                for (int i = r0 + sub; i < r1; i += NSUB) {
                    const T qi = row_dot<T, LANES>(a.rowptr, a.colind, vs, pg, i, lane, n, a.nnz);
                    if (lane == 0) {
                        qg[i] = qi;
                        acc[0] += (double)pg[i] * (double)qi;
                    }
                }
            }
            block_sums<NT, 1>(acc, red);
            if (tid == 0) P0[tile] = acc[0];
        }
        if (!grid_sync(a.sync, target, a.timeout_ns, &flag)) { give_up(a); return; }
        ++k;

        // ---- phase B: alpha; r -= alpha q; partials of r.z and r.r
        for (int lt = 0; lt < nlt; ++lt) {
            if (l_state[lt] != kActive) continue;
            const int tile = blockIdx.x + lt * G;
            const int s = tile / a.ntiles, tt = tile % a.ntiles;
            const double *const arr[1] = {P0 + s * a.ntiles};
            double sg[1];
            system_sums<NT, 1>(arr, a.ntiles, sg, red);
            const double sigma = sg[0];
            if (!isfinite(sigma) || !(sigma > 0.0)) {
                const int st = isfinite(sigma) ? SLA_BREAKDOWN : SLA_NONFINITE;
                if (tid == 0) {
                    l_state[lt] = st;
                    if (tt == 0) finalize(a, s, st, k - 1, sqrt(l_rr[lt]) / l_nb[lt], true);
                }
                __syncthreads();
                continue;
            }
            const double alpha = l_rho[lt] / sigma;
            const T al = (T)alpha;
            const int r0 = tt * a.tile_rows, r1 = min(n, r0 + a.tile_rows);
            double acc[2] = {0.0, 0.0};
            if constexpr (ONCHIP) {
#pragma unroll
                for (int j = 0; j < RPT; ++j) {
                    const int i = r0 + tid + j * NT;
                    if (i < r1) {
                        const T ri = rs_[i - r0] - al * qreg[j];
                        rs_[i - r0] = ri;
                        const T zi = ds_[i - r0] * ri;
                        acc[0] += (double)ri * (double)zi;
                        acc[1] += (double)ri * (double)ri;
                    }
                }
            } else {
                T *rg = a.r + (int64_t)s * n;
                const T *qg = a.q + (int64_t)s * n, *dg = a.d + (int64_t)s * n;
#pragma unroll 4
                for (int i = r0 + tid; i < r1; i += NT) {
                    const T ri = rg[i] - al * qg[i];
                    rg[i] = ri;
                    const T zi = dg[i] * ri;
                    acc[0] += (double)ri * (double)zi;
                    acc[1] += (double)ri * (double)ri;
                }
            }
            block_sums<NT, 2>(acc, red);
            if (tid == 0) {
                P1[tile] = acc[0];
                P2[tile] = acc[1];
                l_alpha[lt] = alpha;
            }
        }
        // x += alpha p needs neither beta nor other blocks: it runs while the
        // barrier completes
        grid_arrive(a.sync, target);
        for (int lt = 0; lt < nlt; ++lt) {
            if (l_state[lt] != kActive) continue;
            const int tile = blockIdx.x + lt * G;
            const int s = tile / a.ntiles, tt = tile % a.ntiles;
            const T al = (T)l_alpha[lt];
            const int r0 = tt * a.tile_rows, r1 = min(n, r0 + a.tile_rows);
            const T *pg = a.p + (int64_t)s * n;
            if constexpr (ONCHIP) {
#pragma unroll
                for (int j = 0; j < RPT; ++j) {
                    const int i = r0 + tid + j * NT;
                    if (i < r1) {
                        const T pj = pg[i];
                        if constexpr (KEEP_P) preg[j] = pj;
                        xs_[i - r0] = xs_[i - r0] + al * pj;
                    }
                }
            } else {
                T *xg = a.x + (int64_t)s * n;
#pragma unroll 4
                for (int i = r0 + tid; i < r1; i += NT) xg[i] = xg[i] + al * pg[i];
            }
        }
        if (!grid_wait(a.sync, target, a.timeout_ns, &flag)) { give_up(a); return; }

        // ---- phase C: stopping test; beta; p = z + beta p
        for (int lt = 0; lt < nlt; ++lt) {
            if (l_state[lt] != kActive) continue;
            const int tile = blockIdx.x + lt * G;
            const int s = tile / a.ntiles, tt = tile % a.ntiles;
            const double *const arr[2] = {P1 + s * a.ntiles, P2 + s * a.ntiles};
            double sum[2];
            system_sums<NT, 2>(arr, a.ntiles, sum, red);
            const double rho_new = sum[0], rr = sum[1];
            const double nb = l_nb[lt];
            const double tol = fmax(a.rtol * nb, a.atol);
            int st = kActive;
            if (!isfinite(rr)) st = SLA_NONFINITE;
            else if (!a.fixed && sqrt(rr) <= tol) st = SLA_CONVERGED;
            else if (rr == 0.0) st = SLA_CONVERGED;
            else if (k >= a.limit) st = a.fixed ? SLA_FIXED_DONE : SLA_NOT_CONVERGED;
            const T bt = (T)(rho_new / l_rho[lt]);
            const bool go_on = st == kActive;
            const int r0 = tt * a.tile_rows, r1 = min(n, r0 + a.tile_rows);
            T *pg = a.p + (int64_t)s * n;
            if (go_on) {
                if constexpr (ONCHIP) {
#pragma unroll
                    for (int j = 0; j < RPT; ++j) {
                        const int i = r0 + tid + j * NT;
                        if (i < r1) {
                            T pj;
                            if constexpr (KEEP_P) pj = preg[j];
                            else pj = pg[i];
                            pg[i] = ds_[i - r0] * rs_[i - r0] + bt * pj;
                        }
                    }
                } else {
                    const T *rg = a.r + (int64_t)s * n, *dg = a.d + (int64_t)s * n;
#pragma unroll 4
                    for (int i = r0 + tid; i < r1; i += NT) pg[i] = dg[i] * rg[i] + bt * pg[i];
                }
            }
            __syncthreads();
            if (tid == 0) {
                if (tile_flags && go_on) {
                    st_release_u32(a.pflag + tt, (unsigned)k);   // release: the tile's p first
                }
                if (go_on) {
                    l_rho[lt] = rho_new;
                    l_rr[lt] = rr;
                } else {
                    l_state[lt] = st;
                    if (tt == 0) finalize(a, s, st, k, sqrt(rr) / nb, true);
                }
            }
        }
        if (tile_flags) {
            __syncthreads();
            more = l_state[0] == kActive;
        } else if (local_end) {
            if (!grid_sync(a.sync, target, a.timeout_ns, &flag)) { give_up(a); return; }
            more = l_state[0] == kActive;
        } else {
            if (!grid_sync(a.sync, target, a.timeout_ns, &flag, a.sync + 3, &active)) { give_up(a); return; }
            more = active != 0;
        }
    }
    if constexpr (ONCHIP) {
        for (int lt = 0; lt < nlt; ++lt) {
            const int tile = blockIdx.x + lt * G;
            const int s = tile / a.ntiles, tt = tile % a.ntiles;
            const int r0 = tt * a.tile_rows, r1 = min(n, r0 + a.tile_rows);
            T *xg = a.x + (int64_t)s * n;
            for (int i = r0 + tid; i < r1; i += NT) xg[i] = xs_[i - r0];
        }
    }
}

// --------------------------------------------- two-sync grid kernel ----
// The persistent solver for one system with x, r and M^-1 on chip and the
// sliced layout, with two device-wide barriers per iteration instead of three:
// the SpMV of iteration k forms p_k(j) = z_{k-1}(j) + beta p_{k-1}(j) per
// gathered entry from z = M^-1 r (written by each row's owner when it updates
// r) and the previous direction (p double buffered), and x and r are updated
// together once alpha is known.  Workspace vectors: a.r holds z, a.p and a.q
// the two directions.
template <typename T, int RPT, int NT>
__global__ void __launch_bounds__(NT, 1)
cg_grid2_kernel(CgArgs<T> a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ double red[4 * 33];
    __shared__ int flag;
    const int tid = threadIdx.x;
    const int n = a.n;
    const int tile = blockIdx.x;                 // one tile per block, one system
    const bool has_tile = tile < a.ntiles;
    const int r0 = tile * a.tile_rows, r1 = has_tile ? min(n, r0 + a.tile_rows) : r0;
    double *P0 = a.part, *P1 = P0 + a.ntiles, *P2 = P1 + a.ntiles, *P3 = P2 + a.ntiles;
    T *xs = reinterpret_cast<T *>(smem_raw);
    T *rs = xs + a.tile_rows, *ds = rs + a.tile_rows;
    T *zg = a.r, *pbuf[2] = {a.p, a.q};
    const T *svals = a.sell_vals;
    unsigned target = 0;
    T qreg[RPT];

    // ---- init: r = b - A x0 (or b), M^-1, z_0 = M^-1 r_0, p_0 = 0
    {
        const T *bs = a.b;
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        if (a.x0_given && has_tile) {
#pragma unroll
            for (int j = 0; j < RPT; ++j) {
                const int i = r0 + tid + j * NT;
                if (i < r1) qreg[j] = row_dot<T, 1>(a.rowptr, a.colind, a.vals, a.x, i, 0, a.n, a.nnz);
            }
        }
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
            const int i = r0 + tid + j * NT;
            if (i < r1) {
                const T bi = bs[i];
                const T xi = a.x0_given ? a.x[i] : T(0);
                const T ri = a.x0_given ? bi - qreg[j] : bi;
                T di = T(1);
                if (a.precond) {
                    const int dp = __ldg(a.diagpos + i);
                    const T dv = dp >= 0 ? __ldg(a.vals + SLA_IDX(dp, a.nnz, kBndDiag)) : T(0);
                    if (!(dv > T(0))) acc[3] += 1.0;
                    di = T(1) / dv;
                }
                const T zi = di * ri;
                xs[i - r0] = xi;
                rs[i - r0] = ri;
                ds[i - r0] = di;
                zg[i] = zi;
                pbuf[0][i] = T(0);
                acc[0] += (double)bi * (double)bi;
                acc[1] += (double)ri * (double)zi;
                acc[2] += (double)ri * (double)ri;
            }
        }
        block_sums<NT, 4>(acc, red);
        if (tid == 0 && has_tile) {
            P0[tile] = acc[0];
            P1[tile] = acc[1];
            P2[tile] = acc[2];
            P3[tile] = acc[3];
        }
    }
    if (!grid_sync(a.sync, target, a.timeout_ns, &flag)) { give_up(a); return; }
    double nb, tol, rho, rr;
    int st = kActive;
    double relres = 0.0;
    {
        const double *const arr[4] = {P0, P1, P2, P3};
        double sum[4];
        system_sums<NT, 4>(arr, a.ntiles, sum, red);
        nb = sqrt(sum[0]);
        rho = sum[1];
        rr = sum[2];
        tol = fmax(a.rtol * nb, a.atol);
        if (nb == 0.0) st = SLA_CONVERGED;
        else if (!isfinite(nb)) st = SLA_NONFINITE;
        else if (a.precond && sum[3] > 0.0) { st = SLA_BREAKDOWN; relres = sqrt(rr) / nb; }
        else if (!a.fixed && sqrt(rr) <= tol) { st = SLA_CONVERGED; relres = sqrt(rr) / nb; }
        else if (rr == 0.0) st = SLA_CONVERGED;
        if (nb == 0.0)
            for (int i = r0 + tid; i < r1; i += NT) xs[i - r0] = T(0);
    }
    int k = 0;
    T bt = T(0);
    while (st == kActive) {
        // ---- SpMV with p_{k+1} = z_k + beta_k p_k, partials of p.q
        const T *pprev = pbuf[k & 1];
        T *pcur = pbuf[(k + 1) & 1];
        double acc[1] = {0.0};
        if (a.sell_d16 && a.sell_w == 5 && a.sell_pipe) {
            // the next row's column offsets load while this row gathers
            int dn[5];
            if (r0 + tid < r1) sell_d16_fetch<5>(a.sell_d16, r0 + tid, a.sell_nnz, dn);
#pragma unroll
            for (int j = 0; j < RPT; ++j) {
                const int i = r0 + tid + j * NT;
                int d[5];
#pragma unroll
                for (int k = 0; k < 5; ++k) d[k] = dn[k];
                if (j + 1 < RPT && i + NT < r1) sell_d16_fetch<5>(a.sell_d16, i + NT, a.sell_nnz, dn);
                if (i < r1) {
                    const T qi = sell_row_dir_w<5>(svals, zg, pprev, bt, d, i, a.n, a.sell_nnz);
                    qreg[j] = qi;
                    T pi;
                    if constexpr (sizeof(T) == 8) pi = __fma_rn(bt, pprev[i], __dmul_rn(ds[i - r0], rs[i - r0]));
                    else pi = __fmaf_rn(bt, pprev[i], __fmul_rn(ds[i - r0], rs[i - r0]));
                    pcur[i] = pi;
                    acc[0] += (double)pi * (double)qi;
                }
            }
        } else {
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
            const int i = r0 + tid + j * NT;
            if (i < r1) {
                const T qi = a.sell_d16
                    ? sell_row_dir<true>(a.sell_ptr, a.sell_cols, a.sell_d16, svals, zg, pprev, bt, i, a.n,
                                         a.sell_nnz, a.sell_w)
                    : sell_row_dir<false>(a.sell_ptr, a.sell_cols, a.sell_d16, svals, zg, pprev, bt, i, a.n,
                                          a.sell_nnz, a.sell_w);
                qreg[j] = qi;
                T pi;
                if constexpr (sizeof(T) == 8) pi = __fma_rn(bt, pprev[i], __dmul_rn(ds[i - r0], rs[i - r0]));
                else pi = __fmaf_rn(bt, pprev[i], __fmul_rn(ds[i - r0], rs[i - r0]));
                pcur[i] = pi;
                acc[0] += (double)pi * (double)qi;
            }
        }
        }
        block_sums<NT, 1>(acc, red);
        if (tid == 0 && has_tile) P0[tile] = acc[0];
        if (!grid_sync(a.sync, target, a.timeout_ns, &flag)) { give_up(a); return; }
        double sg[1];
        {
            const double *const arr[1] = {P0};
            system_sums<NT, 1>(arr, a.ntiles, sg, red);
        }
        const double sigma = sg[0];
        if (!isfinite(sigma) || !(sigma > 0.0)) {
            st = isfinite(sigma) ? SLA_BREAKDOWN : SLA_NONFINITE;
            relres = sqrt(rr) / nb;
            break;
        }
        const T al = (T)(rho / sigma);
        ++k;
        // ---- x += alpha p; r -= alpha q; z = M^-1 r; partials of r.z, r.r
        double acc2[2] = {0.0, 0.0};
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
            const int i = r0 + tid + j * NT;
            if (i < r1) {
                xs[i - r0] = xs[i - r0] + al * pcur[i];
                const T ri = rs[i - r0] - al * qreg[j];
                rs[i - r0] = ri;
                T zi;
                if constexpr (sizeof(T) == 8) zi = __dmul_rn(ds[i - r0], ri);
                else zi = __fmul_rn(ds[i - r0], ri);
                zg[i] = zi;
                acc2[0] += (double)ri * (double)zi;
                acc2[1] += (double)ri * (double)ri;
            }
        }
        block_sums<NT, 2>(acc2, red);
        if (tid == 0 && has_tile) {
            P1[tile] = acc2[0];
            P2[tile] = acc2[1];
        }
        if (!grid_sync(a.sync, target, a.timeout_ns, &flag)) { give_up(a); return; }
        double sum[2];
        {
            const double *const arr[2] = {P1, P2};
            system_sums<NT, 2>(arr, a.ntiles, sum, red);
        }
        const double rho_new = sum[0];
        rr = sum[1];
        relres = sqrt(rr) / nb;
        if (!isfinite(rr)) st = SLA_NONFINITE;
        else if (!a.fixed && sqrt(rr) <= tol) st = SLA_CONVERGED;
        else if (rr == 0.0) st = SLA_CONVERGED;
        else if (k >= a.limit) st = a.fixed ? SLA_FIXED_DONE : SLA_NOT_CONVERGED;
        bt = (T)(rho_new / rho);
        rho = rho_new;
    }
    for (int i = r0 + tid; i < r1; i += NT) a.x[i] = xs[i - r0];
    if (blockIdx.x == 0 && tid == 0) finalize(a, 0, st, k, relres, false);
}

// ------------------------------------------------------ block kernel ----
// One block per system (a block loops over systems).  With MRES the whole
// system lives in shared memory: the shared pattern is loaded once per block,
// a system's values once per solve, and the iterations touch no global memory.
template <typename T, int LANES, bool MRES>
__global__ void __launch_bounds__(kCgThreads)
cg_block_kernel(CgArgs<T> a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ double red[72];
    constexpr int NSUB = kCgThreads / LANES;
    const int tid = threadIdx.x, sub = tid / LANES, lane = tid % LANES;
    const int n = a.n;
    T *xs = reinterpret_cast<T *>(smem_raw);
    T *rs = xs + n, *ps = rs + n, *qs = ps + n, *ds = qs + n;
    // matrix-resident layout: values, then column indices, then row pointers
    T *vals_s = ds + n;
    int32_t *cols_s = reinterpret_cast<int32_t *>(vals_s + (MRES ? a.nnz : 0));
    int32_t *rp_s = cols_s + (MRES ? a.nnz : 0);
    if constexpr (MRES) {
        for (int64_t t = tid; t < a.nnz; t += kCgThreads) cols_s[t] = __ldg(a.colind + t);
        for (int i = tid; i <= n; i += kCgThreads) rp_s[i] = __ldg(a.rowptr + i);
    }

    for (int s = blockIdx.x; s < a.B; s += gridDim.x) {
        const T *vs = a.vals + (int64_t)s * a.nnz;
        const T *bs = a.b + (int64_t)s * n;
        T *xg = a.x + (int64_t)s * n;
        __syncthreads();
        if constexpr (MRES) {
            for (int64_t t = tid; t < a.nnz; t += kCgThreads) vals_s[t] = __ldg(vs + t);
            __syncthreads();
        }
        auto spmv_row = [&](const T *v, int i) -> T {
            if constexpr (MRES) return row_dot_shared<T, LANES>(rp_s, cols_s, vals_s, v, i, lane, n, a.nnz);
            else return row_dot<T, LANES>(a.rowptr, a.colind, vs, v, i, lane, n, a.nnz);
        };
        if (a.x0_given) {
            for (int i = tid; i < n; i += kCgThreads) xs[i] = xg[i];
            __syncthreads();
            for (int i = sub; i < n; i += NSUB) {
                const T v = spmv_row(xs, i);
                if (lane == 0) qs[i] = v;
            }
            __syncthreads();
        }
        double bb = 0.0, rho = 0.0, rr = 0.0, bad = 0.0;
        for (int i = tid; i < n; i += kCgThreads) {
            const T bi = bs[i];
            T ri;
            if (a.x0_given) {
                ri = bi - qs[i];
            } else {
                ri = bi;
                xs[i] = T(0);
            }
            T di = T(1);
            if (a.precond) {
                const int dp = __ldg(a.diagpos + i);
                const T dv = dp >= 0 ? __ldg(vs + SLA_IDX(dp, a.nnz, kBndDiag)) : T(0);
                if (!(dv > T(0))) bad += 1.0;
                di = T(1) / dv;
            }
            const T zi = di * ri;
            rs[i] = ri;
            ps[i] = zi;
            ds[i] = di;
            bb += (double)bi * (double)bi;
            rho += (double)ri * (double)zi;
            rr += (double)ri * (double)ri;
        }
        block_sum2<kCgThreads>(bb, rho, red);
        block_sum2<kCgThreads>(rr, bad, red);
        const double nb = sqrt(bb);
        const double tol = fmax(a.rtol * nb, a.atol);
        int st = kActive, k = 0;
        double relres = 0.0;
        if (nb == 0.0) st = SLA_CONVERGED;
        else if (!isfinite(nb)) st = SLA_NONFINITE;
        else if (a.precond && bad > 0.0) { st = SLA_BREAKDOWN; relres = sqrt(rr) / nb; }
        else if (!a.fixed && sqrt(rr) <= tol) { st = SLA_CONVERGED; relres = sqrt(rr) / nb; }
        else if (rr == 0.0) st = SLA_CONVERGED;
        if (nb == 0.0)
            for (int i = tid; i < n; i += kCgThreads) xs[i] = T(0);
        __syncthreads();
        while (st == kActive) {
            double sg = 0.0;
            for (int i = sub; i < n; i += NSUB) {
                const T qi = spmv_row(ps, i);
                if (lane == 0) {
                    qs[i] = qi;
                    sg += (double)ps[i] * (double)qi;
                }
            }
            const double sigma = block_sum<kCgThreads>(sg, red);
            if (!isfinite(sigma) || !(sigma > 0.0)) {
                st = isfinite(sigma) ? SLA_BREAKDOWN : SLA_NONFINITE;
                relres = sqrt(rr) / nb;
                break;
            }
            const T al = (T)(rho / sigma);
            double lrho = 0.0, lrr = 0.0;
            for (int i = tid; i < n; i += kCgThreads) {
                xs[i] = xs[i] + al * ps[i];
                const T ri = rs[i] - al * qs[i];
                rs[i] = ri;
                const T zi = ds[i] * ri;
                lrho += (double)ri * (double)zi;
                lrr += (double)ri * (double)ri;
            }
            ++k;
            block_sum2<kCgThreads>(lrho, lrr, red);
            rr = lrr;
            relres = sqrt(rr) / nb;
            if (!isfinite(rr)) { st = SLA_NONFINITE; break; }
            if (!a.fixed && sqrt(rr) <= tol) { st = SLA_CONVERGED; break; }
            if (rr == 0.0) { st = SLA_CONVERGED; break; }
            if (k >= a.limit) { st = a.fixed ? SLA_FIXED_DONE : SLA_NOT_CONVERGED; break; }
            const T bt = (T)(lrho / rho);
            rho = lrho;
            for (int i = tid; i < n; i += kCgThreads) ps[i] = ds[i] * rs[i] + bt * ps[i];
            __syncthreads();
        }
        __syncthreads();
        for (int i = tid; i < n; i += kCgThreads) xg[i] = xs[i];
        if (tid == 0) {
            if (a.out_status) a.out_status[s] = st;
            if (a.out_iters) a.out_iters[s] = k;
            if (a.out_relres) a.out_relres[s] = relres;
        }
    }
}

// ------------------------------------------- interleaved batch kernel ----
// The persistent solver for a batch of BW systems sharing a pattern, with the
// values laid out [entry][system] (the sliced layout's slots, BW values each)
// and every vector [row][system]: one column-index load and one gather address
// serve all BW systems, and BW values move in one vector load.  Rows are
// split into tiles shared by the BW systems, at most one per block.  Each
// system keeps its own scalars, stop test and iteration count; every block
// takes the same per-system decisions from the tile partials, and a system
// that has stopped is left untouched until all have.  The phases and the
// arithmetic per system are those of cg_grid_kernel.
template <typename T, int BW>
struct VecLoad {
    // BW consecutive values starting at a multiple of BW elements
    static __device__ __forceinline__ void ld(const T *p, T (&v)[BW]) {
        constexpr int bytes = BW * (int)sizeof(T);
        if constexpr (bytes % 16 == 0) {
#pragma unroll
            for (int c = 0; c < bytes / 16; ++c) {
                const float4 u = *reinterpret_cast<const float4 *>(reinterpret_cast<const char *>(p) + 16 * c);
                memcpy(reinterpret_cast<char *>(v) + 16 * c, &u, 16);
            }
        } else if constexpr (bytes == 8) {
            const float2 u = *reinterpret_cast<const float2 *>(p);
            memcpy(v, &u, 8);
        } else {
#pragma unroll
            for (int s = 0; s < BW; ++s) v[s] = p[s];
        }
    }
    static __device__ __forceinline__ void st(T *p, const T (&v)[BW]) {
#pragma unroll
        for (int s = 0; s < BW; ++s) p[s] = v[s];
    }
};

template <typename T, int BW>
__device__ __forceinline__ void il_row(const int32_t *__restrict__ sptr, const int32_t *__restrict__ cols,
                                       const T *__restrict__ sv, const T *v, int i, T (&q)[BW],
                                       int ncols, int64_t nslots) {
    const int sl = i / kSellRows;
    const int b0 = __ldg(sptr + sl);
    const int w = (__ldg(sptr + sl + 1) - b0) / kSellRows;
    const int base = b0 + i % kSellRows;
#pragma unroll
    for (int s = 0; s < BW; ++s) q[s] = T(0);
    for (int k = 0; k < w; ++k) {
        const int t = SLA_IDX(base + k * kSellRows, nslots, kBndEntry);
        const int c = SLA_IDX(sell_load<true>(cols + t), ncols, kBndColumn);
        T av[BW], pv[BW];
        VecLoad<T, BW>::ld(sv + (int64_t)t * BW, av);
        VecLoad<T, BW>::ld(v + (int64_t)c * BW, pv);
#pragma unroll
        for (int s = 0; s < BW; ++s) q[s] += av[s] * pv[s];
    }
}

// il_row for slices all W wide with 16-bit columns (offsets d from row i,
// loaded ahead by the caller): same entries, order and rounding.
template <int W, typename T, int BW>
__device__ __forceinline__ void il_row_w(const T *__restrict__ sv, const T *v, const int (&d)[W], int i,
                                         T (&q)[BW], int ncols, int64_t nslots) {
    const int base = (i / kSellRows) * kSellRows * W + i % kSellRows;
#pragma unroll
    for (int s = 0; s < BW; ++s) q[s] = T(0);
#pragma unroll
    for (int k = 0; k < W; ++k) {
        const int t = SLA_IDX(base + k * kSellRows, nslots, kBndEntry);
        const int c = SLA_IDX(i + d[k], ncols, kBndColumn);
        T av[BW], pv[BW];
        VecLoad<T, BW>::ld(sv + (int64_t)t * BW, av);
        VecLoad<T, BW>::ld(v + (int64_t)c * BW, pv);
#pragma unroll
        for (int s = 0; s < BW; ++s) q[s] += av[s] * pv[s];
    }
}

// Phase A of the interleaved solver over a tile whose slices are all W wide
// with 16-bit columns: the next row's offsets load while this row gathers.
template <int W, int NT, typename T, int BW>
__device__ __forceinline__ void il_tile_w(const CgArgs<T> &a, const T *sv, const T *p, T *q, int r0, int r1,
                                          double (&acc)[BW]) {
    int i = r0 + threadIdx.x;
    if (i >= r1) return;
    int dn[W];
    sell_d16_fetch<W, 1>(a.sell_d16, i, a.sell_nnz, dn);
    for (; i < r1; i += NT) {
        int d[W];
#pragma unroll
        for (int k = 0; k < W; ++k) d[k] = dn[k];
        if (i + NT < r1) sell_d16_fetch<W, 1>(a.sell_d16, i + NT, a.sell_nnz, dn);
        T qv[BW], pv[BW];
        il_row_w<W>(sv, p, d, i, qv, a.n, a.sell_nnz);
        VecLoad<T, BW>::ld(p + (int64_t)i * BW, pv);
        VecLoad<T, BW>::st(q + (int64_t)i * BW, qv);
#pragma unroll
        for (int s = 0; s < BW; ++s) acc[s] += (double)pv[s] * (double)qv[s];
    }
}

template <typename T, int BW>
__global__ void __launch_bounds__(kCgThreads, 2)
cg_grid_il_kernel(CgArgs<T> a, T *xi, const T *bi, double *part, int tile_rows, int ntiles) {
    constexpr int NT = kCgThreads;
    __shared__ double red[4 * BW * 33];
    __shared__ double s_rho[BW], s_nb[BW], s_rr[BW], s_alpha[BW];
    __shared__ int s_state[BW], s_iters[BW];
    __shared__ int flag;
    const int tid = threadIdx.x;
    const int n = a.n;
    const int tile = blockIdx.x;
    const bool has_tile = tile < ntiles;
    const int r0 = tile * tile_rows, r1 = has_tile ? min(n, r0 + tile_rows) : r0;
    // partial of quantity qn for system s: part[(qn * BW + s) * ntiles + tile]
    auto P = [&](int qn, int s) { return part + (int64_t)(qn * BW + s) * ntiles; };
    const T *sv = a.sell_vals;
    T *r = a.r, *p = a.p, *q = a.q, *d = a.d;
    unsigned target = 0;
    auto give_up_il = [&]() {
        if (tid == 0)
            for (int s = 0; s < BW; ++s)
                if (s_state[s] == kActive && a.out_status) a.out_status[s] = SLA_TIMED_OUT;
    };
    if (tid < BW) s_state[tid] = kActive;

    // ---- init: r = b - A x0 (or b), M^-1, p = z; partials of b.b, r.z, r.r, bad diagonals
    {
        double acc[4 * BW];
#pragma unroll
        for (int j = 0; j < 4 * BW; ++j) acc[j] = 0.0;
        for (int i = r0 + tid; i < r1; i += NT) {
            T qx[BW];
            if (a.x0_given) il_row<T, BW>(a.sell_ptr, a.sell_cols, sv, xi, i, qx, a.n, a.sell_nnz);
            const int dp = a.precond ? SLA_IDX(__ldg(a.diagpos + i), a.nnz, kBndDiag) : -1;
#pragma unroll
            for (int s = 0; s < BW; ++s) {
                const int64_t o = (int64_t)i * BW + s;
                const T b_ = bi[o];
                const T ri = a.x0_given ? b_ - qx[s] : b_;
                T di = T(1);
                if (a.precond) {
                    const T dv = dp >= 0 ? __ldg(a.vals + (int64_t)s * a.nnz + dp) : T(0);
                    if (!(dv > T(0))) acc[3 * BW + s] += 1.0;
                    di = T(1) / dv;
                }
                const T zi = di * ri;
                if (!a.x0_given) xi[o] = T(0);
                r[o] = ri;
                d[o] = di;
                p[o] = zi;
                acc[s] += (double)b_ * (double)b_;
                acc[BW + s] += (double)ri * (double)zi;
                acc[2 * BW + s] += (double)ri * (double)ri;
            }
        }
        block_sums<NT, 4 * BW>(acc, red);
        if (tid == 0 && has_tile)
            for (int j = 0; j < 4 * BW; ++j) P(j / BW, j % BW)[tile] = acc[j];
    }
    if (!grid_sync(a.sync, target, a.timeout_ns, &flag)) { give_up_il(); return; }
    {
        const double *arr[4 * BW];
        for (int j = 0; j < 4 * BW; ++j) arr[j] = P(j / BW, j % BW);
        double sum[4 * BW];
        system_sums_dyn<NT, 4 * BW>(arr, ntiles, sum, red);
        if (tid == 0) {
            for (int s = 0; s < BW; ++s) {
                const double nb = sqrt(sum[s]), rho0 = sum[BW + s], rr = sum[2 * BW + s];
                const double tol = fmax(a.rtol * nb, a.atol);
                int st = kActive;
                double relres = 0.0;
                if (nb == 0.0) st = SLA_CONVERGED;
                else if (!isfinite(nb)) st = SLA_NONFINITE;
                else if (a.precond && sum[3 * BW + s] > 0.0) { st = SLA_BREAKDOWN; relres = sqrt(rr) / nb; }
                else if (!a.fixed && sqrt(rr) <= tol) { st = SLA_CONVERGED; relres = sqrt(rr) / nb; }
                else if (rr == 0.0) st = SLA_CONVERGED;
                s_state[s] = st;
                s_rho[s] = rho0;
                s_nb[s] = nb;
                s_rr[s] = rr;
                s_iters[s] = 0;
                if (st != kActive && blockIdx.x == 0) finalize(a, s, st, 0, relres, false);
            }
        }
        __syncthreads();
        // systems with b = 0 report x = 0
        for (int s = 0; s < BW; ++s)
            if (s_nb[s] == 0.0)
                for (int i = r0 + tid; i < r1; i += NT) xi[(int64_t)i * BW + s] = T(0);
    }
    auto any_active = [&]() {
        bool m = false;
        for (int s = 0; s < BW; ++s) m |= s_state[s] == kActive;
        return m;
    };
    while (any_active()) {
        bool act[BW];
#pragma unroll
        for (int s = 0; s < BW; ++s) act[s] = s_state[s] == kActive;
        // ---- phase A: q = A p for all systems, partials of p.q
        {
            double acc[BW];
#pragma unroll
            for (int s = 0; s < BW; ++s) acc[s] = 0.0;
            if (a.sell_d16 && a.sell_w == 7 && a.sell_pipe) {
                il_tile_w<7, NT>(a, sv, p, q, r0, r1, acc);
            } else if (a.sell_d16 && a.sell_w == 5 && a.sell_pipe) {
                il_tile_w<5, NT>(a, sv, p, q, r0, r1, acc);
            } else {
                for (int i = r0 + tid; i < r1; i += NT) {
                    T qv[BW], pv[BW];
                    il_row<T, BW>(a.sell_ptr, a.sell_cols, sv, p, i, qv, a.n, a.sell_nnz);
                    VecLoad<T, BW>::ld(p + (int64_t)i * BW, pv);
                    VecLoad<T, BW>::st(q + (int64_t)i * BW, qv);
#pragma unroll
                    for (int s = 0; s < BW; ++s) acc[s] += (double)pv[s] * (double)qv[s];
                }
            }
            block_sums<NT, BW>(acc, red);
            if (tid == 0 && has_tile)
                for (int s = 0; s < BW; ++s) P(0, s)[tile] = acc[s];
        }
        if (!grid_sync(a.sync, target, a.timeout_ns, &flag)) { give_up_il(); return; }
        // ---- phase B: alpha per system; r -= alpha q; partials of r.z and r.r
        {
            const double *arr[BW];
            for (int s = 0; s < BW; ++s) arr[s] = P(0, s);
            double sg[BW];
            system_sums_dyn<NT, BW>(arr, ntiles, sg, red);
            if (tid == 0) {
                for (int s = 0; s < BW; ++s) {
                    if (!act[s]) continue;
                    const double sigma = sg[s];
                    if (!isfinite(sigma) || !(sigma > 0.0)) {
                        const int st = isfinite(sigma) ? SLA_BREAKDOWN : SLA_NONFINITE;
                        s_state[s] = st;
                        if (blockIdx.x == 0) finalize(a, s, st, s_iters[s], sqrt(s_rr[s]) / s_nb[s], false);
                    } else {
                        s_alpha[s] = s_rho[s] / sigma;
                        s_iters[s] += 1;
                    }
                }
            }
            __syncthreads();
#pragma unroll
            for (int s = 0; s < BW; ++s) act[s] = s_state[s] == kActive;
            T al[BW];
#pragma unroll
            for (int s = 0; s < BW; ++s) al[s] = (T)s_alpha[s];
            double acc[2 * BW];
#pragma unroll
            for (int j = 0; j < 2 * BW; ++j) acc[j] = 0.0;
            for (int i = r0 + tid; i < r1; i += NT) {
                T rv[BW], qv[BW], dv[BW];
                VecLoad<T, BW>::ld(r + (int64_t)i * BW, rv);
                VecLoad<T, BW>::ld(q + (int64_t)i * BW, qv);
                VecLoad<T, BW>::ld(d + (int64_t)i * BW, dv);
#pragma unroll
                for (int s = 0; s < BW; ++s) {
                    if (!act[s]) continue;
                    const T ri = rv[s] - al[s] * qv[s];
                    rv[s] = ri;
                    const T zi = dv[s] * ri;
                    acc[s] += (double)ri * (double)zi;
                    acc[BW + s] += (double)ri * (double)ri;
                }
                VecLoad<T, BW>::st(r + (int64_t)i * BW, rv);
            }
            block_sums<NT, 2 * BW>(acc, red);
            if (tid == 0 && has_tile)
                for (int j = 0; j < 2 * BW; ++j) P(1 + j / BW, j % BW)[tile] = acc[j];
        }
        if (!grid_sync(a.sync, target, a.timeout_ns, &flag)) { give_up_il(); return; }
        // ---- phase C: stop tests; x += alpha p; beta; p = z + beta p
        {
            const double *arr[2 * BW];
            for (int j = 0; j < 2 * BW; ++j) arr[j] = P(1 + j / BW, j % BW);
            double sum[2 * BW];
            system_sums_dyn<NT, 2 * BW>(arr, ntiles, sum, red);
            __shared__ int s_go[BW];
            __shared__ double s_beta[BW];
            if (tid == 0) {
                for (int s = 0; s < BW; ++s) {
                    s_go[s] = 0;
                    if (!act[s]) continue;
                    const double rho_new = sum[s], rr = sum[BW + s];
                    const double nb = s_nb[s];
                    const double tol = fmax(a.rtol * nb, a.atol);
                    const int k = s_iters[s];
                    int st = kActive;
                    if (!isfinite(rr)) st = SLA_NONFINITE;
                    else if (!a.fixed && sqrt(rr) <= tol) st = SLA_CONVERGED;
                    else if (rr == 0.0) st = SLA_CONVERGED;
                    else if (k >= a.limit) st = a.fixed ? SLA_FIXED_DONE : SLA_NOT_CONVERGED;
                    s_beta[s] = rho_new / s_rho[s];
                    s_rr[s] = rr;
                    if (st == kActive) {
                        s_go[s] = 1;
                        s_rho[s] = rho_new;
                    } else {
                        s_state[s] = st;
                        if (blockIdx.x == 0) finalize(a, s, st, k, sqrt(rr) / nb, false);
                    }
                }
            }
            __syncthreads();
            T al[BW], bt[BW];
            bool go[BW];
#pragma unroll
            for (int s = 0; s < BW; ++s) {
                al[s] = (T)s_alpha[s];
                bt[s] = (T)s_beta[s];
                go[s] = s_go[s] != 0;
            }
            for (int i = r0 + tid; i < r1; i += NT) {
                T xv[BW], pv[BW], rv[BW], dv[BW];
                VecLoad<T, BW>::ld(xi + (int64_t)i * BW, xv);
                VecLoad<T, BW>::ld(p + (int64_t)i * BW, pv);
                VecLoad<T, BW>::ld(r + (int64_t)i * BW, rv);
                VecLoad<T, BW>::ld(d + (int64_t)i * BW, dv);
#pragma unroll
                for (int s = 0; s < BW; ++s) {
                    if (!act[s]) continue;
                    const T pi = pv[s];
                    xv[s] = xv[s] + al[s] * pi;
                    if (go[s]) pv[s] = dv[s] * rv[s] + bt[s] * pi;
                }
                VecLoad<T, BW>::st(xi + (int64_t)i * BW, xv);
                VecLoad<T, BW>::st(p + (int64_t)i * BW, pv);
            }
        }
        if (!grid_sync(a.sync, target, a.timeout_ns, &flag)) { give_up_il(); return; }
    }
}

// The sliced layout's value-and-column records of every system.
template <typename T>
__global__ void sell_pack_kernel(int64_t sell_nnz, int64_t nnz, int B, const int32_t *__restrict__ map,
                                 const int32_t *__restrict__ cols, const T *__restrict__ vals,
                                 SellRec<T> *__restrict__ out) {
    const int64_t slot = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (slot >= sell_nnz) return;
    const int t = map[slot];
    const int c = cols[slot];
    for (int b = 0; b < B; ++b) {
        SellRec<T> r{};
        r.v = t >= 0 ? vals[(int64_t)b * nnz + t] : T(0);
        r.c = c;
        out[(int64_t)b * sell_nnz + slot] = r;
    }
}

// Batch-major [B][n] <-> interleaved [n][B].
template <typename T>
__global__ void interleave_kernel(int64_t n, int B, const T *__restrict__ in, T *__restrict__ out) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= n * B) return;
    const int64_t i = g / B;
    const int s = (int)(g % B);
    out[g] = in[(int64_t)s * n + i];
}
template <typename T>
__global__ void deinterleave_kernel(int64_t n, int B, const T *__restrict__ in, T *__restrict__ out) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= n * B) return;
    const int s = (int)(g / n);
    const int64_t i = g % n;
    out[g] = in[i * B + s];
}
// The sliced layout's values, slot-major: out[slot * B + s] = vals[s][map[slot]].
template <typename T>
__global__ void sell_values_il_kernel(int64_t sell_nnz, int64_t nnz, int B, const int32_t *__restrict__ map,
                                      const T *__restrict__ vals, T *__restrict__ out) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= sell_nnz * B) return;
    const int64_t slot = g / B;
    const int s = (int)(g % B);
    const int t = map[slot];
    out[g] = t >= 0 ? vals[(int64_t)s * nnz + t] : T(0);
}

// ---------------------------------------------------- segment kernel ----
// A list of independent systems with their own patterns, stored as one
// block-diagonal CSR whose item s owns rows (and columns) [seg[s], seg[s+1]).
// Each block claims items from an atomic counter, largest first (order[]),
// and runs the whole PCG of an item itself, exactly as cg_block_kernel does for
// one system; an item's vectors live in shared memory when it has at most
// smem_rows rows, else in the workspace vectors at the item's offset.  An item
// is always solved by one block, so results do not depend on the schedule.
template <typename T, int LANES>
__global__ void __launch_bounds__(kCgThreads)
cg_segment_kernel(CgArgs<T> a, const int32_t *__restrict__ seg, const int32_t *__restrict__ order,
                  int n_items, int smem_rows, unsigned *work) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ double red[72];
    __shared__ int s_next;
    constexpr int NSUB = kCgThreads / LANES;
    const int tid = threadIdx.x, sub = tid / LANES, lane = tid % LANES;
    T *sm = reinterpret_cast<T *>(smem_raw);
    while (true) {
        __syncthreads();
        if (tid == 0) s_next = (int)atomicAdd(work, 1u);
        __syncthreads();
        const int q = s_next;
        if (q >= n_items) break;
        const int s = __ldg(order + q);
        const int o = __ldg(seg + s), m = __ldg(seg + s + 1) - o;
        const bool on_chip = m <= smem_rows;
        T *xs = on_chip ? sm : a.x + o;
        T *rs = on_chip ? sm + m : a.r + o;
        T *ps = on_chip ? sm + 2 * m : a.p + o;
        T *qs = on_chip ? sm + 3 * m : a.q + o;
        T *ds = on_chip ? sm + 4 * m : a.d + o;
        const T *bs = a.b + o;
        T *xg = a.x + o;
        // row li of the item is global row o + li; its columns are global too
        auto spmv_row = [&](const T *v, int li) -> T {
            const int t0 = __ldg(a.rowptr + o + li), t1 = __ldg(a.rowptr + o + li + 1);
            T acc = T(0);
            for (int t = t0 + lane; t < t1; t += LANES) {
                const int tt = SLA_IDX(t, a.nnz, kBndEntry);
                acc += __ldg(a.vals + tt) * v[SLA_IDX(__ldg(a.colind + tt) - o, m, kBndLocal)];
            }
            if constexpr (LANES > 1) {
                const unsigned mk = subwarp_mask<LANES>();
#pragma unroll
                for (int off = LANES / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(mk, acc, off, LANES);
            }
            return acc;
        };
        if (a.x0_given) {
            if (on_chip) {
                for (int i = tid; i < m; i += kCgThreads) xs[i] = xg[i];
                __syncthreads();
            }
            for (int i = sub; i < m; i += NSUB) {
                const T v = spmv_row(xs, i);
                if (lane == 0) qs[i] = v;
            }
            __syncthreads();
        }
        double bb = 0.0, rho = 0.0, rr = 0.0, bad = 0.0;
        for (int i = tid; i < m; i += kCgThreads) {
            const T bi = bs[i];
            T ri;
            if (a.x0_given) {
                ri = bi - qs[i];
            } else {
                ri = bi;
                xs[i] = T(0);
            }
            T di = T(1);
            if (a.precond) {
                const int dp = __ldg(a.diagpos + o + i);
                const T dv = dp >= 0 ? __ldg(a.vals + SLA_IDX(dp, a.nnz, kBndDiag)) : T(0);
                if (!(dv > T(0))) bad += 1.0;
                di = T(1) / dv;
            }
            const T zi = di * ri;
            rs[i] = ri;
            ps[i] = zi;
            ds[i] = di;
            bb += (double)bi * (double)bi;
            rho += (double)ri * (double)zi;
            rr += (double)ri * (double)ri;
        }
        block_sum2<kCgThreads>(bb, rho, red);
        block_sum2<kCgThreads>(rr, bad, red);
        const double nb = sqrt(bb);
        const double tol = fmax(a.rtol * nb, a.atol);
        int st = kActive, k = 0;
        double relres = 0.0;
        if (nb == 0.0) st = SLA_CONVERGED;
        else if (!isfinite(nb)) st = SLA_NONFINITE;
        else if (a.precond && bad > 0.0) { st = SLA_BREAKDOWN; relres = sqrt(rr) / nb; }
        else if (!a.fixed && sqrt(rr) <= tol) { st = SLA_CONVERGED; relres = sqrt(rr) / nb; }
        else if (rr == 0.0) st = SLA_CONVERGED;
        if (nb == 0.0)
            for (int i = tid; i < m; i += kCgThreads) xs[i] = T(0);
        __syncthreads();
        while (st == kActive) {
            double sg = 0.0;
            for (int i = sub; i < m; i += NSUB) {
                const T qi = spmv_row(ps, i);
                if (lane == 0) {
                    qs[i] = qi;
                    sg += (double)ps[i] * (double)qi;
                }
            }
            const double sigma = block_sum<kCgThreads>(sg, red);
            if (!isfinite(sigma) || !(sigma > 0.0)) {
                st = isfinite(sigma) ? SLA_BREAKDOWN : SLA_NONFINITE;
                relres = sqrt(rr) / nb;
                break;
            }
            const T al = (T)(rho / sigma);
            double lrho = 0.0, lrr = 0.0;
            for (int i = tid; i < m; i += kCgThreads) {
                xs[i] = xs[i] + al * ps[i];
                const T ri = rs[i] - al * qs[i];
                rs[i] = ri;
                const T zi = ds[i] * ri;
                lrho += (double)ri * (double)zi;
                lrr += (double)ri * (double)ri;
            }
            ++k;
            block_sum2<kCgThreads>(lrho, lrr, red);
            rr = lrr;
            relres = sqrt(rr) / nb;
            if (!isfinite(rr)) { st = SLA_NONFINITE; break; }
            if (!a.fixed && sqrt(rr) <= tol) { st = SLA_CONVERGED; break; }
            if (rr == 0.0) { st = SLA_CONVERGED; break; }
            if (k >= a.limit) { st = a.fixed ? SLA_FIXED_DONE : SLA_NOT_CONVERGED; break; }
            const T bt = (T)(lrho / rho);
            rho = lrho;
            for (int i = tid; i < m; i += kCgThreads) ps[i] = ds[i] * rs[i] + bt * ps[i];
            __syncthreads();
        }
        __syncthreads();
        if (on_chip)
            for (int i = tid; i < m; i += kCgThreads) xg[i] = xs[i];
        if (tid == 0) {
            if (a.out_status) a.out_status[s] = st;
            if (a.out_iters) a.out_iters[s] = k;
            if (a.out_relres) a.out_relres[s] = relres;
        }
    }
}

// ---------------------------------------------------- cluster kernel ----
// One thread-block cluster per system (kClusterCTAs blocks): each block owns a
// contiguous run of rows and keeps its rows' matrix entries, x, r, M^-1, q and
// p in its own shared memory for the whole solve.  The SpMV reads other
// blocks' p through distributed shared memory; cluster-wide sums go through
// per-block partial slots read over DSMEM in rank order, so every block takes
// the same decisions.  Waits inside the loop are a software barrier on a
// counter in rank 0's shared memory, bounded like grid_sync; every exit path
// ends in one hardware cluster barrier so that no block leaves while another
// may still read its shared memory.
constexpr int kClusterCTAs = 8;
constexpr int kClusterThreads = 512;

__device__ __forceinline__ void red_release_cluster(unsigned *p, unsigned v) {
    asm volatile("red.release.cluster.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire_cluster(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.cluster.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ bool cluster_sync_bounded(unsigned *count0, unsigned *err0, unsigned &target,
                                                     long long timeout_ns, int *flag) {
    __syncthreads();
    target += kClusterCTAs;
    if (threadIdx.x == 0) {
        int ok = 1;
        // the arrive is a release and the poll an acquire at cluster scope; the
        // block barriers around them order the other threads' shared-memory work
        red_release_cluster(count0, 1u);
        const unsigned long long t0 = global_timer_ns();
        unsigned spins = 0;
        while ((int)(ld_acquire_cluster(count0) - target) < 0) {
            if ((spins++ & 7u) == 0) {
                if (ld_acquire_cluster(err0) != 0) { ok = 0; break; }
                if ((long long)(global_timer_ns() - t0) > timeout_ns) {
                    atomicExch(err0, 1u);
                    ok = 0;
                    break;
                }
            }
        }
        if (ok && ld_acquire_cluster(err0) != 0) ok = 0;
        *flag = ok;
    }
    __syncthreads();
    return *flag != 0;
}

// p_k = z_{k-1} + beta p_{k-1} with z = M^-1 r, computed the same way (one
// rounded product, one fused multiply-add) by the owner and by every gatherer.
template <typename T>
__device__ __forceinline__ T direction(T d, T r, T p, T beta) {
    if constexpr (sizeof(T) == 8) return __fma_rn(beta, p, __dmul_rn(d, r));
    else return __fmaf_rn(beta, p, __fmul_rn(d, r));
}

// Two cluster-wide synchronisations per iteration: the SpMV of iteration k
// forms each gathered p_k(j) from the owner's M^-1, r and p_{k-1} (double
// buffered) instead of waiting for the owner to write p_k; x and r are updated
// together once alpha is known.
template <typename T, int NT>
__global__ void __launch_bounds__(NT)
cg_cluster_kernel(CgArgs<T> a, int rows_cta, int nnz_cap) {
    namespace cgs = cooperative_groups;
    constexpr int CS = kClusterCTAs;
    cgs::cluster_group cl = cgs::this_cluster();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ double red[4 * 33];
    __shared__ double cpart[2][4];
    __shared__ unsigned cbar_count, cbar_err;
    __shared__ int flag;
    __shared__ double bc[4];
    __shared__ T *pb[2][CS], *rb[CS], *db[CS];
    const int rank = (int)cl.block_rank();
    const int sys = blockIdx.x / CS;
    const int tid = threadIdx.x;
    const int n = a.n;
    T *p0_s = reinterpret_cast<T *>(smem_raw);
    T *p1_s = p0_s + rows_cta, *x_s = p1_s + rows_cta, *r_s = x_s + rows_cta, *d_s = r_s + rows_cta;
    T *q_s = d_s + rows_cta;
    T *v_s = q_s + rows_cta;
    int32_t *c_s = reinterpret_cast<int32_t *>(v_s + nnz_cap);
    int32_t *rp_s = c_s + nnz_cap;

    if (tid == 0) { cbar_count = 0; cbar_err = 0; }
    if (tid < CS) {
        pb[0][tid] = cl.map_shared_rank(p0_s, tid);
        pb[1][tid] = cl.map_shared_rank(p1_s, tid);
        rb[tid] = cl.map_shared_rank(r_s, tid);
        db[tid] = cl.map_shared_rank(d_s, tid);
    }
    unsigned *count0 = cl.map_shared_rank(&cbar_count, 0);
    unsigned *err0 = cl.map_shared_rank(&cbar_err, 0);
    unsigned target = 0;
    int exch = 0;
    cl.sync();   // every block's counters and pointers are set before first use

    const int r0 = rank * rows_cta, r1 = min(n, r0 + rows_cta);
    const int m = r1 > r0 ? r1 - r0 : 0;
    const T *vs = a.vals + (int64_t)sys * a.nnz;
    const T *bs = a.b + (int64_t)sys * n;
    T *xg = a.x + (int64_t)sys * n;
    const int t0 = m > 0 ? __ldg(a.rowptr + r0) : 0, t1 = m > 0 ? __ldg(a.rowptr + r1) : 0;
    for (int i = tid; i <= m; i += NT) rp_s[i] = m > 0 ? __ldg(a.rowptr + r0 + i) - t0 : 0;
    for (int t = t0 + tid; t < t1; t += NT) {
        const int lt = SLA_IDX(t - t0, nnz_cap, kBndLocal);
        c_s[lt] = __ldg(a.colind + SLA_IDX(t, a.nnz, kBndEntry));
        v_s[lt] = __ldg(vs + SLA_IDX(t, a.nnz, kBndEntry));
    }
    __syncthreads();

    // cluster-wide sums of nv values: block sums -> this block's slot -> barrier
    // -> every block adds the CS slots in rank order
    auto cluster_sums = [&](double *v, int nv) -> bool {
        double tmp[4] = {v[0], nv > 1 ? v[1] : 0.0, nv > 2 ? v[2] : 0.0, nv > 3 ? v[3] : 0.0};
        block_sums<NT, 4>(tmp, red);
        const int slot = exch & 1;
        if (tid == 0)
            for (int k = 0; k < 4; ++k) cpart[slot][k] = tmp[k];
        ++exch;
        if (!cluster_sync_bounded(count0, err0, target, a.timeout_ns, &flag)) return false;
        if (tid < 32) {
            for (int k = 0; k < nv; ++k) {
                double x = tid < CS ? *cl.map_shared_rank(&cpart[slot][k], tid) : 0.0;
                x = warp_sum(x);
                if (tid == 0) bc[k] = x;
            }
        }
        __syncthreads();
        for (int k = 0; k < nv; ++k) v[k] = bc[k];
        __syncthreads();
        return true;
    };

    int st = kActive, k = 0;
    double relres = 0.0, nb = 0.0, tol = 0.0, rho = 0.0, rr = 0.0;
    bool alive = true;
    {   // r = b - A x0 (or b), M^-1; p_0 = 0 so that p_1 = z_0
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        for (int li = tid; li < m; li += NT) {
            const int i = r0 + li;
            const T bi = bs[i];
            T ri = bi, xi = T(0), dv = T(0);
            T ax = T(0);
            for (int t = rp_s[li]; t < rp_s[li + 1]; ++t) {
                if (c_s[t] == i) dv = v_s[t];
                if (a.x0_given) ax += v_s[t] * xg[SLA_IDX(c_s[t], n, kBndColumn)];
            }
            if (a.x0_given) {
                xi = xg[i];
                ri = bi - ax;
            }
            T di = T(1);
            if (a.precond) {
                if (!(dv > T(0))) acc[3] += 1.0;
                di = T(1) / dv;
            }
            const T zi = di * ri;
            x_s[li] = xi;
            r_s[li] = ri;
            d_s[li] = di;
            p0_s[li] = T(0);
            acc[0] += (double)bi * (double)bi;
            acc[1] += (double)ri * (double)zi;
            acc[2] += (double)ri * (double)ri;
        }
        alive = cluster_sums(acc, 4);
        nb = sqrt(acc[0]);
        rho = acc[1];
        rr = acc[2];
        tol = fmax(a.rtol * nb, a.atol);
        if (nb == 0.0) st = SLA_CONVERGED;
        else if (!isfinite(nb)) st = SLA_NONFINITE;
        else if (a.precond && acc[3] > 0.0) { st = SLA_BREAKDOWN; relres = sqrt(rr) / nb; }
        else if (!a.fixed && sqrt(rr) <= tol) { st = SLA_CONVERGED; relres = sqrt(rr) / nb; }
        else if (rr == 0.0) st = SLA_CONVERGED;
        if (nb == 0.0)
            for (int li = tid; li < m; li += NT) x_s[li] = T(0);
    }
    T bt = T(0);   // beta_{k-1}; 0 before the first step
    while (alive && st == kActive) {
        // SpMV of iteration k+1 with p_{k+1} = z_k + beta_k p_k formed on the fly
        const int cur = (k + 1) & 1, prev = k & 1;
        T *pcur = cur ? p1_s : p0_s;
        const T *pprev = prev ? p1_s : p0_s;
        double sg[1] = {0.0};
        for (int li = tid; li < m; li += NT) {
            T qi = T(0);
            for (int t = rp_s[li]; t < rp_s[li + 1]; ++t) {
                const int j = SLA_IDX(c_s[t], n, kBndColumn);
                const int o = SLA_IDX(j / rows_cta, CS, kBndLocal), lj = j - o * rows_cta;
                qi += v_s[t] * direction(db[o][lj], rb[o][lj], pb[prev][o][lj], bt);
            }
            q_s[li] = qi;
            const T pi = direction(d_s[li], r_s[li], pprev[li], bt);
            pcur[li] = pi;
            sg[0] += (double)pi * (double)qi;
        }
        if (!(alive = cluster_sums(sg, 1))) break;
        const double sigma = sg[0];
        if (!isfinite(sigma) || !(sigma > 0.0)) {
            st = isfinite(sigma) ? SLA_BREAKDOWN : SLA_NONFINITE;
            relres = sqrt(rr) / nb;
            break;
        }
        const T al = (T)(rho / sigma);
        ++k;
        double acc[2] = {0.0, 0.0};
        for (int li = tid; li < m; li += NT) {
            x_s[li] = x_s[li] + al * pcur[li];
            const T ri = r_s[li] - al * q_s[li];
            r_s[li] = ri;
            const T zi = d_s[li] * ri;
            acc[0] += (double)ri * (double)zi;
            acc[1] += (double)ri * (double)ri;
        }
        if (!(alive = cluster_sums(acc, 2))) break;
        const double rho_new = acc[0];
        rr = acc[1];
        relres = sqrt(rr) / nb;
        if (!isfinite(rr)) st = SLA_NONFINITE;
        else if (!a.fixed && sqrt(rr) <= tol) st = SLA_CONVERGED;
        else if (rr == 0.0) st = SLA_CONVERGED;
        else if (k >= a.limit) st = a.fixed ? SLA_FIXED_DONE : SLA_NOT_CONVERGED;
        bt = (T)(rho_new / rho);
        rho = rho_new;
    }
    if (alive)
        for (int li = tid; li < m; li += NT) xg[r0 + li] = x_s[li];
    if (rank == 0 && tid == 0) {
        const int out = alive ? st : SLA_TIMED_OUT;
        if (a.out_status) a.out_status[sys] = out;
        if (a.out_iters) a.out_iters[sys] = k;
        if (a.out_relres) a.out_relres[sys] = relres;
    }
    cl.sync();   // no block leaves while another may still read its shared memory
}

__global__ void info_fill_kernel(int B, int32_t *iters, double *relres, int32_t *status) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= B) return;
    if (iters) iters[s] = 0;
    if (relres) relres[s] = 0.0;
    if (status) status[s] = SLA_CONVERGED;
}

// ----------------------------------------------------------- host side ----
constexpr int kOnchipThreads = 1024;

template <typename T, int L>
static const void *grid_fn() {
    return reinterpret_cast<const void *>(&cg_grid_kernel<T, L, false, 1, kCgThreads, false>);
}
template <typename T>
static const void *grid_sell_fn() {
    return reinterpret_cast<const void *>(&cg_grid_kernel<T, 1, false, 1, kCgThreads, true>);
}
template <typename T, int RPT, bool SELL>
static const void *onchip_fn() {
    return reinterpret_cast<const void *>(&cg_grid_kernel<T, 1, true, RPT, kOnchipThreads, SELL>);
}
template <typename T, int RPT>
static const void *grid2_fn() {
    return reinterpret_cast<const void *>(&cg_grid2_kernel<T, RPT, kOnchipThreads>);
}
template <typename T, int L, bool MRES = false>
static const void *block_fn() { return reinterpret_cast<const void *>(&cg_block_kernel<T, L, MRES>); }

template <typename T>
static const void *cluster_fn() {
    return reinterpret_cast<const void *>(&cg_cluster_kernel<T, kClusterThreads>);
}

static const void *pick_block(sla_dtype dt, int lanes, bool mres) {
    const void *f = nullptr;
    with_lanes(lanes, [&](auto L) -> sla_status {
        constexpr int LN = decltype(L)::value;
        if (dt == SLA_F64) f = mres ? block_fn<double, LN, true>() : block_fn<double, LN, false>();
        else f = mres ? block_fn<float, LN, true>() : block_fn<float, LN, false>();
        return SLA_OK;
    });
    return f;
}

static const void *pick_fn(bool grid, sla_dtype dt, int lanes) {
    const void *f = nullptr;
    with_lanes(lanes, [&](auto L) -> sla_status {
        constexpr int LN = decltype(L)::value;
        if (dt == SLA_F64) f = grid ? grid_fn<double, LN>() : block_fn<double, LN>();
        else f = grid ? grid_fn<float, LN>() : block_fn<float, LN>();
        return SLA_OK;
    });
    return f;
}

static const void *pick_onchip(sla_dtype dt, int rpt, bool sell) {
    if (dt == SLA_F64) {
        if (rpt <= 4) return sell ? onchip_fn<double, 4, true>() : onchip_fn<double, 4, false>();
        return sell ? onchip_fn<double, 8, true>() : onchip_fn<double, 8, false>();
    }
    if (rpt <= 4) return sell ? onchip_fn<float, 4, true>() : onchip_fn<float, 4, false>();
    if (rpt <= 8) return sell ? onchip_fn<float, 8, true>() : onchip_fn<float, 8, false>();
    return sell ? onchip_fn<float, 16, true>() : onchip_fn<float, 16, false>();
}

static const void *pick_grid2(sla_dtype dt, int rpt) {
    if (dt == SLA_F64) return rpt <= 4 ? grid2_fn<double, 4>() : grid2_fn<double, 8>();
    if (rpt <= 4) return grid2_fn<float, 4>();
    return rpt <= 8 ? grid2_fn<float, 8>() : grid2_fn<float, 16>();
}

static const void *pick_il(sla_dtype dt, int B) {
    if (dt == SLA_F64)
        return B == 2 ? reinterpret_cast<const void *>(&cg_grid_il_kernel<double, 2>)
                      : reinterpret_cast<const void *>(&cg_grid_il_kernel<double, 4>);
    return B == 2 ? reinterpret_cast<const void *>(&cg_grid_il_kernel<float, 2>)
                  : reinterpret_cast<const void *>(&cg_grid_il_kernel<float, 4>);
}

static const void *pick_grid(const Csr *h, bool sell) {
    if (h->onchip) return pick_onchip(h->dtype, h->onchip_rpt, sell);
    if (sell) return h->dtype == SLA_F64 ? grid_sell_fn<double>() : grid_sell_fn<float>();
    return pick_fn(true, h->dtype, h->lanes);
}

// One dynamic shared-memory ceiling per kernel for every handle (static shared
// memory of these kernels stays below 8 KB), so no handle lowers another's.
static sla_status smem_ceiling(const void *f, int device) {
    int optin = 0;
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
    SLA_CHECK_CUDA(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - 8192));
    return SLA_OK;
}

// Tile layout: tiles never straddle systems, and B * ntiles <= blocks whenever
// B <= blocks, so that each block owns at most one tile in the common case.
static void layout(Csr *h, int blocks, int32_t *tile_rows, int32_t *ntiles) {
    const int n = h->n_rows, B = h->batch;
    int nt = blocks / B;
    if (nt < 1) nt = 1;
    int64_t tr = n > 0 ? ((int64_t)n + nt - 1) / nt : 1;
    if (tr > 32) tr = (tr + 31) / 32 * 32;
    *tile_rows = (int32_t)tr;
    *ntiles = n > 0 ? (int32_t)(((int64_t)n + tr - 1) / tr) : 1;
}

sla_status cg_configure(Csr *h) {
    const size_t ts = dtype_size(h->dtype);
    const int n = h->n_rows;
    int optin = 0;
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, h->device);
    h->block_smem = 5 * (size_t)n * ts;
    h->block_fits = n > 0 && h->block_smem + 2048 <= (size_t)optin;
    h->block_mres = false;
    h->block_grid = 4 * h->num_sms;
    if (h->block_fits) {
        // the same ceiling for every handle, so one handle never lowers another's
        SLA_CHECK_CUDA(cudaFuncSetAttribute(pick_fn(false, h->dtype, h->lanes),
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            optin - 2048));
        // the whole system (values, pattern, vectors) in shared memory when it fits
        const size_t mres = h->block_smem + (size_t)h->nnz * (ts + 4) + ((size_t)n + 1) * 4;
        const char *e = getenv("SLA_BLOCK_RESIDENT");
        if (mres + 2048 <= (size_t)optin && !(e && e[0] == '0')) {
            const void *f = pick_block(h->dtype, h->lanes, true);
            SLA_CHECK_CUDA(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                optin - 2048));
            int per_sm = 0;
            SLA_CHECK_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, f, kCgThreads, mres));
            // Only when the whole batch runs in one resident wave: with more systems
            // than resident blocks, more concurrent (non-resident) blocks win.
            if (per_sm >= 1 && h->batch <= per_sm * h->num_sms) {
                h->block_mres = true;
                h->block_smem = mres;
                h->block_grid = per_sm * h->num_sms;   // each block keeps its pattern copy
            }
        }
    }
    // On-chip variant: one 1024-thread block per SM, x, r, M^-1 of the block's
    // rows in shared memory, at most 16 rows a thread.
    h->onchip = false;
    const char *oc = getenv("SLA_GRID_ONCHIP");
    if (h->lanes == 1 && n > 0 && !(oc && oc[0] == '0')) {
        int32_t tr = 0, nt = 0;
        layout(h, h->num_sms, &tr, &nt);
        const int rpt = (tr + kOnchipThreads - 1) / kOnchipThreads;
        const size_t smem = 3 * (size_t)tr * ts;
        const int rpt_cap = h->dtype == SLA_F64 ? 8 : 16;   // beyond this the q registers spill
        if ((int64_t)h->batch * nt <= h->num_sms && rpt <= rpt_cap && smem + 16384 <= (size_t)optin) {
            for (int sv = 0; sv < 3; ++sv)
                SLA_CHECK_CUDA(cudaFuncSetAttribute(
                    sv < 2 ? pick_onchip(h->dtype, rpt, sv != 0) : pick_grid2(h->dtype, rpt),
                    cudaFuncAttributeMaxDynamicSharedMemorySize, optin - 16384));
            const void *f = pick_onchip(h->dtype, rpt, true);
            int per_sm = 0;
            SLA_CHECK_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, f, kOnchipThreads, smem));
            if (per_sm >= 1) {
                h->onchip = true;
                h->onchip_rpt = rpt;
                h->grid_smem = smem;
                h->grid_threads = kOnchipThreads;
                h->grid_blocks = h->num_sms;
                h->tile_rows = tr;
                h->ntiles = nt;
                // One system with one tile a block: the two-barrier solver (it
                // needs the sliced layout, decided after this).  It gathers two
                // vectors where the three-barrier one gathers one, so it is
                // taken only while both gathered tiles stay in L1 beside the
                // on-chip vectors (measured on a 10^6-row 2-D Poisson system:
                // +5% in fp32, where they fit; -35% in fp64, where they do not).
                const char *g2 = getenv("SLA_GRID2");
                int per_sm2 = 0, smem_sm = 0;
                SLA_CHECK_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                    &per_sm2, pick_grid2(h->dtype, rpt), kOnchipThreads, smem));
                cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, h->device);
                const bool l1_fits = smem + 2 * (size_t)tr * ts <= (size_t)smem_sm;
                h->grid2 = h->batch == 1 && nt <= h->num_sms && per_sm2 >= 1 &&
                           (l1_fits || (g2 && g2[0] == '2')) && !(g2 && g2[0] == '0');

            }
        }
    }
    if (!h->onchip) {
        int per_sm = 0;
        SLA_CHECK_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &per_sm, pick_fn(true, h->dtype, h->lanes), kCgThreads, 0));
        int want = 2;
        if (const char *e = getenv("SLA_GRID_BLOCKS_PER_SM")) want = atoi(e);
        if (want < 1) want = 1;
        per_sm = per_sm < want ? per_sm : want;
        if (per_sm < 1) {
            set_error("cg_configure: persistent kernel cannot be resident");
            return SLA_ERR_CUDA;
        }
        h->grid_blocks = per_sm * h->num_sms;
        h->grid_threads = kCgThreads;
        h->grid_smem = 0;
        layout(h, h->grid_blocks, &h->tile_rows, &h->ntiles);
        // fp32 batches of 2 or 4 systems: the interleaved solver (values
        // [entry][system]).  fp64 batches run batch-major, which measured
        // faster once rows load their column offsets a row ahead (4 x 128^3:
        // 14.3 k against 8.7 k system-iterations/s); SLA_INTERLEAVE=1 or 0
        // forces the choice.
        const char *ie = getenv("SLA_INTERLEAVE");
        const bool want_il = ie ? ie[0] == '1' : h->dtype == SLA_F32;
        h->il_blocks = 0;
        if ((h->batch == 2 || h->batch == 4) && n > 0 && want_il) {
            const void *f = pick_il(h->dtype, h->batch);
            int per_il = 0;
            SLA_CHECK_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_il, f, kCgThreads, 0));
            per_il = std::min(per_il, 2);
            if (per_il >= 1) h->il_blocks = per_il * h->num_sms;
        }
    }
    // Cluster solver: rows split over kClusterCTAs blocks on 32-row boundaries,
    // each block's matrix slice, vectors and p in its shared memory.
    h->cluster_fits = false;
    const char *ce = getenv("SLA_CLUSTER");
    if (n > 0 && n <= 65536 && !(ce && ce[0] == '0')) {
        int64_t rc = ((int64_t)n + kClusterCTAs - 1) / kClusterCTAs;
        rc = (rc + 31) / 32 * 32;
        std::vector<int32_t> rp((size_t)n + 1);
        SLA_CHECK_CUDA(cudaMemcpy(rp.data(), h->rowptr, rp.size() * sizeof(int32_t), cudaMemcpyDeviceToHost));
        int64_t cap = 0;
        for (int r = 0; r < kClusterCTAs; ++r) {
            const int64_t a0 = std::min<int64_t>(n, r * rc), a1 = std::min<int64_t>(n, (r + 1) * rc);
            cap = std::max<int64_t>(cap, (int64_t)rp[a1] - rp[a0]);
        }
        const size_t smem = 6 * (size_t)rc * ts + (size_t)cap * (ts + 4) + ((size_t)rc + 1) * 4;
        if (smem + 8192 <= (size_t)optin) {
            const void *f = h->dtype == SLA_F64 ? cluster_fn<double>() : cluster_fn<float>();
            sla_status st = smem_ceiling(f, h->device);
            if (st != SLA_OK) return st;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(kClusterCTAs);
            cfg.blockDim = dim3(kClusterThreads);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = kClusterCTAs;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int nclusters = 0;
            if (cudaOccupancyMaxActiveClusters(&nclusters, f, &cfg) == cudaSuccess && nclusters >= 1) {
                h->cluster_fits = true;
                h->cluster_rows = (int32_t)rc;
                h->cluster_nnz = (int32_t)std::max<int64_t>(cap, 1);
                h->cluster_smem = smem;
            }
            cudaGetLastError();
        }
    }
    return SLA_OK;
}

// Range of tiles whose rows a tile's columns reach (one system): per tile the
// smallest and largest column index over its entries, divided by tile_rows.
__global__ void tile_deps_kernel(int n, int tile_rows, const int32_t *__restrict__ rowptr,
                                 const int32_t *__restrict__ colind, int32_t *lo, int32_t *hi) {
    __shared__ int smin[32], smax[32];
    const int tt = blockIdx.x;
    const int r0 = tt * tile_rows, r1 = min(n, r0 + tile_rows);
    int cmin = INT_MAX, cmax = -1;
    for (int t = rowptr[r0] + threadIdx.x; t < rowptr[r1]; t += blockDim.x) {
        const int c = colind[t];
        cmin = min(cmin, c);
        cmax = max(cmax, c);
    }
    for (int o = 16; o > 0; o >>= 1) {
        cmin = min(cmin, __shfl_xor_sync(0xffffffffu, cmin, o));
        cmax = max(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
    }
    if ((threadIdx.x & 31) == 0) { smin[threadIdx.x >> 5] = cmin; smax[threadIdx.x >> 5] = cmax; }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) { cmin = min(cmin, smin[w]); cmax = max(cmax, smax[w]); }
        cmin = min(cmin, smin[0]);
        cmax = max(cmax, smax[0]);
        // a tile always depends on itself (its own p enters p.q)
        lo[tt] = cmax < 0 ? tt : min(tt, cmin / tile_rows);
        hi[tt] = cmax < 0 ? tt : max(tt, cmax / tile_rows);
    }
}

// Dependency ranges for p-ready flags (single-system handles whose tiles each
// reach at most 32 tiles); otherwise the solver keeps its third barrier.
sla_status cg_tile_deps(Csr *h, cudaStream_t s) {
    if (h->batch != 1 || h->n_rows == 0 || h->ntiles < h->grid_blocks) return SLA_OK;
    const char *e = getenv("SLA_TILE_FLAGS");
    if (e && e[0] == '0') return SLA_OK;
    SLA_CHECK_CUDA(cudaMalloc(&h->dep_lo, (size_t)h->ntiles * sizeof(int32_t)));
    SLA_CHECK_CUDA(cudaMalloc(&h->dep_hi, (size_t)h->ntiles * sizeof(int32_t)));
    tile_deps_kernel<<<h->ntiles, 256, 0, s>>>(h->n_rows, h->tile_rows, h->rowptr, h->colind,
                                                h->dep_lo, h->dep_hi);
    SLA_CHECK_LAUNCH();
    std::vector<int32_t> lo(h->ntiles), hi(h->ntiles);
    SLA_CHECK_CUDA(cudaMemcpyAsync(lo.data(), h->dep_lo, lo.size() * 4, cudaMemcpyDeviceToHost, s));
    SLA_CHECK_CUDA(cudaMemcpyAsync(hi.data(), h->dep_hi, hi.size() * 4, cudaMemcpyDeviceToHost, s));
    SLA_CHECK_CUDA(cudaStreamSynchronize(s));
    int span = 0;
    for (int t = 0; t < h->ntiles; ++t) span = std::max(span, hi[t] - lo[t] + 1);
    if (span > 32) {
        cudaFree(h->dep_lo);
        cudaFree(h->dep_hi);
        h->dep_lo = h->dep_hi = nullptr;
    }
    return SLA_OK;
}

static const void *pick_segment(sla_dtype dt, int lanes) {
    const void *f = nullptr;
    with_lanes(lanes, [&](auto L) -> sla_status {
        constexpr int LN = decltype(L)::value;
        f = dt == SLA_F64 ? reinterpret_cast<const void *>(&cg_segment_kernel<double, LN>)
                          : reinterpret_cast<const void *>(&cg_segment_kernel<float, LN>);
        return SLA_OK;
    });
    return f;
}

// Segment solver layout of a list handle: shared memory for the vectors of
// the largest item if it fits (else as many rows as fit; larger items use the
// workspace vectors), and as many resident blocks as that allows.
sla_status cg_configure_list(Csr *h) {
    const size_t ts = dtype_size(h->dtype);
    int optin = 0;
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, h->device);
    const void *f = pick_segment(h->dtype, h->lanes);
    sla_status st = smem_ceiling(f, h->device);
    if (st != SLA_OK) return st;
    const int64_t cap_rows = (int64_t)(optin - 8192) / (int64_t)(5 * ts);
    h->seg_smem_rows = (int32_t)std::min<int64_t>(h->seg_max, cap_rows);
    h->seg_smem = 5 * (size_t)h->seg_smem_rows * ts;
    int per_sm = 0;
    SLA_CHECK_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, f, kCgThreads, h->seg_smem));
    if (per_sm < 1) {
        set_error("sla_csr_list_create: the segment solver cannot be resident");
        return SLA_ERR_CUDA;
    }
    const int64_t blocks = (int64_t)per_sm * h->num_sms;
    h->seg_grid = (int32_t)std::max<int64_t>(1, std::min<int64_t>(h->n_items, blocks));
    return SLA_OK;
}

static size_t cg_ws_bytes(const Csr *h, bool adjoint) {
    const size_t ts = dtype_size(h->dtype);
    const size_t B = h->batch, n = h->n_rows, ntot = B * (size_t)h->ntiles;
    size_t b = align_up(64) + align_up(4 * B * 8) + align_up(B * 4) + align_up(4 * ntot * 8);
    b += 4 * align_up(B * n * ts);
    if (h->has_sell) b += align_up(B * (size_t)h->sell_nnz * (ts == 8 ? 16 : 8));   // values or records
    b += align_up((size_t)h->ntiles * 4);   // p-ready flags
    if (h->il_blocks > 0)                   // interleaved x and b, tile partials
        b += 2 * align_up(B * n * ts) + align_up(4 * B * (size_t)h->il_blocks * 8);
    if (adjoint && !(h->flags & SLA_FLAG_SYMMETRIC)) b += align_up(B * (size_t)h->nnz * ts);
    return b;
}

// Tile dependencies hold for the pattern they were built from (the forward
// pattern; the adjoint reuses it only on symmetric handles).
static bool pattern_is_forward_or_sym(const Csr *h, const int32_t *rowptr) {
    return rowptr == h->rowptr;
}

template <typename T>
static sla_status launch_cg(Csr *h, const int32_t *rowptr, const int32_t *colind,
                            const int32_t *diagpos, const T *vals, const T *b, T *x,
                            const sla_cg_opts *o, sla_cg_info info, Carver &c, cudaStream_t s,
                            bool pattern_is_forward) {
    CgArgs<T> a{};
    a.n = h->n_rows;
    a.B = h->batch;
    a.nnz = h->nnz;
    a.rowptr = rowptr;
    a.colind = colind;
    a.diagpos = diagpos;
    a.vals = vals;
    a.b = b;
    a.x = x;
    a.sync = c.take<unsigned>(16);
    a.sysd = c.take<double>(4 * (size_t)a.B);
    a.state = c.take<int>(a.B);
    a.part = c.take<double>(4 * (size_t)a.B * h->ntiles);
    const size_t vn = (size_t)a.B * a.n;
    a.r = c.take<T>(vn);
    a.p = c.take<T>(vn);
    a.q = c.take<T>(vn);
    a.d = c.take<T>(vn);
    a.out_iters = info.iters;
    a.out_relres = info.relres;
    a.out_status = info.status;
    a.rtol = o->rtol;
    a.atol = o->atol;
    a.fixed = o->fixed_iters > 0;
    a.limit = a.fixed ? o->fixed_iters
                      : (o->max_iter > 0 ? o->max_iter : (a.n < 10000 ? 10 * a.n : 100000));
    a.precond = o->precond ? 1 : 0;
    a.x0_given = o->x0_given ? 1 : 0;
    a.timeout_ns = o->wait_timeout_ns > 0 ? o->wait_timeout_ns : kDefaultTimeoutNs;
    a.tile_rows = h->tile_rows;
    a.ntiles = h->ntiles;
    if (h->dep_lo != nullptr && pattern_is_forward_or_sym(h, rowptr)) {
        a.dep_lo = h->dep_lo;
        a.dep_hi = h->dep_hi;
        a.pflag = c.take<unsigned>((size_t)h->ntiles);
    }
    if (h->n_items > 0) {
        SLA_REQUIRE(o->strategy == SLA_STRATEGY_AUTO || o->strategy == SLA_STRATEGY_BLOCK,
                    "sla_cg: a list of systems is solved one item a block (AUTO or BLOCK strategy)");
        SLA_CHECK_CUDA(cudaMemsetAsync(a.sync, 0, 16 * sizeof(unsigned), s));
        const int32_t *seg = h->seg, *order = h->seg_order;
        const int n_items = h->n_items, smem_rows = h->seg_smem_rows;
        unsigned *work = a.sync + 4;
        return with_lanes(h->lanes, [&](auto L) -> sla_status {
            constexpr int LN = decltype(L)::value;
            cg_segment_kernel<T, LN><<<h->seg_grid, kCgThreads, h->seg_smem, s>>>(
                a, seg, order, n_items, smem_rows, work);
            SLA_CHECK_LAUNCH();
            return SLA_OK;
        });
    }
    bool use_grid = true, use_cluster = false;
    if (o->strategy == SLA_STRATEGY_BLOCK) {
        SLA_REQUIRE(h->block_fits, "sla_cg: block strategy needs 5*n*sizeof(T) bytes of shared memory");
        use_grid = false;
    } else if (o->strategy == SLA_STRATEGY_CLUSTER) {
        SLA_REQUIRE(h->cluster_fits, "sla_cg: the system does not fit the cluster solver");
        use_grid = false;
        use_cluster = true;
    } else if (o->strategy == SLA_STRATEGY_AUTO) {
        // a cluster per system while the batch leaves SMs for all clusters at once
        use_cluster = h->cluster_fits && (int64_t)a.B * kClusterCTAs <= h->num_sms;
        use_grid = !use_cluster && !h->block_fits;
    }
    if (use_cluster) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)a.B * kClusterCTAs);
        cfg.blockDim = dim3(kClusterThreads);
        cfg.dynamicSmemBytes = h->cluster_smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kClusterCTAs;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        SLA_CHECK_CUDA(cudaLaunchKernelEx(&cfg, cg_cluster_kernel<T, kClusterThreads>, a,
                                          (int)h->cluster_rows, (int)h->cluster_nnz));
    } else if (use_grid) {
        const int ntot = a.B * a.ntiles;
        const int nlt = (ntot + h->grid_blocks - 1) / h->grid_blocks;
        if (nlt > kMaxLocalTiles) {
            set_error("sla_cg: %d systems of %d rows need %d tiles a block (limit %d); "
                      "use smaller batches", a.B, a.n, nlt, kMaxLocalTiles);
            return SLA_ERR_UNSUPPORTED;
        }
        // short rows on the forward pattern: the sliced layout, values laid out now
        const bool sell = h->has_sell && pattern_is_forward;
        if (sell && h->il_blocks > 0 && !h->onchip && (a.B == 2 || a.B == 4)) {
            // interleaved batch: values [slot][system], vectors [row][system]
            const int64_t n64 = a.n;
            T *sv = c.take<T>((size_t)a.B * h->sell_nnz);
            T *xi = c.take<T>((size_t)a.B * a.n);
            T *bi = c.take<T>((size_t)a.B * a.n);
            double *part = c.take<double>(4 * (size_t)a.B * h->il_blocks);
            const int tile_rows = (int)((n64 + h->il_blocks - 1) / h->il_blocks);
            const int ntiles = (int)((n64 + tile_rows - 1) / tile_rows);
            const unsigned gv = (unsigned)((n64 * a.B + 255) / 256);
            const unsigned gs = (unsigned)((h->sell_nnz * a.B + 255) / 256);
            sell_values_il_kernel<T><<<gs, 256, 0, s>>>(h->sell_nnz, h->nnz, a.B, h->sell_map, vals, sv);
            interleave_kernel<T><<<gv, 256, 0, s>>>(n64, a.B, b, bi);
            if (a.x0_given) interleave_kernel<T><<<gv, 256, 0, s>>>(n64, a.B, x, xi);
            SLA_CHECK_LAUNCH();
            a.sell_ptr = h->sell_ptr;
            a.sell_cols = h->sell_cols;
            a.sell_vals = sv;
            a.sell_nnz = h->sell_nnz;
            a.sell_w = h->sell_w;
            a.sell_d16 = h->sell_d16;
            const char *sp = getenv("SLA_SELL_PIPE");
            a.sell_pipe = sp && sp[0] == '0' ? 0 : 1;
            SLA_CHECK_CUDA(cudaMemsetAsync(a.sync, 0, 16 * sizeof(unsigned), s));
            const T *bic = bi;
            void *args[] = {&a, &xi, &bic, &part, (void *)&tile_rows, (void *)&ntiles};
            SLA_CHECK_CUDA(cudaLaunchCooperativeKernel(pick_il(h->dtype, a.B), dim3(h->il_blocks),
                                                       dim3(kCgThreads), args, 0, s));
            deinterleave_kernel<T><<<gv, 256, 0, s>>>(n64, a.B, xi, x);
            SLA_CHECK_LAUNCH();
            return SLA_OK;
        }
        if (sell) {
            a.sell_ptr = h->sell_ptr;
            a.sell_cols = h->sell_cols;
            a.sell_nnz = h->sell_nnz;
            a.sell_w = h->sell_w;
            const char *sp = getenv("SLA_SELL_PIPE");
            a.sell_pipe = sp && sp[0] == '0' ? 0 : 1;
            a.sell_perm = h->sell_perm;
            a.sell_d16 = h->sell_d16;
            const char *pk = getenv("SLA_SELL_PACK");
            const bool pack = pk && pk[0] == '1' && !(h->grid2 && a.B == 1);
            if (pack) {
                SellRec<T> *rec = c.take<SellRec<T>>((size_t)a.B * h->sell_nnz);
                sell_pack_kernel<T><<<(unsigned)((h->sell_nnz + 255) / 256), 256, 0, s>>>(
                    h->sell_nnz, h->nnz, a.B, h->sell_map, h->sell_cols, vals, rec);
                SLA_CHECK_LAUNCH();
                a.sell_rec = rec;
            } else {
                T *sv = c.take<T>((size_t)a.B * h->sell_nnz);
                sla_status st = sell_values(h, vals, sv, s);
                if (st != SLA_OK) return st;
                a.sell_vals = sv;
            }
        }
        SLA_CHECK_CUDA(cudaMemsetAsync(a.sync, 0, 16 * sizeof(unsigned), s));
        if (a.pflag) SLA_CHECK_CUDA(cudaMemsetAsync(a.pflag, 0, (size_t)h->ntiles * sizeof(unsigned), s));
        void *args[] = {&a};
        const void *f = sell && h->grid2 && a.B == 1 ? pick_grid2(h->dtype, h->onchip_rpt)
                                                     : pick_grid(h, sell);
        SLA_CHECK_CUDA(cudaLaunchCooperativeKernel(f, dim3(h->grid_blocks), dim3(h->grid_threads),
                                                   args, h->grid_smem, s));
    } else {
        const int grid = a.B < h->block_grid ? a.B : h->block_grid;
        void *args[] = {&a};
        SLA_CHECK_CUDA(cudaLaunchKernel(pick_block(h->dtype, h->lanes, h->block_mres), dim3(grid),
                                        dim3(kCgThreads), args, h->block_smem, s));
    }
    return SLA_OK;
}

static sla_status check_opts(const sla_cg_opts *o) {
    SLA_REQUIRE(o != nullptr, "sla_cg: NULL opts");
    SLA_REQUIRE(o->rtol >= 0.0 && o->atol >= 0.0 && std::isfinite(o->rtol) && std::isfinite(o->atol),
                "sla_cg: rtol/atol must be finite and >= 0");
    SLA_REQUIRE(o->fixed_iters >= 0, "sla_cg: fixed_iters < 0");
    SLA_REQUIRE(o->strategy >= 0 && o->strategy <= 3, "sla_cg: unknown strategy %d", o->strategy);
    SLA_REQUIRE(o->reserved == 0, "sla_cg: reserved field must be 0");
    return SLA_OK;
}

static sla_status cg_entry(Csr *h, const void *vals, const void *rhs, void *x,
                           const sla_cg_opts *o, sla_cg_info info, void *ws, size_t ws_bytes,
                           void *stream, bool adjoint) {
    SLA_REQUIRE(h != nullptr, "sla_cg: NULL handle");
    sla_status st = check_opts(o);
    if (st != SLA_OK) return st;
    SLA_REQUIRE(h->n_rows == h->n_cols, "sla_cg: matrix must be square (%d x %d)", h->n_rows, h->n_cols);
    cudaStream_t s = as_stream(stream);
    if (h->n_rows == 0) {
        const int count = h->n_items > 0 ? h->n_items : h->batch;
        info_fill_kernel<<<(count + 255) / 256, 256, 0, s>>>(count, info.iters, info.relres,
                                                             info.status);
        SLA_CHECK_LAUNCH();
        return SLA_OK;
    }
    SLA_REQUIRE(vals && rhs && x, "sla_cg: NULL vals, rhs or x");
    const size_t need = cg_ws_bytes(h, adjoint);
    SLA_REQUIRE(ws != nullptr && ws_bytes >= need, "sla_cg: workspace too small (%zu < %zu)",
                ws_bytes, need);
    SLA_REQUIRE(((uintptr_t)ws & 255) == 0, "sla_cg: workspace must be 256-byte aligned");
    Carver c(ws);
    const int32_t *rp = h->rowptr, *ci = h->colind, *dp = h->diagpos;
    const void *v = vals;
    if (adjoint && !(h->flags & SLA_FLAG_SYMMETRIC)) {
        st = ensure_transpose(h, s);
        if (st != SLA_OK) return st;
        rp = h->rowptrT;
        ci = h->colindT;
        dp = h->diagposT;
        // A^T's values: a gather through the stable transpose permutation
        void *vt = c.take<char>((size_t)h->batch * h->nnz * dtype_size(h->dtype));
        st = transpose_values(h, vals, vt, s);
        if (st != SLA_OK) return st;
        v = vt;
    }
    const bool forward_pattern = rp == h->rowptr;
    if (h->dtype == SLA_F64)
        return launch_cg<double>(h, rp, ci, dp, (const double *)v, (const double *)rhs,
                                 (double *)x, o, info, c, s, forward_pattern);
    return launch_cg<float>(h, rp, ci, dp, (const float *)v, (const float *)rhs, (float *)x, o,
                            info, c, s, forward_pattern);
}

}  // namespace sla

using namespace sla;

extern "C" size_t sla_workspace_bytes(sla_csr_t hh, int32_t op) {
    const Csr *h = reinterpret_cast<const Csr *>(hh);
    if (!h) return 0;
    if (op == SLA_OP_CG) return h->n_rows == h->n_cols ? cg_ws_bytes(h, false) : 0;
    if (op == SLA_OP_ADJOINT) return h->n_rows == h->n_cols ? cg_ws_bytes(h, true) : 0;
    return 0;
}

extern "C" sla_status sla_cg_solve(sla_csr_t hh, const void *vals, const void *b, void *x,
                                   const sla_cg_opts *opts, sla_cg_info info, void *ws,
                                   size_t ws_bytes, void *stream) {
    SLA_RANGE("sla_cg_solve");
    clear_error();
    return cg_entry(reinterpret_cast<Csr *>(hh), vals, b, x, opts, info, ws, ws_bytes, stream, false);
}

extern "C" sla_status sla_cg_adjoint(sla_csr_t hh, const void *vals, const void *g, void *lambda,
                                     const sla_cg_opts *opts, sla_cg_info info, void *ws,
                                     size_t ws_bytes, void *stream) {
    SLA_RANGE("sla_cg_adjoint");
    clear_error();
    return cg_entry(reinterpret_cast<Csr *>(hh), vals, g, lambda, opts, info, ws, ws_bytes, stream,
                    true);
}

// ------------------------------------------------ allocation-free solve ----
// The same persistent solver for callers that may not allocate device memory
// while they solve: runtimes that reserve all device memory up front and hand
// it out themselves, loops that cannot afford the device-wide synchronisation
// that cudaMalloc and cudaFree may imply, and plugins that must not call into
// their host application's allocator.  Its scratch (synchronisation words, partial sums, per-system
// scalars, diagonal positions and the r, p, q, M^-1 vectors) lives in one
// file-scope device array that every GPU loading this library keeps until the
// process exits.  The array is shared by all calls on a device and keeps what
// the last call left there, so this entry point clears what must start at
// zero, and calls whose kernels overlap on the GPU race on it.
namespace sla {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Host code sees g_noalloc_scratch only as a host-side stand-in; the device
// address comes from cudaGetSymbolAddress with the caller's context current.
// It is looked up on every call (a host-side table lookup once the module is
// loaded): a cached address would go stale when the caller switches to another
// context of the same device or resets the device, because the library's
// module, and with it the array, is then loaded again at another address.
static sla_status noalloc_scratch(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
        set_error("sla_cg_solve_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
        return SLA_ERR_CUDA;
    }
    *out = p;
    return SLA_OK;
}

template <typename T>
static sla_status noalloc_launch(const Csr &h, const T *vals, const T *b, T *x,
                                 const sla_cg_opts *o, sla_cg_info info, void *scratch,
                                 size_t need, cudaStream_t s) {
    Carver c(scratch);
    int32_t *diagpos = c.take<int32_t>((size_t)h.n_rows);
    CgArgs<T> a{};
    a.n = h.n_rows;
    a.B = h.batch;
    a.nnz = h.nnz;
    a.rowptr = h.rowptr;
    a.colind = h.colind;
    a.diagpos = diagpos;
    a.vals = vals;
    a.b = b;
    a.x = x;
    a.sync = c.take<unsigned>(16);
    a.sysd = c.take<double>(4 * (size_t)a.B);
    a.state = c.take<int>(a.B);
    a.part = c.take<double>(4 * (size_t)a.B * h.ntiles);
    const size_t vn = (size_t)a.B * a.n;
    a.r = c.take<T>(vn);
    a.p = c.take<T>(vn);
    a.q = c.take<T>(vn);
    a.d = c.take<T>(vn);
    if (c.off > need) {
        set_error("sla_cg_solve_noalloc: internal scratch layout mismatch");
        return SLA_ERR_CUDA;
    }
    a.out_iters = info.iters;
    a.out_relres = info.relres;
    a.out_status = info.status;
    a.rtol = o->rtol;
    a.atol = o->atol;
    a.fixed = o->fixed_iters > 0;
    a.limit = a.fixed ? o->fixed_iters
                      : (o->max_iter > 0 ? o->max_iter : (a.n < 10000 ? 10 * a.n : 100000));
    a.precond = o->precond ? 1 : 0;
    a.x0_given = o->x0_given ? 1 : 0;
    a.timeout_ns = o->wait_timeout_ns > 0 ? o->wait_timeout_ns : kDefaultTimeoutNs;
    a.tile_rows = h.tile_rows;
    a.ntiles = h.ntiles;
    // the previous call's arrival counter and flags must not leak into this one
    SLA_CHECK_CUDA(cudaMemsetAsync(a.sync, 0, 16 * sizeof(unsigned), s));
    sla_status st = diag_positions(h.n_rows, h.rowptr, h.colind, diagpos, s);
    if (st != SLA_OK) return st;
    void *args[] = {&a};
    SLA_CHECK_CUDA(cudaLaunchCooperativeKernel(pick_fn(true, h.dtype, h.lanes), dim3(h.grid_blocks),
                                               dim3(kCgThreads), args, 0, s));
    return SLA_OK;
}

}  // namespace sla

extern "C" sla_status sla_cg_solve_noalloc(int32_t n, int64_t nnz, const int32_t *rowptr,
                                           const int32_t *colind, int32_t batch, sla_dtype dtype,
                                           const void *vals, const void *b, void *x,
                                           const sla_cg_opts *opts, sla_cg_info info,
                                           void *stream) {
    SLA_RANGE("sla_cg_solve_noalloc");
    clear_error();
    SLA_REQUIRE(n >= 0 && nnz >= 0 && nnz <= 0x7fffffff, "sla_cg_solve_noalloc: bad sizes n=%d nnz=%lld",
                n, (long long)nnz);
    SLA_REQUIRE(batch >= 1, "sla_cg_solve_noalloc: batch must be >= 1");
    SLA_REQUIRE(dtype == SLA_F64 || dtype == SLA_F32, "sla_cg_solve_noalloc: bad dtype %d", (int)dtype);
    sla_status st = check_opts(opts);
    if (st != SLA_OK) return st;
    SLA_REQUIRE(opts->strategy != SLA_STRATEGY_BLOCK,
                "sla_cg_solve_noalloc: runs the grid solver only");
    cudaStream_t s = as_stream(stream);
    if (n == 0) {
        info_fill_kernel<<<(batch + 255) / 256, 256, 0, s>>>(batch, info.iters, info.relres, info.status);
        SLA_CHECK_LAUNCH();
        return SLA_OK;
    }
    SLA_REQUIRE(rowptr && (nnz == 0 || colind) && vals && b && x, "sla_cg_solve_noalloc: NULL pointer");
    // A handle description on the host stack: no device memory is involved.
    Csr h;
    h.n_rows = h.n_cols = n;
    h.nnz = nnz;
    h.batch = batch;
    h.dtype = dtype;
    h.rowptr = rowptr;
    h.colind = colind;
    h.lanes = lanes_for_mean((double)nnz / n);
    SLA_CHECK_CUDA(cudaGetDevice(&h.device));
    SLA_CHECK_CUDA(cudaDeviceGetAttribute(&h.num_sms, cudaDevAttrMultiProcessorCount, h.device));
    int per_sm = 0;
    SLA_CHECK_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &per_sm, pick_fn(true, dtype, h.lanes), kCgThreads, 0));
    per_sm = per_sm < 2 ? per_sm : 2;
    if (per_sm < 1) {
        set_error("sla_cg_solve_noalloc: persistent kernel cannot be resident");
        return SLA_ERR_CUDA;
    }
    h.grid_blocks = per_sm * h.num_sms;
    layout(&h, h.grid_blocks, &h.tile_rows, &h.ntiles);
    const int ntot = batch * h.ntiles;
    if ((ntot + h.grid_blocks - 1) / h.grid_blocks > kMaxLocalTiles) {
        set_error("sla_cg_solve_noalloc: batch of %d systems too large for one launch", batch);
        return SLA_ERR_UNSUPPORTED;
    }
    const size_t ts = dtype_size(dtype), B = batch, rows = (size_t)n;
    const size_t need = align_up(rows * 4) + align_up(64) + align_up(4 * B * 8) + align_up(B * 4) +
                        align_up(4 * (size_t)ntot * 8) + 4 * align_up(B * rows * ts);
    SLA_REQUIRE(need <= kNoAllocScratchBytes,
                "sla_cg_solve_noalloc: %d system(s) of %d rows need %zu bytes of scratch; the "
                "built-in limit is %zu bytes (use sla_cg_solve with a caller workspace)",
                batch, n, need, kNoAllocScratchBytes);
    void *scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != SLA_OK) return st;
    if (dtype == SLA_F64)
        return noalloc_launch<double>(h, (const double *)vals, (const double *)b, (double *)x, opts,
                                      info, scratch, need, s);
    return noalloc_launch<float>(h, (const float *)vals, (const float *)b, (float *)x, opts, info,
                                 scratch, need, s);
}
