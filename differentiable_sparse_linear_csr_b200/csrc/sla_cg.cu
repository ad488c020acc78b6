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
// Two kernels implement it:
//  * cg_grid_kernel -- one persistent cooperative grid (all blocks resident)
//    for systems too large for one block.  Rows are split into fixed tiles; a
//    block owns the same tiles in every phase.  Three device-wide barriers per
//    iteration separate SpMV+p.q, the x/r update with r.z and r.r, and the
//    direction update.  Every block reduces the per-tile partials of a system
//    itself, in one fixed order, so all blocks take identical decisions
//    without extra communication; results are bit-reproducible run to run.
//  * cg_block_kernel -- one thread block per system with x, r, p, q, M^-1 in
//    shared memory (small systems, large batches): no device-wide barrier.
#include <cmath>
#include <cstdlib>

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
};

// ------------------------------------------------------------ helpers ----
template <typename T>
__device__ __forceinline__ void finalize(const CgArgs<T> &a, int s, int status, int iters,
                                         double relres, bool count_down) {
    a.state[s] = status;
    if (a.out_status) a.out_status[s] = status;
    if (a.out_iters) a.out_iters[s] = iters;
    if (a.out_relres) a.out_relres[s] = relres;
    if (count_down) atomicSub(a.sync + 3, 1u);
}

// Sum of a system's tile partials, in tile order per lane and a fixed xor tree
// across lanes: the same value in every block.  NV arrays at once; results in
// out[0..NV) for all threads of the block.
template <int NV>
__device__ __forceinline__ void system_sums(const double *const (&arr)[NV], int ntiles,
                                            double *out) {
    __syncthreads();
    if (threadIdx.x < 32) {
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            double acc = 0.0;
            for (int j = threadIdx.x; j < ntiles; j += 32) acc += __ldcg(arr[v] + j);
            acc = warp_sum(acc);
            if (threadIdx.x == 0) out[v] = acc;
        }
    }
    __syncthreads();
}

__device__ __forceinline__ int read_state_uniform(const int *state, int s, int *sh) {
    __syncthreads();
    if (threadIdx.x == 0) *sh = __ldcg(state + s);
    __syncthreads();
    return *sh;
}

// Device-wide barrier that also reports, block-uniformly, the number of
// systems still active as seen after the barrier.
__device__ __forceinline__ bool barrier_and_watch(unsigned *sync, long long timeout_ns,
                                                  int *flag, unsigned *active) {
    const bool ok = grid_barrier(sync, gridDim.x, timeout_ns, flag);
    if (threadIdx.x == 0) *active = ld_acquire_u32(sync + 3);
    __syncthreads();
    return ok;
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
template <typename T, int LANES>
__global__ void __launch_bounds__(kCgThreads)
cg_grid_kernel(CgArgs<T> a) {
    __shared__ double red[72];
    __shared__ double bc[4];
    __shared__ int flag, st_sh;
    __shared__ unsigned active;
    constexpr int NSUB = kCgThreads / LANES;
    const int tid = threadIdx.x, sub = tid / LANES, lane = tid % LANES;
    const int ntot = a.B * a.ntiles;
    double *P0 = a.part, *P1 = P0 + ntot, *P2 = P1 + ntot, *P3 = P2 + ntot;
    double *rho = a.sysd, *nbv = a.sysd + 2 * a.B, *rrv = a.sysd + 3 * a.B;
    const int n = a.n;

    if (blockIdx.x == 0 && tid == 0) a.sync[3] = (unsigned)a.B;

    // ---- init: r = b - A x0 (or b), z = M^-1 r, p = z; partials of b.b, r.z, r.r
    for (int tile = blockIdx.x; tile < ntot; tile += gridDim.x) {
        const int s = tile / a.ntiles, tt = tile % a.ntiles;
        const int r0 = tt * a.tile_rows, r1 = min(n, r0 + a.tile_rows);
        const T *vs = a.vals + (int64_t)s * a.nnz;
        const T *bs = a.b + (int64_t)s * n;
        T *xs = a.x + (int64_t)s * n, *rs = a.r + (int64_t)s * n, *ps = a.p + (int64_t)s * n;
        T *qs = a.q + (int64_t)s * n, *ds = a.d + (int64_t)s * n;
        if (a.x0_given) {
            for (int i = r0 + sub; i < r1; i += NSUB) {
                const T v = row_dot<T, LANES>(a.rowptr, a.colind, vs, xs, i, lane);
                if (lane == 0) qs[i] = v;
            }
            __syncthreads();
        }
        double lbb = 0.0, lrho = 0.0, lrr = 0.0, lbad = 0.0;
        for (int i = r0 + tid; i < r1; i += kCgThreads) {
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
                const T dv = dp >= 0 ? __ldg(vs + dp) : T(0);
                if (!(dv > T(0))) lbad += 1.0;
                di = T(1) / dv;
            }
            const T zi = di * ri;
            rs[i] = ri;
            ps[i] = zi;
            ds[i] = di;
            lbb += (double)bi * (double)bi;
            lrho += (double)ri * (double)zi;
            lrr += (double)ri * (double)ri;
        }
        block_sum2<kCgThreads>(lbb, lrho, red);
        block_sum2<kCgThreads>(lrr, lbad, red);
        if (tid == 0) {
            P0[tile] = lbb;
            P1[tile] = lrho;
            P2[tile] = lrr;
            P3[tile] = lbad;
        }
    }
    if (!grid_barrier(a.sync, gridDim.x, a.timeout_ns, &flag)) { give_up(a); return; }

    // ---- initial decisions, made identically by every block holding a tile
    for (int tile = blockIdx.x; tile < ntot; tile += gridDim.x) {
        const int s = tile / a.ntiles, tt = tile % a.ntiles;
        const int off = s * a.ntiles;
        const double *const arr[4] = {P0 + off, P1 + off, P2 + off, P3 + off};
        system_sums<4>(arr, a.ntiles, bc);
        const double bb = bc[0], rho0 = bc[1], rr = bc[2], bad = bc[3];
        const double nb = sqrt(bb);
        const double tol = fmax(a.rtol * nb, a.atol);
        int st = kActive;
        double relres = 0.0;
        if (nb == 0.0) st = SLA_CONVERGED;
        else if (!isfinite(nb)) st = SLA_NONFINITE;
        else if (a.precond && bad > 0.0) { st = SLA_BREAKDOWN; relres = sqrt(rr) / nb; }
        else if (!a.fixed && sqrt(rr) <= tol) { st = SLA_CONVERGED; relres = sqrt(rr) / nb; }
        else if (rr == 0.0) st = SLA_CONVERGED;
        if (nb == 0.0 && a.x0_given) {
            const int r0 = tt * a.tile_rows, r1 = min(n, r0 + a.tile_rows);
            T *xs = a.x + (int64_t)s * n;
            for (int i = r0 + tid; i < r1; i += kCgThreads) xs[i] = T(0);
        }
        if (tt == 0 && tid == 0) {
            rho[s] = rho0;
            nbv[s] = nb;
            rrv[s] = rr;
            if (st == kActive) a.state[s] = kActive;
            else finalize(a, s, st, 0, relres, true);
        }
    }
    if (!barrier_and_watch(a.sync, a.timeout_ns, &flag, &active)) { give_up(a); return; }

    int k = 0;
    while (active != 0) {
        // ---- phase A: q = A p and the partials of p.q
        for (int tile = blockIdx.x; tile < ntot; tile += gridDim.x) {
            const int s = tile / a.ntiles, tt = tile % a.ntiles;
            if (read_state_uniform(a.state, s, &st_sh) != kActive) continue;
            const int r0 = tt * a.tile_rows, r1 = min(n, r0 + a.tile_rows);
            const T *vs = a.vals + (int64_t)s * a.nnz;
            const T *ps = a.p + (int64_t)s * n;
            T *qs = a.q + (int64_t)s * n;
            double ls = 0.0;
            for (int i = r0 + sub; i < r1; i += NSUB) {
                const T qi = row_dot<T, LANES>(a.rowptr, a.colind, vs, ps, i, lane);
                if (lane == 0) {
                    qs[i] = qi;
                    ls += (double)ps[i] * (double)qi;
                }
            }
            ls = block_sum<kCgThreads>(ls, red);
            if (tid == 0) P0[tile] = ls;
        }
        if (!grid_barrier(a.sync, gridDim.x, a.timeout_ns, &flag)) { give_up(a); return; }
        ++k;

        // ---- phase B: alpha; x += alpha p; r -= alpha q; partials of r.z, r.r
        for (int tile = blockIdx.x; tile < ntot; tile += gridDim.x) {
            const int s = tile / a.ntiles, tt = tile % a.ntiles;
            if (read_state_uniform(a.state, s, &st_sh) != kActive) continue;
            const double *const arr[1] = {P0 + s * a.ntiles};
            system_sums<1>(arr, a.ntiles, bc);
            const double sigma = bc[0];
            if (!isfinite(sigma) || !(sigma > 0.0)) {
                if (tt == 0 && tid == 0)
                    finalize(a, s, isfinite(sigma) ? SLA_BREAKDOWN : SLA_NONFINITE, k - 1,
                             sqrt(rrv[s]) / nbv[s], true);
                continue;
            }
            const T al = (T)(__ldcg(rho + ((k - 1) & 1) * a.B + s) / sigma);
            const int r0 = tt * a.tile_rows, r1 = min(n, r0 + a.tile_rows);
            T *xs = a.x + (int64_t)s * n, *rs = a.r + (int64_t)s * n;
            const T *ps = a.p + (int64_t)s * n, *qs = a.q + (int64_t)s * n, *ds = a.d + (int64_t)s * n;
            double lrho = 0.0, lrr = 0.0;
            for (int i = r0 + tid; i < r1; i += kCgThreads) {
                const T pi = ps[i];
                xs[i] = xs[i] + al * pi;
                const T ri = rs[i] - al * qs[i];
                rs[i] = ri;
                const T zi = ds[i] * ri;
                lrho += (double)ri * (double)zi;
                lrr += (double)ri * (double)ri;
            }
            block_sum2<kCgThreads>(lrho, lrr, red);
            if (tid == 0) {
                P1[tile] = lrho;
                P2[tile] = lrr;
            }
        }
        if (!grid_barrier(a.sync, gridDim.x, a.timeout_ns, &flag)) { give_up(a); return; }

        // ---- phase C: stopping test; beta; p = z + beta p
        for (int tile = blockIdx.x; tile < ntot; tile += gridDim.x) {
            const int s = tile / a.ntiles, tt = tile % a.ntiles;
            if (read_state_uniform(a.state, s, &st_sh) != kActive) continue;
            const double *const arr[2] = {P1 + s * a.ntiles, P2 + s * a.ntiles};
            system_sums<2>(arr, a.ntiles, bc);
            const double rho_new = bc[0], rr = bc[1];
            const double nb = __ldcg(nbv + s);
            const double tol = fmax(a.rtol * nb, a.atol);
            int st = kActive;
            if (!isfinite(rr)) st = SLA_NONFINITE;
            else if (!a.fixed && sqrt(rr) <= tol) st = SLA_CONVERGED;
            else if (rr == 0.0) st = SLA_CONVERGED;
            else if (k >= a.limit) st = a.fixed ? SLA_FIXED_DONE : SLA_NOT_CONVERGED;
            if (st != kActive) {
                if (tt == 0 && tid == 0) finalize(a, s, st, k, sqrt(rr) / nb, true);
                continue;
            }
            const double rho_old = __ldcg(rho + ((k - 1) & 1) * a.B + s);
            const T bt = (T)(rho_new / rho_old);
            const int r0 = tt * a.tile_rows, r1 = min(n, r0 + a.tile_rows);
            const T *rs = a.r + (int64_t)s * n, *ds = a.d + (int64_t)s * n;
            T *ps = a.p + (int64_t)s * n;
            for (int i = r0 + tid; i < r1; i += kCgThreads) ps[i] = ds[i] * rs[i] + bt * ps[i];
            if (tt == 0 && tid == 0) {
                rho[(k & 1) * a.B + s] = rho_new;
                rrv[s] = rr;
            }
        }
        if (!barrier_and_watch(a.sync, a.timeout_ns, &flag, &active)) { give_up(a); return; }
    }
}

// ------------------------------------------------------ block kernel ----
template <typename T, int LANES>
__global__ void __launch_bounds__(kCgThreads)
cg_block_kernel(CgArgs<T> a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ double red[72];
    constexpr int NSUB = kCgThreads / LANES;
    const int tid = threadIdx.x, sub = tid / LANES, lane = tid % LANES;
    const int n = a.n;
    T *xs = reinterpret_cast<T *>(smem_raw);
    T *rs = xs + n, *ps = rs + n, *qs = ps + n, *ds = qs + n;

    for (int s = blockIdx.x; s < a.B; s += gridDim.x) {
        const T *vs = a.vals + (int64_t)s * a.nnz;
        const T *bs = a.b + (int64_t)s * n;
        T *xg = a.x + (int64_t)s * n;
        __syncthreads();
        if (a.x0_given) {
            for (int i = tid; i < n; i += kCgThreads) xs[i] = xg[i];
            __syncthreads();
            for (int i = sub; i < n; i += NSUB) {
                const T v = row_dot<T, LANES>(a.rowptr, a.colind, vs, xs, i, lane);
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
                const T dv = dp >= 0 ? __ldg(vs + dp) : T(0);
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
                const T qi = row_dot<T, LANES>(a.rowptr, a.colind, vs, ps, i, lane);
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

__global__ void info_fill_kernel(int B, int32_t *iters, double *relres, int32_t *status) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= B) return;
    if (iters) iters[s] = 0;
    if (relres) relres[s] = 0.0;
    if (status) status[s] = SLA_CONVERGED;
}

// ----------------------------------------------------------- host side ----
template <typename T, int L>
static const void *grid_fn() { return reinterpret_cast<const void *>(&cg_grid_kernel<T, L>); }
template <typename T, int L>
static const void *block_fn() { return reinterpret_cast<const void *>(&cg_block_kernel<T, L>); }

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

sla_status cg_configure(Csr *h) {
    const size_t ts = dtype_size(h->dtype);
    const int n = h->n_rows;
    int optin = 0;
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, h->device);
    h->block_smem = 5 * (size_t)n * ts;
    h->block_fits = n > 0 && h->block_smem + 2048 <= (size_t)optin;
    if (h->block_fits) {
        // the same ceiling for every handle, so one handle never lowers another's
        SLA_CHECK_CUDA(cudaFuncSetAttribute(pick_fn(false, h->dtype, h->lanes),
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            optin - 2048));
    }
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
    const int B = h->batch;
    int ntiles = h->grid_blocks / B;
    if (ntiles < 1) ntiles = 1;
    int64_t tr = n > 0 ? ((int64_t)n + ntiles - 1) / ntiles : 1;
    if (tr > 32) tr = (tr + 31) / 32 * 32;
    h->tile_rows = (int32_t)tr;
    h->ntiles = n > 0 ? (int32_t)(((int64_t)n + tr - 1) / tr) : 1;
    return SLA_OK;
}

static size_t cg_ws_bytes(const Csr *h, bool adjoint) {
    const size_t ts = dtype_size(h->dtype);
    const size_t B = h->batch, n = h->n_rows, ntot = B * (size_t)h->ntiles;
    size_t b = align_up(64) + align_up(4 * B * 8) + align_up(B * 4) + align_up(4 * ntot * 8);
    b += 4 * align_up(B * n * ts);
    if (adjoint && !(h->flags & SLA_FLAG_SYMMETRIC)) b += align_up(B * (size_t)h->nnz * ts);
    return b;
}

template <typename T>
static sla_status launch_cg(Csr *h, const int32_t *rowptr, const int32_t *colind,
                            const int32_t *diagpos, const T *vals, const T *b, T *x,
                            const sla_cg_opts *o, sla_cg_info info, Carver &c, cudaStream_t s) {
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
    bool use_grid = true;
    if (o->strategy == SLA_STRATEGY_BLOCK) {
        SLA_REQUIRE(h->block_fits, "sla_cg: block strategy needs 5*n*sizeof(T) bytes of shared memory");
        use_grid = false;
    } else if (o->strategy == SLA_STRATEGY_AUTO) {
        use_grid = !h->block_fits;
    }
    if (use_grid) {
        SLA_CHECK_CUDA(cudaMemsetAsync(a.sync, 0, 16 * sizeof(unsigned), s));
        void *args[] = {&a};
        SLA_CHECK_CUDA(cudaLaunchCooperativeKernel(pick_fn(true, h->dtype, h->lanes),
                                                   dim3(h->grid_blocks), dim3(kCgThreads), args,
                                                   0, s));
    } else {
        const int per = h->num_sms * 4;
        const int grid = a.B < per ? a.B : per;
        void *args[] = {&a};
        SLA_CHECK_CUDA(cudaLaunchKernel(pick_fn(false, h->dtype, h->lanes), dim3(grid),
                                        dim3(kCgThreads), args, h->block_smem, s));
    }
    return SLA_OK;
}

static sla_status check_opts(const sla_cg_opts *o) {
    SLA_REQUIRE(o != nullptr, "sla_cg: NULL opts");
    SLA_REQUIRE(o->rtol >= 0.0 && o->atol >= 0.0 && std::isfinite(o->rtol) && std::isfinite(o->atol),
                "sla_cg: rtol/atol must be finite and >= 0");
    SLA_REQUIRE(o->fixed_iters >= 0, "sla_cg: fixed_iters < 0");
    SLA_REQUIRE(o->strategy >= 0 && o->strategy <= 2, "sla_cg: unknown strategy %d", o->strategy);
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
        info_fill_kernel<<<(h->batch + 255) / 256, 256, 0, s>>>(h->batch, info.iters, info.relres,
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
    if (h->dtype == SLA_F64)
        return launch_cg<double>(h, rp, ci, dp, (const double *)v, (const double *)rhs,
                                 (double *)x, o, info, c, s);
    return launch_cg<float>(h, rp, ci, dp, (const float *)v, (const float *)rhs, (float *)x, o,
                            info, c, s);
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
    clear_error();
    return cg_entry(reinterpret_cast<Csr *>(hh), vals, b, x, opts, info, ws, ws_bytes, stream, false);
}

extern "C" sla_status sla_cg_adjoint(sla_csr_t hh, const void *vals, const void *g, void *lambda,
                                     const sla_cg_opts *opts, sla_cg_info info, void *ws,
                                     size_t ws_bytes, void *stream) {
    clear_error();
    return cg_entry(reinterpret_cast<Csr *>(hh), vals, g, lambda, opts, info, ws, ws_bytes, stream,
                    true);
}
