// Batched CSR SpMV (the `.matvec` call) and the sparse value gradients on the
// stored entries: dL/dA_ij = -lambda_i x_j after a solve, and dL/dA_ij =
// gy_i x_j for y = A x.
//   torch-sla summary page, technical summary: "Methodology" 1 (`.matvec`)
//   and "Methodology" 2 (linear systems: gradient on the sparsity pattern).
//
// Short rows (one thread a row):
//  - SpMV: a block takes 256 consecutive rows, whose entries are one contiguous
//    range of the CSR arrays; it copies the range's columns and values into
//    shared memory with coalesced loads, then each thread sums its own row
//    there in stored order while gathering x (the rounding of a thread walking
//    the row in global memory).  Gathering row by row keeps a warp's gathers of
//    x together for banded patterns (consecutive rows reach consecutive
//    columns); gathering entry by entry measured slower.
//    Resident blocks run a pipelined form of this when the arrays are on the
//    16-byte grid (after the staged kernel).
//  - Value gradients: each warp takes 32 rows and walks their entry range in
//    order, the row of each entry taken from a per-warp table, so column reads
//    and gradient stores are coalesced.
// Both issue a group of kStage loads into registers before using any, so that
// they are in flight together.  A block or warp whose range exceeds its shared
// memory walks its rows in global memory.  Long rows (LANES > 1 threads a row)
// are walked by sub-warps, which already read consecutive entries.
#include "sla_rows.cuh"

namespace sla {

constexpr int kChunkRows = 256;          // rows (and threads) of one staged SpMV block
constexpr int kWarpRows = 32;            // rows of one warp in the one-thread-row gradient
constexpr int kRowWarps = 8;             // warps of one block there
constexpr int kStage = 8;                // SpMV: loads issued before any is used
constexpr int kGradStage = 4;            // the same for the gradient (more registers a step)

// Entries a staged SpMV block holds: room for rows 2 entries longer than the
// mean (so that 8 blocks fit an SM for rows of 7), at most 4096; a chunk with
// more walks its rows in global memory.
static int chunk_cap(double row_mean) {
    const double c = kChunkRows * (row_mean + 2.0);
    return c >= 4096.0 ? 4096 : ((int)c + 31) / 32 * 32;
}

static dim3 chunk_grid(int rows, int B) {
    return dim3((unsigned)((rows + kChunkRows - 1) / kChunkRows), (unsigned)(B < 65535 ? B : 65535));
}

// Entries one gradient warp tabulates: room for rows 4 entries longer than
// the mean, at most 1024; a warp with more walks its rows in global memory.
// A product rounded on its own (the compiler must not fuse it into a
// following add), as the gradient's definition rounds it.
template <typename T>
__device__ __forceinline__ T mul_rn(T a, T b) {
    if constexpr (sizeof(T) == 8) return __dmul_rn(a, b);
    else return __fmul_rn(a, b);
}

static int warp_cap(double row_mean) {
    const double c = kWarpRows * (row_mean + 4.0);
    return c >= 1024.0 ? 1024 : ((int)c + 31) / 32 * 32;
}

static dim3 warp_grid(int rows, int B) {
    const int rpb = kWarpRows * kRowWarps;
    return dim3((unsigned)((rows + rpb - 1) / rpb), (unsigned)(B < 65535 ? B : 65535));
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

// y = alpha A x + beta y for one-thread rows, 256 rows a block (see the file
// comment).
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
    for (int sys = blockIdx.y; sys < B; sys += gridDim.y) {
        const T *vb = vals + (int64_t)sys * nnz;
        const T *xb = x + (int64_t)sys * x_stride;
        T s = T(0);
        if (staged) {
            for (int base = e0 + tid; base < e1; base += kChunkRows * kStage) {
                int c[kStage];
                T v[kStage];
#pragma unroll
                for (int u = 0; u < kStage; ++u) {
                    const int t = base + kChunkRows * u;
                    if (t < e1) {
                        const int tt = SLA_IDX(t, nnz, kBndEntry);
                        c[u] = __ldg(colind + tt);
                        v[u] = __ldg(vb + tt);
                    }
                }
#pragma unroll
                for (int u = 0; u < kStage; ++u) {
                    const int t = base + kChunkRows * u;
                    if (t < e1) {
                        s_cols[t - e0] = c[u];
                        s_vals[t - e0] = v[u];
                    }
                }
            }
            __syncthreads();
            for (int t = t0; t < t1; t += kStage) {
                T v[kStage], xv[kStage];
#pragma unroll
                for (int u = 0; u < kStage; ++u) {
                    v[u] = T(0);
                    xv[u] = T(0);
                    if (t + u < t1) {
                        v[u] = s_vals[t + u - e0];
                        xv[u] = __ldg(xb + SLA_IDX(s_cols[t + u - e0], x_stride, kBndColumn));
                    }
                }
#pragma unroll
                for (int u = 0; u < kStage; ++u)
                    if (t + u < t1) s += v[u] * xv[u];
            }
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

// ---- pipelined one-thread-row SpMV ----------------------------------------
// A block stays resident and takes the chunks (kChunkRows consecutive rows of
// one system) blockIdx.x, blockIdx.x + gridDim.x, ... .  A chunk's entries are
// one contiguous range of the CSR arrays: its values, columns and row pointers
// are copied into one of kPipe shared-memory stages by 16-byte asynchronous
// copies (cp.async, cached in L2 only), issued one chunk ahead of the chunk
// being summed, so the block's next HBM reads are in flight while it gathers x
// for the current chunk.  Each copied range starts at its first byte rounded
// down to 16 (the arrays start on 16-byte boundaries) and reads nothing past
// the array's end.  A chunk with more entries than a stage holds walks its
// rows in global memory (its row pointers are still staged).  Two stages keep
// three blocks (24 warps) on an SM for rows of 7 in fp64; three stages (two
// chunks ahead) left room for two blocks and measured slower, and so did the
// same pipeline for the value gradient.

constexpr int kPipe = 2;                 // stages: the chunk in flight + the one being summed

__host__ __device__ constexpr int pipe_region(int64_t bytes) {
    return (int)((bytes + 32 + 15) / 16 * 16);   // the range plus both roundings
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Queue the copy of bytes [lo, hi) of an array ending at `end` to shared
// address dst (from lo rounded down to 16); 16 bytes a thread-step, the last
// piece cut at `end` (cp.async fills the rest of it with zeros).
__device__ __forceinline__ void stage_range(uint32_t dst, const void *lo, const void *hi, const void *end,
                                            int tid) {
    const uintptr_t a0 = (uintptr_t)lo & ~(uintptr_t)15;
    const int pieces = (int)(((uintptr_t)hi - a0 + 15) >> 4);
    // pieces before `end` that are whole, and the bytes of the one it cuts
    const uintptr_t room = (uintptr_t)end - a0;
    const int whole = room >= (uintptr_t)pieces * 16 ? pieces : (int)(room >> 4);
    const int cut = (int)(room & 15);
    const char *src = reinterpret_cast<const char *>(a0);
    for (int q = tid; q < pieces; q += kChunkRows)
        cp_async16(dst + 16 * q, src + 16 * q, q < whole ? 16 : cut);
}

// Element offset of p within its 16-byte line.
template <typename E>
__device__ __forceinline__ int line_off(const E *p) {
    return (int)(((uintptr_t)p & 15) / sizeof(E));
}

// Byte sizes of one stage's regions: values (VB bytes an entry), columns, row
// pointers.
struct PipeStage {
    int rv, rc, rr;
    __host__ __device__ PipeStage(int cap, int vb)
        : rv(pipe_region((int64_t)cap * vb)), rc(pipe_region((int64_t)cap * 4)),
          rr(pipe_region((int64_t)(kChunkRows + 1) * 4)) {}
    __host__ __device__ int bytes() const { return rv + rc + rr; }
};

// Queue a chunk's copies (rows from r0, entries [e0, e1), values of its system
// from vb) into the stage at shared address st.
template <typename T>
__device__ __forceinline__ void pipe_issue(uint32_t st, const PipeStage &L, int cap, int n_rows,
                                           int64_t nnz, int r0, int e0, int e1,
                                           const int32_t *__restrict__ rowptr,
                                           const int32_t *__restrict__ colind, const T *vb, int tid) {
    const int r1 = min(n_rows, r0 + kChunkRows);
    stage_range(st + L.rv + L.rc, rowptr + r0, rowptr + r1 + 1, rowptr + n_rows + 1, tid);
    if (e1 - e0 <= cap) {
        stage_range(st, vb + e0, vb + e1, vb + nnz, tid);
        stage_range(st + L.rv, colind + e0, colind + e1, colind + nnz, tid);
    }
}

// y = alpha A x + beta y (one-thread rows), pipelined as above.  Each thread
// sums its row in stored order, like every other one-thread-row kernel.
template <typename T>
__global__ void __launch_bounds__(kChunkRows)
spmv_pipe_kernel(int n_rows, int64_t nnz, int64_t x_stride, int B, const int32_t *__restrict__ rowptr,
                 const int32_t *__restrict__ colind, const T *__restrict__ vals,
                 const T *__restrict__ x, T *__restrict__ y, T alpha, T beta, int cap) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int tid = threadIdx.x;
    const PipeStage L(cap, (int)sizeof(T));
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem_raw);
    const int nchunks = (n_rows + kChunkRows - 1) / kChunkRows;
    const int units = nchunks * B;     // below 2^31 (checked by the caller)
    const int G = gridDim.x;
    const int mine = (int)blockIdx.x < units ? (units - (int)blockIdx.x + G - 1) / G : 0;
    // system and first row of unit u (no division for one system)
    auto unit = [&](int u, int &sys, int &r0) {
        if (B == 1) {
            sys = 0;
            r0 = u * kChunkRows;
        } else {
            sys = (int)((unsigned)u / (unsigned)nchunks);
            r0 = (u - sys * nchunks) * kChunkRows;
        }
    };
    // entry range of my k-th chunk (read one iteration before its copy is queued)
    auto range = [&](int k, int &e0, int &e1) {
        if (k >= mine) return;
        int sys, r0;
        unit((int)blockIdx.x + k * G, sys, r0);
        e0 = SLA_IDX(__ldg(rowptr + r0), nnz + 1, kBndEntry);
        e1 = SLA_IDX(__ldg(rowptr + min(n_rows, r0 + kChunkRows)), nnz + 1, kBndEntry);
    };
    auto issue = [&](int k, int e0, int e1) {
        if (k >= mine) return;
        int sys, r0;
        unit((int)blockIdx.x + k * G, sys, r0);
        pipe_issue<T>(sbase + (k % kPipe) * L.bytes(), L, cap, n_rows, nnz, r0, e0, e1, rowptr, colind,
                      vals + (int64_t)sys * nnz, tid);
    };
    int ne0 = 0, ne1 = 0;
#pragma unroll
    for (int k = 0; k < kPipe - 1; ++k) {
        range(k, ne0, ne1);
        issue(k, ne0, ne1);
        cp_async_commit();
    }
    range(kPipe - 1, ne0, ne1);
    for (int j = 0; j < mine; ++j) {
        cp_async_wait<kPipe - 2>();   // chunk j's copies (this thread's) have landed
        __syncthreads();              // everyone's have; chunk j - 1's stage is free
        issue(j + kPipe - 1, ne0, ne1);
        cp_async_commit();
        range(j + kPipe, ne0, ne1);
        int sys, r0;
        unit((int)blockIdx.x + j * G, sys, r0);
        const int r1 = min(n_rows, r0 + kChunkRows), i = r0 + tid;
        unsigned char *stage = smem_raw + (j % kPipe) * L.bytes();
        const int32_t *srp = reinterpret_cast<const int32_t *>(stage + L.rv + L.rc) + line_off(rowptr + r0);
        const int e0 = srp[0], e1 = srp[r1 - r0];
        const T *vb = vals + (int64_t)sys * nnz;
        const T *xb = x + (int64_t)sys * x_stride;
        if (i >= r1) continue;
        const int t0 = srp[tid], t1 = srp[tid + 1];
        T s = T(0);
        if (e1 - e0 <= cap) {
            const T *sv = reinterpret_cast<const T *>(stage) + line_off(vb + e0) - e0;
            const int32_t *sc = reinterpret_cast<const int32_t *>(stage + L.rv) + line_off(colind + e0) - e0;
            for (int t = t0; t < t1; t += kStage) {
                T v[kStage], xv[kStage];
#pragma unroll
                for (int u2 = 0; u2 < kStage; ++u2) {
                    v[u2] = T(0);
                    xv[u2] = T(0);
                    if (t + u2 < t1) {
                        const int q = SLA_IDX(t + u2 - e0, cap + 4, kBndLocal) + e0;
                        v[u2] = sv[q];
                        xv[u2] = __ldg(xb + SLA_IDX(sc[q], x_stride, kBndColumn));
                    }
                }
#pragma unroll
                for (int u2 = 0; u2 < kStage; ++u2)
                    if (t + u2 < t1) s += v[u2] * xv[u2];
            }
        } else {
            for (int t = t0; t < t1; ++t) {
                const int tt = SLA_IDX(t, nnz, kBndEntry);
                s += __ldg(vb + tt) * __ldg(xb + SLA_IDX(__ldg(colind + tt), x_stride, kBndColumn));
            }
        }
        T *yb = y + (int64_t)sys * n_rows;
        yb[i] = (beta == T(0)) ? alpha * s : alpha * s + beta * yb[i];
    }
    cp_async_wait<0>();
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
            const T p = mul_rn(li, __ldg(xb + SLA_IDX(__ldg(colind + tt), n_cols, kBndColumn)));
            const T g = NEG ? -p : p;
            gb[tt] = accumulate ? gb[tt] + g : g;
        }
    }
}

// The same for one-thread rows, a warp per 32 rows: each lane marks the
// warp's table slots of its row with its lane, then the warp walks the entry
// range in order, so column reads and gradient stores are coalesced (loads of
// a group of kStage steps in registers before any is used).  Each entry is the
// same single product as above.
template <typename T, bool NEG>
__global__ void __launch_bounds__(kWarpRows * kRowWarps)
grad_warp_kernel(int n_rows, int n_cols, int64_t nnz, int B, const int32_t *__restrict__ rowptr,
                 const int32_t *__restrict__ colind, const T *__restrict__ lam,
                 const T *__restrict__ x, T *__restrict__ grad, int accumulate, int cap) {
    extern __shared__ uint8_t s_all[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint8_t *s_row = s_all + (size_t)warp * cap;   // [cap]: lane (row) of each entry
    const int r0 = (blockIdx.x * kRowWarps + warp) * kWarpRows;
    if (r0 >= n_rows) return;
    const int r1 = min(n_rows, r0 + kWarpRows);
    const int i = r0 + lane;
    const int t0 = i < r1 ? __ldg(rowptr + i) : 0, t1 = i < r1 ? __ldg(rowptr + i + 1) : 0;
    const int e0 = __ldg(rowptr + r0), e1 = __ldg(rowptr + r1);
    const bool staged = e1 - e0 <= cap;
    if (staged) {
        for (int t = t0; t < t1; ++t) s_row[t - e0] = (uint8_t)lane;
        __syncwarp();
    }
    for (int sys = blockIdx.y; sys < B; sys += gridDim.y) {
        const T *lb = lam + (int64_t)sys * n_rows + r0;
        const T *xb = x + (int64_t)sys * n_cols;
        T *gb = grad + (int64_t)sys * nnz;
        if (staged) {
            for (int base = e0 + lane; base < e1; base += 32 * kGradStage) {
                int c[kGradStage];
                T li[kGradStage], xv[kGradStage], old[kGradStage];
#pragma unroll
                for (int u = 0; u < kGradStage; ++u) {
                    const int t = base + 32 * u;
                    c[u] = 0;
                    li[u] = T(0);
                    old[u] = T(0);
                    if (t < e1) {
                        const int tt = SLA_IDX(t, nnz, kBndEntry);
                        c[u] = SLA_IDX(__ldg(colind + tt), n_cols, kBndColumn);
                        li[u] = __ldg(lb + s_row[t - e0]);
                        if (accumulate) old[u] = gb[tt];
                    }
                }
#pragma unroll
                for (int u = 0; u < kGradStage; ++u) xv[u] = base + 32 * u < e1 ? __ldg(xb + c[u]) : T(0);
#pragma unroll
                for (int u = 0; u < kGradStage; ++u) {
                    const int t = base + 32 * u;
                    if (t < e1) {
                        const T p = mul_rn(li[u], xv[u]);   // rounded on its own, never fused
                        const T g = NEG ? -p : p;
                        gb[t] = accumulate ? old[u] + g : g;
                    }
                }
            }
        } else if (i < r1) {
            const T l = __ldg(lb + lane);
            for (int t = t0; t < t1; ++t) {
                const int tt = SLA_IDX(t, nnz, kBndEntry);
                const T p = mul_rn(l, __ldg(xb + SLA_IDX(__ldg(colind + tt), n_cols, kBndColumn)));
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

static bool aligned16(const void *p) { return ((uintptr_t)p & 15) == 0; }

// The pipelined SpMV needs 16-byte aligned pattern arrays and per-system value
// arrays; SLA_SPMV_PIPE=0 turns it off.
static bool pipe_ok(const Csr *h, const void *vals) {
    const char *e = getenv("SLA_SPMV_PIPE");
    if ((e && e[0] == '0') || !aligned16(h->rowptr) || !aligned16(h->colind)) return false;
    if ((int64_t)((h->n_rows + kChunkRows - 1) / kChunkRows) * h->batch >= INT32_MAX) return false;
    return aligned16(vals) && (h->batch == 1 || (h->nnz * (int64_t)dtype_size(h->dtype)) % 16 == 0);
}

// Resident blocks of the pipelined kernel: SMs x blocks an SM holds with
// `smem` bytes each (computed on first use and kept in the handle).
template <typename K>
static sla_status pipe_grid(K kernel, size_t smem, int32_t *cached, int *out) {
    if (*cached == 0) {
        SLA_CHECK_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        int per_sm = 0, dev = 0, sms = 0;
        SLA_CHECK_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kChunkRows, smem));
        SLA_CHECK_CUDA(cudaGetDevice(&dev));
        SLA_CHECK_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
        SLA_REQUIRE(per_sm > 0, "pipelined kernel: %zu bytes of shared memory do not fit an SM", smem);
        *cached = per_sm * sms;
    }
    *out = *cached;
    return SLA_OK;
}

static int pipe_blocks(int grid, int rows, int B) {
    const int64_t units = (int64_t)((rows + kChunkRows - 1) / kChunkRows) * B;
    return (int)(units < grid ? units : grid);
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
        const dim3 grid = warp_grid(h->n_rows, h->batch);
        const int cap = warp_cap(h->row_mean);
        const size_t smem = (size_t)cap * kRowWarps;
        if (h->dtype == SLA_F64)
            grad_warp_kernel<double, NEG><<<grid, kWarpRows * kRowWarps, smem, s>>>(
                h->n_rows, h->n_cols, h->nnz, h->batch, h->rowptr, h->colind, (const double *)u,
                (const double *)x, (double *)grad, accumulate, cap);
        else
            grad_warp_kernel<float, NEG><<<grid, kWarpRows * kRowWarps, smem, s>>>(
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
    if (!use_perm && lanes == 1 && pipe_ok(h, vals)) {
        const int cap = chunk_cap(h->row_mean);
        const size_t smem = (size_t)kPipe * PipeStage(cap, (int)dtype_size(h->dtype)).bytes();
        int grid = 0;
        const sla_status st = h->dtype == SLA_F64
                                  ? pipe_grid(spmv_pipe_kernel<double>, smem, &h->pipe_grid_spmv, &grid)
                                  : pipe_grid(spmv_pipe_kernel<float>, smem, &h->pipe_grid_spmv, &grid);
        if (st != SLA_OK) return st;
        if (h->dtype == SLA_F64)
            spmv_pipe_kernel<double><<<pipe_blocks(grid, rows, h->batch), kChunkRows, smem, s>>>(
                rows, h->nnz, xlen, h->batch, rp, ci, (const double *)vals, (const double *)x, (double *)y,
                alpha, beta, cap);
        else
            spmv_pipe_kernel<float><<<pipe_blocks(grid, rows, h->batch), kChunkRows, smem, s>>>(
                rows, h->nnz, xlen, h->batch, rp, ci, (const float *)vals, (const float *)x, (float *)y,
                (float)alpha, (float)beta, cap);
        SLA_CHECK_LAUNCH();
        return SLA_OK;
    }
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
