// Edge-weighted graph Laplacian on a handle's pattern and its chain rule: the
// conductivity-to-matrix map of inverse coefficient learning (torch-sla summary
// page, technical summary, "Experimental results", end-to-end application).
//
//   A_ij = A_ji = -w_e per edge e = (i, j);  A_ii = (w of i's edges, added
//   from 0 in ascending neighbour index) + shift;  other entries 0.
//   dL/dw_e = ((G_ii + G_jj) - G_ij) - G_ji;  dL/dshift = sum_i G_ii.
//
// The plan maps every pattern entry to the edge whose weight it carries
// (emap, -1 for none) and every edge to its two entries, once.  Assembly runs
// one thread per (system, row) and walks the row in stored order, so the
// diagonal is the same ordered sum the definition states.  The gradients run
// one thread per (system, edge); the shift gradient is a per-system sum in
// double over a fixed tree (tile partials, then one block per system).
#include "sla_common.cuh"

namespace sla {

namespace {

struct Edges {
    Csr *h = nullptr;
    int64_t E = 0;
    int32_t *ei = nullptr, *ej = nullptr;     // owned copies [E]
    int32_t *sij = nullptr, *sji = nullptr;   // owned [E]: positions of (i, j) and (j, i)
    int32_t *emap = nullptr;                  // owned [nnz]: edge of each entry, -1 for none
    int32_t ntiles = 0;                       // row tiles of the shift-gradient sum
};

constexpr int kEdgeThreads = 256;
constexpr int kSumRows = 4096;                // rows a block adds up for the shift gradient
constexpr int kNoEdge = 0x7fffffff;

__device__ __forceinline__ void report(unsigned long long *err, unsigned long long code, int64_t at) {
    atomicMin(err, (code << 40) | (unsigned long long)at);
}

// Position of column c in row r (columns strictly increasing), -1 if absent.
__device__ __forceinline__ int find_entry(const int32_t *rowptr, const int32_t *colind, int r, int c) {
    int lo = __ldg(rowptr + r), hi = __ldg(rowptr + r + 1) - 1;
    while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        const int v = __ldg(colind + mid);
        if (v == c) return mid;
        if (v < c) lo = mid + 1;
        else hi = mid - 1;
    }
    return -1;
}

__global__ void emap_fill_kernel(int64_t nnz, int32_t *emap) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t < nnz) emap[t] = kNoEdge;
}

// Endpoints, self loops and missing entries; surviving edges claim their two
// entries with atomicMin, so the smallest edge naming a pair owns it.
__global__ void edge_claim_kernel(int n, const int32_t *rowptr, const int32_t *colind, int64_t E,
                                  const int32_t *ei, const int32_t *ej, int32_t *sij, int32_t *sji,
                                  int32_t *emap, unsigned long long *err) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const int i = __ldg(ei + e), j = __ldg(ej + e);
    int a = -1, b = -1;
    if (i < 0 || i >= n || j < 0 || j >= n) {
        report(err, 1, e);
    } else if (i == j) {
        report(err, 2, e);
    } else {
        a = find_entry(rowptr, colind, i, j);
        b = find_entry(rowptr, colind, j, i);
        if (a < 0 || b < 0) {
            report(err, 3, e);
            a = b = -1;
        } else {
            atomicMin(emap + a, (int)e);
            atomicMin(emap + b, (int)e);
        }
    }
    sij[e] = a;
    sji[e] = b;
}

// An edge that does not own its entries repeats an earlier edge's pair.
__global__ void edge_dup_kernel(int64_t E, const int32_t *sij, const int32_t *sji,
                                const int32_t *emap, unsigned long long *err) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const int a = sij[e], b = sji[e];
    if (a >= 0 && (emap[a] != (int)e || emap[b] != (int)e)) report(err, 4, e);
}

__global__ void edge_diag_kernel(int n, const int32_t *diagpos, unsigned long long *err) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n && diagpos[i] < 0) report(err, 5, i);
}

__global__ void emap_finish_kernel(int64_t nnz, int32_t *emap) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t < nnz && emap[t] == kNoEdge) emap[t] = -1;
}

// One thread per (system, row): the row's entries in stored order.
template <typename T>
__global__ void __launch_bounds__(kEdgeThreads)
assemble_kernel(int n, int64_t nnz, int B, int64_t E, const int32_t *__restrict__ rowptr,
                const int32_t *__restrict__ colind, const int32_t *__restrict__ emap,
                const T *__restrict__ w, const T *__restrict__ shift, T *__restrict__ vals) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= (int64_t)n * B) return;
    const int b = (int)(g / n), i = (int)(g % n);
    const T *wb = w + (int64_t)b * E;
    T *vb = vals + (int64_t)b * nnz;
    const int t0 = __ldg(rowptr + i), t1 = __ldg(rowptr + i + 1);
    T d = T(0);
    int dpos = -1;
    for (int t = t0; t < t1; ++t) {
        const int e = __ldg(emap + t);
        if (e >= 0) {
            const T we = __ldg(wb + SLA_IDX(e, E, kBndEdge));
            vb[t] = -we;
            d = d + we;
        } else if (__ldg(colind + t) == i) {
            dpos = t;
        } else {
            vb[t] = T(0);
        }
    }
    if (dpos >= 0) vb[dpos] = d + (shift ? __ldg(shift + b) : T(0));
}

template <typename T>
__device__ __forceinline__ T neg_prod(T a, T b) {
    if constexpr (sizeof(T) == 8) return -__dmul_rn(a, b);
    else return -__fmul_rn(a, b);
}

// dw for edges [blockIdx.x * kEdgeThreads, ...) of system blockIdx.y, from G
// (FROM_G) or from lambda and x (each G entry formed as -(lambda_i * x_j)).
template <typename T, bool FROM_G>
__global__ void __launch_bounds__(kEdgeThreads)
edge_grad_kernel(int n, int64_t nnz, int64_t E, const int32_t *__restrict__ ei,
                 const int32_t *__restrict__ ej, const int32_t *__restrict__ sij,
                 const int32_t *__restrict__ sji, const int32_t *__restrict__ diagpos,
                 const T *__restrict__ G, const T *__restrict__ lam, const T *__restrict__ x,
                 T *__restrict__ dw, int accumulate) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const int b = blockIdx.y;
    const int i = SLA_IDX(__ldg(ei + e), n, kBndEdge), j = SLA_IDX(__ldg(ej + e), n, kBndEdge);
    T gii, gjj, gij, gji;
    if constexpr (FROM_G) {
        const T *gb = G + (int64_t)b * nnz;
        gii = __ldg(gb + SLA_IDX(__ldg(diagpos + i), nnz, kBndDiag));
        gjj = __ldg(gb + SLA_IDX(__ldg(diagpos + j), nnz, kBndDiag));
        gij = __ldg(gb + SLA_IDX(__ldg(sij + e), nnz, kBndEdge));
        gji = __ldg(gb + SLA_IDX(__ldg(sji + e), nnz, kBndEdge));
    } else {
        const T *lb = lam + (int64_t)b * n, *xb = x + (int64_t)b * n;
        const T li = __ldg(lb + i), lj = __ldg(lb + j), xi = __ldg(xb + i), xj = __ldg(xb + j);
        gii = neg_prod(li, xi);
        gjj = neg_prod(lj, xj);
        gij = neg_prod(li, xj);
        gji = neg_prod(lj, xi);
    }
    const T v = ((gii + gjj) - gij) - gji;
    T *out = dw + (int64_t)b * E + e;
    *out = accumulate ? *out + v : v;
}

// Tile partials of sum_i G_ii (in double) for system blockIdx.y.
template <typename T, bool FROM_G>
__global__ void __launch_bounds__(kEdgeThreads)
diag_partial_kernel(int n, int64_t nnz, int ntiles, const int32_t *__restrict__ diagpos,
                    const T *__restrict__ G, const T *__restrict__ lam, const T *__restrict__ x,
                    double *__restrict__ part) {
    __shared__ double red[33];
    const int b = blockIdx.y;
    const int r0 = blockIdx.x * kSumRows, r1 = min(n, r0 + kSumRows);
    double s = 0.0;
    for (int i = r0 + threadIdx.x; i < r1; i += kEdgeThreads) {
        if constexpr (FROM_G) {
            s += (double)__ldg(G + (int64_t)b * nnz + SLA_IDX(__ldg(diagpos + i), nnz, kBndDiag));
        } else {
            const int64_t o = (int64_t)b * n + i;
            s += (double)neg_prod(__ldg(lam + o), __ldg(x + o));
        }
    }
    s = block_sum<kEdgeThreads>(s, red);
    if (threadIdx.x == 0) part[(int64_t)b * ntiles + blockIdx.x] = s;
}

// dshift[b] = the sum of block b's `count` partials (a fixed tree); with one
// block over all B * ntiles partials this is the shared shift's gradient.
template <typename T>
__global__ void __launch_bounds__(kEdgeThreads)
diag_finish_kernel(int64_t count, const double *__restrict__ part, T *__restrict__ dshift,
                   int accumulate) {
    __shared__ double red[33];
    const int b = blockIdx.x;
    double s = 0.0;
    for (int64_t t = threadIdx.x; t < count; t += kEdgeThreads) s += part[(int64_t)b * count + t];
    s = block_sum<kEdgeThreads>(s, red);
    if (threadIdx.x == 0) dshift[b] = accumulate ? dshift[b] + (T)s : (T)s;
}

unsigned grid_of(int64_t count) { return (unsigned)((count + kEdgeThreads - 1) / kEdgeThreads); }

template <typename T, bool FROM_G>
sla_status edge_grad(const Edges *p, const T *G, const T *lam, const T *x, T *dw, T *dshift,
                     int flags, void *ws, size_t ws_bytes, cudaStream_t s) {
    const int accumulate = (flags & SLA_GRAD_ACCUMULATE) != 0;
    const bool shared = (flags & SLA_GRAD_SHIFT_SHARED) != 0;
    const Csr *h = p->h;
    const int B = h->batch, n = h->n_rows;
    SLA_REQUIRE(B <= 65535, "sla_laplacian_grad: batch %d exceeds 65535", B);
    if (p->E > 0) {
        SLA_REQUIRE(dw != nullptr, "sla_laplacian_grad: NULL dw");
        edge_grad_kernel<T, FROM_G><<<dim3(grid_of(p->E), B), kEdgeThreads, 0, s>>>(
            n, h->nnz, p->E, p->ei, p->ej, p->sij, p->sji, h->diagpos, G, lam, x, dw, accumulate);
        SLA_CHECK_LAUNCH();
    }
    if (dshift != nullptr) {
        const size_t need = align_up((size_t)B * p->ntiles * sizeof(double));
        SLA_REQUIRE(ws != nullptr && ws_bytes >= need, "sla_laplacian_grad: workspace too small (%zu < %zu)",
                    ws_bytes, need);
        SLA_REQUIRE(((uintptr_t)ws & 255) == 0, "sla_laplacian_grad: workspace must be 256-byte aligned");
        double *part = static_cast<double *>(ws);
        if (p->ntiles > 0) {
            diag_partial_kernel<T, FROM_G><<<dim3(p->ntiles, B), kEdgeThreads, 0, s>>>(
                n, h->nnz, p->ntiles, h->diagpos, G, lam, x, part);
            SLA_CHECK_LAUNCH();
        }
        if (shared)
            diag_finish_kernel<T><<<1, kEdgeThreads, 0, s>>>((int64_t)B * p->ntiles, part, dshift, accumulate);
        else
            diag_finish_kernel<T><<<B, kEdgeThreads, 0, s>>>(p->ntiles, part, dshift, accumulate);
        SLA_CHECK_LAUNCH();
    }
    return SLA_OK;
}

void free_edges(Edges *p) {
    if (!p) return;
    cudaFree(p->ei);
    cudaFree(p->ej);
    cudaFree(p->sij);
    cudaFree(p->sji);
    cudaFree(p->emap);
    delete p;
}

}  // namespace

}  // namespace sla

using namespace sla;

extern "C" sla_status sla_edges_create(sla_csr_t hh, int64_t n_edges, const int32_t *ei,
                                       const int32_t *ej, int64_t *check, void *stream,
                                       sla_edges_t *out) {
    SLA_RANGE("sla_edges_create");
    clear_error();
    if (check) *check = 0;
    SLA_REQUIRE(out != nullptr, "sla_edges_create: NULL out");
    *out = nullptr;
    Csr *h = reinterpret_cast<Csr *>(hh);
    SLA_REQUIRE(h != nullptr, "sla_edges_create: NULL handle");
    SLA_REQUIRE(h->n_rows == h->n_cols, "sla_edges_create: matrix must be square (%d x %d)",
                h->n_rows, h->n_cols);
    SLA_REQUIRE(n_edges >= 0 && n_edges < (int64_t)1 << 31, "sla_edges_create: bad edge count %lld",
                (long long)n_edges);
    SLA_REQUIRE(n_edges == 0 || (ei && ej), "sla_edges_create: NULL ei or ej");
    cudaStream_t s = as_stream(stream);
    Edges *p = new Edges();
    p->h = h;
    p->E = n_edges;
    p->ntiles = (h->n_rows + kSumRows - 1) / kSumRows;
    const size_t eb = (size_t)(n_edges > 0 ? n_edges : 1) * sizeof(int32_t);
    unsigned long long *err = nullptr;
    auto fail = [&](sla_status st) {
        cudaFree(err);
        free_edges(p);
        return st;
    };
    if (cudaMalloc(&p->ei, eb) != cudaSuccess || cudaMalloc(&p->ej, eb) != cudaSuccess ||
        cudaMalloc(&p->sij, eb) != cudaSuccess || cudaMalloc(&p->sji, eb) != cudaSuccess ||
        cudaMalloc(&p->emap, (size_t)(h->nnz > 0 ? h->nnz : 1) * sizeof(int32_t)) != cudaSuccess ||
        cudaMalloc(&err, sizeof(unsigned long long)) != cudaSuccess) {
        cudaGetLastError();
        set_error("sla_edges_create: out of device memory");
        return fail(SLA_ERR_OOM);
    }
    if (n_edges > 0) {
        if (cudaMemcpyAsync(p->ei, ei, n_edges * sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(p->ej, ej, n_edges * sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess) {
            set_error("sla_edges_create: copy of the edge list failed");
            return fail(SLA_ERR_CUDA);
        }
    }
    if (cudaMemsetAsync(err, 0xff, sizeof(unsigned long long), s) != cudaSuccess) {
        set_error("sla_edges_create: memset failed");
        return fail(SLA_ERR_CUDA);
    }
    if (h->nnz > 0) emap_fill_kernel<<<grid_of(h->nnz), kEdgeThreads, 0, s>>>(h->nnz, p->emap);
    if (n_edges > 0) {
        edge_claim_kernel<<<grid_of(n_edges), kEdgeThreads, 0, s>>>(
            h->n_rows, h->rowptr, h->colind, n_edges, p->ei, p->ej, p->sij, p->sji, p->emap, err);
        edge_dup_kernel<<<grid_of(n_edges), kEdgeThreads, 0, s>>>(n_edges, p->sij, p->sji, p->emap, err);
    }
    if (h->n_rows > 0) edge_diag_kernel<<<grid_of(h->n_rows), kEdgeThreads, 0, s>>>(h->n_rows, h->diagpos, err);
    if (h->nnz > 0) emap_finish_kernel<<<grid_of(h->nnz), kEdgeThreads, 0, s>>>(h->nnz, p->emap);
    unsigned long long code = 0;
    if (cudaGetLastError() != cudaSuccess ||
        cudaMemcpyAsync(&code, err, sizeof(code), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        set_error("sla_edges_create: edge mapping kernels failed");
        return fail(SLA_ERR_CUDA);
    }
    if (code != ~0ull) {
        static const char *what[] = {"", "endpoint out of range", "self loop",
                                     "entry missing from the pattern", "repeated pair",
                                     "row without a diagonal entry"};
        const int c = (int)(code >> 40);
        const long long at = (long long)(code & ((1ull << 40) - 1));
        if (check) *check = (int64_t)code;
        set_error("sla_edges_create: %s at %s %lld", what[c >= 1 && c <= 5 ? c : 0],
                  c == 5 ? "row" : "edge", at);
        return fail(SLA_ERR_INVALID);
    }
    cudaFree(err);
    *out = reinterpret_cast<sla_edges_t>(p);
    return SLA_OK;
}

extern "C" sla_status sla_edges_destroy(sla_edges_t e) {
    clear_error();
    free_edges(reinterpret_cast<Edges *>(e));
    return SLA_OK;
}

extern "C" sla_status sla_laplacian_assemble(sla_edges_t ee, const void *w, const void *shift,
                                             void *vals, void *stream) {
    SLA_RANGE("sla_laplacian_assemble");
    clear_error();
    const Edges *p = reinterpret_cast<const Edges *>(ee);
    SLA_REQUIRE(p != nullptr, "sla_laplacian_assemble: NULL plan");
    const Csr *h = p->h;
    if (h->n_rows == 0 || h->nnz == 0) return SLA_OK;
    SLA_REQUIRE(vals != nullptr && (w != nullptr || p->E == 0), "sla_laplacian_assemble: NULL w or vals");
    cudaStream_t s = as_stream(stream);
    const unsigned grid = grid_of((int64_t)h->n_rows * h->batch);
    if (h->dtype == SLA_F64)
        assemble_kernel<double><<<grid, kEdgeThreads, 0, s>>>(
            h->n_rows, h->nnz, h->batch, p->E, h->rowptr, h->colind, p->emap, (const double *)w,
            (const double *)shift, (double *)vals);
    else
        assemble_kernel<float><<<grid, kEdgeThreads, 0, s>>>(
            h->n_rows, h->nnz, h->batch, p->E, h->rowptr, h->colind, p->emap, (const float *)w,
            (const float *)shift, (float *)vals);
    SLA_CHECK_LAUNCH();
    return SLA_OK;
}

extern "C" size_t sla_edges_workspace_bytes(sla_edges_t ee) {
    const Edges *p = reinterpret_cast<const Edges *>(ee);
    if (!p) return 0;
    return align_up((size_t)p->h->batch * p->ntiles * sizeof(double));
}

extern "C" sla_status sla_laplacian_grad_values(sla_edges_t ee, const void *G, void *dw, void *dshift,
                                                int32_t flags, void *ws, size_t ws_bytes,
                                                void *stream) {
    SLA_RANGE("sla_laplacian_grad_values");
    clear_error();
    SLA_REQUIRE((flags & ~(int32_t)(SLA_GRAD_ACCUMULATE | SLA_GRAD_SHIFT_SHARED)) == 0,
                "sla_laplacian_grad_values: unknown flags 0x%x", (unsigned)flags);
    const Edges *p = reinterpret_cast<const Edges *>(ee);
    SLA_REQUIRE(p != nullptr, "sla_laplacian_grad_values: NULL plan");
    SLA_REQUIRE(G != nullptr || p->h->nnz == 0, "sla_laplacian_grad_values: NULL G");
    cudaStream_t s = as_stream(stream);
    if (p->h->dtype == SLA_F64)
        return edge_grad<double, true>(p, (const double *)G, nullptr, nullptr, (double *)dw,
                                       (double *)dshift, flags, ws, ws_bytes, s);
    return edge_grad<float, true>(p, (const float *)G, nullptr, nullptr, (float *)dw, (float *)dshift,
                                  flags, ws, ws_bytes, s);
}

extern "C" sla_status sla_laplacian_grad(sla_edges_t ee, const void *lambda, const void *x, void *dw,
                                         void *dshift, int32_t flags, void *ws, size_t ws_bytes,
                                         void *stream) {
    SLA_RANGE("sla_laplacian_grad");
    clear_error();
    SLA_REQUIRE((flags & ~(int32_t)(SLA_GRAD_ACCUMULATE | SLA_GRAD_SHIFT_SHARED)) == 0,
                "sla_laplacian_grad: unknown flags 0x%x", (unsigned)flags);
    const Edges *p = reinterpret_cast<const Edges *>(ee);
    SLA_REQUIRE(p != nullptr, "sla_laplacian_grad: NULL plan");
    SLA_REQUIRE((lambda && x) || p->h->n_rows == 0, "sla_laplacian_grad: NULL lambda or x");
    cudaStream_t s = as_stream(stream);
    if (p->h->dtype == SLA_F64)
        return edge_grad<double, false>(p, nullptr, (const double *)lambda, (const double *)x,
                                        (double *)dw, (double *)dshift, flags, ws, ws_bytes, s);
    return edge_grad<float, false>(p, nullptr, (const float *)lambda, (const float *)x, (float *)dw,
                                   (float *)dshift, flags, ws, ws_bytes, s);
}
