// Row-parallel building blocks: one row of a CSR matrix times a vector, with
// LANES threads of a warp cooperating on the row (LANES in 1..32, a power of
// two), and one row of the sliced layout times a vector (plain, as
// value-and-column records, or forming the CG direction while gathering).
// Matrix arrays are read through the read-only path; the vector is read with
// plain loads because the persistent solver rewrites it between phases.
#pragma once

#include <type_traits>

#include "sla_common.cuh"

namespace sla {

template <int LANES>
__device__ __forceinline__ unsigned subwarp_mask() {
    if constexpr (LANES == 32) {
        return 0xffffffffu;
    } else {
        const unsigned base = (threadIdx.x & 31) & ~(LANES - 1);
        return ((1u << LANES) - 1u) << base;
    }
}

// sum_{t in row i} vals[t] * v[colind[t]]; lane in [0, LANES).  With LANES > 1
// the partial sums are combined by a fixed xor tree, so the result is
// deterministic and identical on every lane of the sub-warp.  ncols (the length
// of v) and nent (of vals and colind) bound the indices in the bounds-checking
// build and are unused otherwise.
template <typename T, int LANES>
__device__ __forceinline__ T row_dot(const int32_t *__restrict__ rowptr,
                                     const int32_t *__restrict__ colind,
                                     const T *__restrict__ vals, const T *v, int i,
                                     int lane, int ncols, int64_t nent) {
    const int t0 = __ldg(rowptr + i), t1 = __ldg(rowptr + i + 1);
    T s = T(0);
    for (int t = t0 + lane; t < t1; t += LANES) {
        const int tt = SLA_IDX(t, nent, kBndEntry);
        s += __ldg(vals + tt) * v[SLA_IDX(__ldg(colind + tt), ncols, kBndColumn)];
    }
    if constexpr (LANES > 1) {
        const unsigned m = subwarp_mask<LANES>();
#pragma unroll
        for (int o = LANES / 2; o > 0; o >>= 1) s += __shfl_xor_sync(m, s, o, LANES);
    }
    return s;
}

// Same product with every array in shared memory (plain loads).
template <typename T, int LANES>
__device__ __forceinline__ T row_dot_shared(const int32_t *rowptr, const int32_t *colind,
                                            const T *vals, const T *v, int i, int lane,
                                            int ncols, int64_t nent) {
    const int t0 = rowptr[i], t1 = rowptr[i + 1];
    T s = T(0);
    for (int t = t0 + lane; t < t1; t += LANES) {
        const int tt = SLA_IDX(t, nent, kBndLocal);
        s += vals[tt] * v[SLA_IDX(colind[tt], ncols, kBndLocal)];
    }
    if constexpr (LANES > 1) {
        const unsigned m = subwarp_mask<LANES>();
#pragma unroll
        for (int o = LANES / 2; o > 0; o >>= 1) s += __shfl_xor_sync(m, s, o, LANES);
    }
    return s;
}

// Same with the values reached through a permutation (A^T's entry s is A's
// entry perm[s]); used by transposed SpMV on non-symmetric handles.
template <typename T, int LANES>
__device__ __forceinline__ T row_dot_perm(const int32_t *__restrict__ rowptr,
                                          const int32_t *__restrict__ colind,
                                          const int32_t *__restrict__ perm,
                                          const T *__restrict__ vals, const T *v, int i,
                                          int lane, int ncols, int64_t nent) {
    const int t0 = __ldg(rowptr + i), t1 = __ldg(rowptr + i + 1);
    T s = T(0);
    for (int t = t0 + lane; t < t1; t += LANES) {
        const int tt = SLA_IDX(t, nent, kBndEntry);
        s += __ldg(vals + SLA_IDX(__ldg(perm + tt), nent, kBndEntry)) *
             v[SLA_IDX(__ldg(colind + tt), ncols, kBndColumn)];
    }
    if constexpr (LANES > 1) {
        const unsigned m = subwarp_mask<LANES>();
#pragma unroll
        for (int o = LANES / 2; o > 0; o >>= 1) s += __shfl_xor_sync(m, s, o, LANES);
    }
    return s;
}

// Loads of the sliced layout's entries: MODE 0 is the default allocating
// read-only load (where the matrix stays in L2, a slice step uses half a
// 128-byte line and the next step the other half); MODE 1 is
// ld.global.nc.L1::no_allocate, for the solver whose vectors live in HBM: the
// matrix streams through once per iteration and L1 is better left to the
// gathered vector.  (L2 evict-first and 256-byte prefetch-size hints, and a
// bulk L2 prefetch of the tile's next rows, measured no faster.)
template <int MODE, typename T>
__device__ __forceinline__ T sell_load(const T *p) {
    static_assert(sizeof(T) == 4 || sizeof(T) == 8, "4- or 8-byte entries");
    if constexpr (MODE == 0) {
        return __ldg(p);
    } else if constexpr (sizeof(T) == 8) {
        double v;
        asm volatile("ld.global.nc.L1::no_allocate.f64 %0, [%1];" : "=d"(v) : "l"(p));
        return (T)v;
    } else if constexpr (std::is_same<T, float>::value) {
        float v;
        asm volatile("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(v) : "l"(p));
        return v;
    } else {
        int v;
        asm volatile("ld.global.nc.L1::no_allocate.s32 %0, [%1];" : "=r"(v) : "l"(p));
        return (T)v;
    }
}

// A column stored as a 16-bit offset from its row (the sliced layout's
// compact columns), loaded like sell_load's MODE and sign-extended.
template <int MODE>
__device__ __forceinline__ int sell_load_d16(const int16_t *p) {
    short v;
    if constexpr (MODE == 0)
        v = __ldg(p);
    else
        asm volatile("ld.global.nc.L1::no_allocate.s16 %0, [%1];" : "=h"(v) : "l"(p));
    return (int)v;
}

// First slot and width of row i's slice: computed when every slice has the
// same width uw (no load), else read from the slice offsets.
__device__ __forceinline__ void sell_slice(const int32_t *__restrict__ sptr, int i, int uw, int &base,
                                           int &w) {
    const int sl = i / kSellRows;
    int b0;
    if (uw > 0) {
        b0 = sl * kSellRows * uw;
        w = uw;
    } else {
        b0 = __ldg(sptr + sl);
        w = (__ldg(sptr + sl + 1) - b0) / kSellRows;
    }
    base = b0 + i % kSellRows;
}

// Row i of the sliced layout (see sla_sell.cu) times v, one thread per row:
// the row's entries in stored order, then the slice's zero padding (which adds
// nothing), so the sum equals row_dot<T, 1>.  One row at a time per thread:
// interleaving a thread's rows spreads its gathers of v and measured slower,
// and so did loading a row's values and columns into registers before
// gathering (the registers spill at the solver's 64-register budget).  For
// uniform widths of 5 and 7 the solvers use sell_row_w below, which loads only
// the next row's column offsets ahead.  uw > 0: every slice is
// uw wide (no slice offsets read).  i is the row's position in the layout and
// row the row itself (they differ when windows are sorted); with D16 the
// columns come from d16 as offsets from row, else from cols.
template <int STREAM, bool D16, typename T>
__device__ __forceinline__ T sell_row(const int32_t *__restrict__ sptr,
                                      const int32_t *__restrict__ cols, const int16_t *__restrict__ d16,
                                      const T *__restrict__ vals, const T *v, int i, int row,
                                      int ncols, int64_t nslots, int uw) {
    int base, w;
    sell_slice(sptr, i, uw, base, w);
    T s = T(0);
    for (int k = 0; k < w; ++k) {
        const int t = SLA_IDX(base + k * kSellRows, nslots, kBndEntry);
        const int c = D16 ? row + sell_load_d16<STREAM>(d16 + t) : sell_load<STREAM>(cols + t);
        s += sell_load<STREAM>(vals + t) * v[SLA_IDX(c, ncols, kBndColumn)];
    }
    return s;
}

// Rows of a sliced layout whose slices are all W wide, with 16-bit columns,
// for a thread that walks several rows: sell_d16_fetch loads a row's column
// offsets ahead of time, so that while one row's values and gathers are in
// flight the next row's offsets are too, and a row waits for one dependent
// load (its gathers) instead of two.  sell_row_w sums the row as sell_row does
// (stored order, the padding adds zeros), so results are bit-identical.
template <int W, int STREAM = 0>
__device__ __forceinline__ void sell_d16_fetch(const int16_t *__restrict__ d16, int i, int64_t nslots,
                                               int (&d)[W]) {
    const int base = (i / kSellRows) * kSellRows * W + i % kSellRows;
#pragma unroll
    for (int k = 0; k < W; ++k)
        d[k] = sell_load_d16<STREAM>(d16 + SLA_IDX(base + k * kSellRows, nslots, kBndEntry));
}

template <int W, int STREAM = 0, typename T>
__device__ __forceinline__ T sell_row_w(const T *__restrict__ vals, const T *v, const int (&d)[W], int i,
                                        int row, int ncols, int64_t nslots) {
    const int base = (i / kSellRows) * kSellRows * W + i % kSellRows;
    T s = T(0);
#pragma unroll
    for (int k = 0; k < W; ++k) {
        const int t = SLA_IDX(base + k * kSellRows, nslots, kBndEntry);
        s += sell_load<STREAM>(vals + t) * v[SLA_IDX(row + d[k], ncols, kBndColumn)];
    }
    return s;
}

// sell_row_dir for slices W wide with the row's column offsets already loaded.
template <int W, typename T>
__device__ __forceinline__ T sell_row_dir_w(const T *__restrict__ vals, const T *z, const T *pprev, T beta,
                                            const int (&d)[W], int i, int ncols, int64_t nslots) {
    const int base = (i / kSellRows) * kSellRows * W + i % kSellRows;
    T s = T(0);
#pragma unroll
    for (int k = 0; k < W; ++k) {
        const int t = SLA_IDX(base + k * kSellRows, nslots, kBndEntry);
        const int c = SLA_IDX(i + d[k], ncols, kBndColumn);
        T pj;
        if constexpr (sizeof(T) == 8) pj = __fma_rn(beta, pprev[c], z[c]);
        else pj = __fmaf_rn(beta, pprev[c], z[c]);
        s += __ldg(vals + t) * pj;
    }
    return s;
}

// A slot of the sliced layout with its value and column in one record, so
// that one vector load brings both: 8 bytes for fp32, 16 (4 of padding) for fp64.
template <typename T> struct SellRec;
template <> struct __align__(16) SellRec<double> { double v; int32_t c, pad; };
template <> struct __align__(8) SellRec<float> { float v; int32_t c; };

template <int STREAM, typename T>
__device__ __forceinline__ void sell_rec_load(const SellRec<T> *p, T &v, int &c) {
    if constexpr (sizeof(T) == 8) {
        int4 u;
        if constexpr (STREAM)
            asm volatile("ld.global.nc.L1::no_allocate.v4.s32 {%0,%1,%2,%3}, [%4];"
                         : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "l"(p));
        else
            u = __ldg(reinterpret_cast<const int4 *>(p));
        v = __hiloint2double(u.y, u.x);
        c = u.z;
    } else {
        int2 u;
        if constexpr (STREAM)
            asm volatile("ld.global.nc.L1::no_allocate.v2.s32 {%0,%1}, [%2];" : "=r"(u.x), "=r"(u.y) : "l"(p));
        else
            u = __ldg(reinterpret_cast<const int2 *>(p));
        v = __int_as_float(u.x);
        c = u.y;
    }
}

// sell_row over packed records: same entries, order and rounding.
template <int STREAM, typename T>
__device__ __forceinline__ T sell_row_rec(const int32_t *__restrict__ sptr, const SellRec<T> *__restrict__ rec,
                                          const T *v, int i, int ncols, int64_t nslots) {
    const int sl = i / kSellRows;
    const int b0 = __ldg(sptr + sl);
    const int w = (__ldg(sptr + sl + 1) - b0) / kSellRows;
    const int base = b0 + i % kSellRows;
    T s = T(0);
    for (int k = 0; k < w; ++k) {
        T a;
        int c;
        sell_rec_load<STREAM>(rec + SLA_IDX(base + k * kSellRows, nslots, kBndEntry), a, c);
        s += a * v[SLA_IDX(c, ncols, kBndColumn)];
    }
    return s;
}

// Row of the sliced layout times the direction p_k = z + beta p_prev, formed
// per gathered entry with one fused multiply-add (the owner of each row forms
// the same value the same way from its own M^-1 r, rounded once, as z).
template <bool D16, typename T>
__device__ __forceinline__ T sell_row_dir(const int32_t *__restrict__ sptr,
                                          const int32_t *__restrict__ cols, const int16_t *__restrict__ d16,
                                          const T *__restrict__ vals, const T *z, const T *pprev,
                                          T beta, int i, int ncols, int64_t nslots, int uw) {
    int base, w;
    sell_slice(sptr, i, uw, base, w);
    T s = T(0);
    for (int k = 0; k < w; ++k) {
        const int t = SLA_IDX(base + k * kSellRows, nslots, kBndEntry);
        const int c = SLA_IDX(D16 ? i + sell_load_d16<0>(d16 + t) : __ldg(cols + t), ncols, kBndColumn);
        T pj;
        if constexpr (sizeof(T) == 8) pj = __fma_rn(beta, pprev[c], z[c]);
        else pj = __fmaf_rn(beta, pprev[c], z[c]);
        s += __ldg(vals + t) * pj;
    }
    return s;
}

// Dispatch a functor templated on LANES.
template <typename F>
sla_status with_lanes(int lanes, F &&f) {
    switch (lanes) {
        case 1: return f(std::integral_constant<int, 1>{});
        case 2: return f(std::integral_constant<int, 2>{});
        case 4: return f(std::integral_constant<int, 4>{});
        case 8: return f(std::integral_constant<int, 8>{});
        case 16: return f(std::integral_constant<int, 16>{});
        default: return f(std::integral_constant<int, 32>{});
    }
}

}  // namespace sla
