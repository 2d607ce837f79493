// gather_common.cuh -- pieces shared by the CUDA-core gather kernels: base-2
// exponentials, 16-byte row slices, group sums over lanes, and the
// enumeration of a query's neighbour list and of a key's transpose list for
// structured (window + distance links) and CSR graphs.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sa_internal.cuh"

namespace gather {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kWarpsPerBlock = 8;

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <typename T>
struct Slice;

template <>
struct Slice<__nv_bfloat16> {
    static constexpr int V = 8;
    __device__ static void load(const __nv_bfloat16 *p, float *f) {
        uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            f[2 * a] = __uint_as_float(w[a] << 16);
            f[2 * a + 1] = __uint_as_float(w[a] & 0xffff0000u);
        }
    }
    __device__ static void store(__nv_bfloat16 *p, const float *f) {
        uint32_t w[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * a], f[2 * a + 1]);
            w[a] = *reinterpret_cast<uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <>
struct Slice<float> {
    static constexpr int V = 4;
    __device__ static void load(const float *p, float *f) {
        float4 u = __ldg(reinterpret_cast<const float4 *>(p));
        f[0] = u.x;
        f[1] = u.y;
        f[2] = u.z;
        f[3] = u.w;
    }
    __device__ static void store(float *p, const float *f) {
        *reinterpret_cast<float4 *>(p) = make_float4(f[0], f[1], f[2], f[3]);
    }
};

// Sum over the L lanes of a group (L a power of two, groups aligned).
template <int L>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int o = 1; o < L; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// ---- neighbour enumeration -------------------------------------------------

// Forward list of query i: distance links (keys ascending), then the window.
struct RowEdges {
    int64_t deg;
    int64_t lo;       // window start (structured)
    int32_t first;    // first distance index with o <= i (structured)
    int32_t ndil;     // number of distance links (structured)
    int64_t start;    // CSR start
};

__device__ __forceinline__ RowEdges row_edges(const GraphView &g, int64_t i) {
    RowEdges r;
    if (g.kind == 0) {
        int32_t first = 0;
        while (first < g.n_off && g.offs[first] > i) ++first;
        r.first = first;
        r.ndil = g.n_off - first;
        r.lo = i - g.W + 1 < 0 ? 0 : i - g.W + 1;
        r.deg = r.ndil + (i - r.lo + 1);
        r.start = 0;
    } else {
        r.start = g.rowptr[i];
        r.deg = g.rowptr[i + 1] - r.start;
        r.first = r.ndil = 0;
        r.lo = 0;
    }
    return r;
}

__device__ __forceinline__ int64_t row_edge(const GraphView &g, const RowEdges &r, int64_t i,
                                            int64_t e) {
    if (g.kind == 0) {
        if (e < r.ndil) return i - g.offs[r.first + e];
        return r.lo + (e - r.ndil);
    }
    return g.colidx[r.start + e];
}

// Transpose list of key j: window queries j .. j+W-1, then j + o ascending.
struct ColEdges {
    int64_t deg;
    int64_t nwin;
    int64_t start;
};

__device__ __forceinline__ ColEdges col_edges(const GraphView &g, int64_t j) {
    ColEdges c;
    if (g.kind == 0) {
        c.nwin = g.T - j < g.W ? g.T - j : g.W;
        int64_t nd = 0;
        for (int a = 0; a < g.n_off; ++a) nd += (j + g.offs[a] < g.T) ? 1 : 0;
        c.deg = c.nwin + nd;
        c.start = 0;
    } else {
        c.start = g.rev_rowptr[j];
        c.deg = g.rev_rowptr[j + 1] - c.start;
        c.nwin = 0;
    }
    return c;
}

__device__ __forceinline__ int64_t col_edge(const GraphView &g, const ColEdges &c, int64_t j,
                                            int64_t e) {
    if (g.kind == 0) {
        if (e < c.nwin) return j + e;
        return j + g.offs[g.n_off - 1 - (e - c.nwin)];
    }
    return g.rev_colidx[c.start + e];
}

// Key/value slice read by query slice bh (grouped-query attention: query head
// h of batch row b reads key/value head h / (H / Hkv) of the same row).
__device__ __forceinline__ int64_t kv_slice(int64_t bh, int64_t H, int64_t Hkv) {
    return (bh / H) * Hkv + (bh % H) / (H / Hkv);
}

}  // namespace gather
