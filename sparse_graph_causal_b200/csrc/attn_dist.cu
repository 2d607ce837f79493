// attn_dist.cu -- learned-coordinate scoring on the same neighbour graph, on
// CUDA cores.
//
// Page "SpatialLM-Mini sped up training with a 16K context by 2.47x on an RTX
// 3050", section "How tokens choose whom to listen to": the hidden state of a
// token gives a learnable three-dimensional query coordinate a_i and key
// coordinate c_j; the shorter their distance, the higher the weight of the
// edge, while the neighbour list stays fixed.  Here, in its plainest form,
//     s_ij = -scale |a_i - c_j|^2          for j in N(i)
//     out_i = sum_j softmax_j(s_ij) v_j,   lse_i = ln sum_j exp(s_ij).
// A score costs three differences and three FMAs, so there is no contraction
// for the tensor cores: these are gather kernels.  A warp owns one query
// (forward, da) or one key (dc, dv) and walks its list 32 edges at a time in
// two phases:
//  1. lane t takes edge t of the chunk: its key (or query) index, the
//     coordinates, the score and the probability -- once per edge, not once
//     per lane that touches the edge's row;
//  2. the 32 lanes form G groups of L lanes (16 bytes of a row per lane); group
//     g takes edges g, g + G, ... of the chunk, their index and probability
//     fetched from the owning lanes by shuffles, and reads the value (or dO)
//     rows.  Per-edge row dot products (dp) go back to the owning lane.
// The forward's running max is warp-wide (one per chunk), so the groups'
// partial sums merge by plain addition at the end.  Base-2 arithmetic
// inside: s2 = log2(e) s.  Every kernel is bounded to 64 registers, so that
// four 256-thread blocks share an SM: these kernels wait on L2, and the extra
// resident warps hide more of it than the few spilled registers cost.
//
// Backward, probabilities recomputed from lse:
//   Delta_i = dO_i . out_i,   p = exp(s_ij - lse_i),   dp = dO_i . v_j,
//   dS = p (dp - Delta_i),    g = dS (-2 scale) (a_i - c_j):
//   da_i = sum_j g (forward lists),  dc_j = -sum_i g,  dv_j = sum_i p dO_i
//   (transpose lists).  Two kernels with disjoint outputs, no atomics.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gather_common.cuh"

namespace {

using namespace gather;

struct Coord {
    float x, y, z;
};

__device__ __forceinline__ Coord load_coord(const float *p, int64_t row) {
    const float *r = p + row * 3;
    return Coord{__ldg(r), __ldg(r + 1), __ldg(r + 2)};
}

// -scale2 |a - c|^2, scale2 = scale log2(e)
__device__ __forceinline__ float dist_score(const Coord &a, const Coord &c, float nscale2) {
    const float dx = a.x - c.x, dy = a.y - c.y, dz = a.z - c.z;
    return nscale2 * fmaf(dx, dx, fmaf(dy, dy, dz * dz));
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// The structured graph's distances in shared memory, so that the lanes of
// phase 1 read theirs without indexing the kernel parameters per lane.
// Every thread of the block must call it (one barrier).
__device__ __forceinline__ void stage_offsets(const GraphView &g, int64_t *s_offs) {
    if (g.kind == 0 && (int)threadIdx.x < g.n_off) s_offs[threadIdx.x] = g.offs[threadIdx.x];
    __syncthreads();
}

// Key of edge e (< deg) of query i's forward list: as row_edge.
__device__ __forceinline__ int64_t fwd_key(const GraphView &g, const RowEdges &r,
                                           const int64_t *s_offs, int64_t i, int64_t e) {
    if (g.kind == 0) return e < r.ndil ? i - s_offs[r.first + e] : r.lo + (e - r.ndil);
    return g.colidx[r.start + e];
}

// Query of edge e (< deg) of key j's transpose list: as col_edge.
__device__ __forceinline__ int64_t col_query(const GraphView &g, const ColEdges &c,
                                             const int64_t *s_offs, int64_t j, int64_t e) {
    if (g.kind == 0) return e < c.nwin ? j + e : j + s_offs[g.n_off - 1 - (e - c.nwin)];
    return g.rev_colidx[c.start + e];
}

// Phase 2's hand-back of the per-edge dot products: in the step that starts
// at chunk edge u0, group x holds dp of edge u0 + x (all L lanes alike); lane
// t = u0 + x keeps it.  Every lane must call it.
template <int L, int G>
__device__ __forceinline__ void take_dp(float dp, int u0, int lane, float &dpt) {
    const float got = __shfl_sync(0xffffffffu, dp, ((lane - u0) & (G - 1)) * L);
    if (lane >= u0 && lane < u0 + G) dpt = got;
}

template <typename T, int D>
__global__ void __launch_bounds__(256, 4) dist_fwd_kernel(const float *__restrict__ qa,
                                                       const float *__restrict__ kc,
                                                       const T *__restrict__ v, GraphView g,
                                                       float nscale2, T *__restrict__ out,
                                                       float *__restrict__ lse, int64_t ntiles) {
    constexpr int V = Slice<T>::V, L = D / V, G = 32 / L;
    static_assert(L >= 1 && L <= 32 && G * L == 32, "slice layout");
    __shared__ int64_t s_offs[SA_MAX_OFFSETS];
    stage_offsets(g, s_offs);
    const int lane = threadIdx.x & 31, grp = lane / L, sub = lane % L;
    const int64_t bh = blockIdx.x / ntiles;
    const int64_t i = (blockIdx.x % ntiles) * kWarpsPerBlock + (threadIdx.x >> 5);
    const int64_t T_ = g.T;
    if (i >= T_) return;
    const int64_t rbase = bh * T_;
    const Coord a = load_coord(qa, rbase + i);
    const RowEdges r = row_edges(g, i);
    float m = -INFINITY, lpart = 0.f, acc[V];  // lpart: this lane's edges' share of l
#pragma unroll
    for (int x = 0; x < V; ++x) acc[x] = 0.f;
    for (int64_t e0 = 0; e0 < r.deg; e0 += 32) {
        // phase 1: lane t scores edge e0 + t (lanes past the list: row i, p = 0)
        const int64_t e = e0 + lane;
        int64_t j = i;
        float s = -INFINITY;
        if (e < r.deg) {
            j = fwd_key(g, r, s_offs, i, e);
            s = dist_score(a, load_coord(kc, rbase + j), nscale2);
        }
        const float mn = fmaxf(m, warp_max(s));  // finite: lane 0 holds an edge
        const float al = ex2(m - mn);            // 0 on the first chunk
        lpart *= al;
#pragma unroll
        for (int x = 0; x < V; ++x) acc[x] *= al;
        m = mn;
        const float p = ex2(s - mn);
        lpart += p;
        // phase 2: group grp weighs the value rows of edges u0 + grp
        const int n = r.deg - e0 < 32 ? (int)(r.deg - e0) : 32;
#pragma unroll 4
        for (int u0 = 0; u0 < n; u0 += G) {
            const int u = u0 + grp;
            const int64_t ju = __shfl_sync(0xffffffffu, j, u);
            const float pu = __shfl_sync(0xffffffffu, p, u);
            float vf[V];
            Slice<T>::load(v + (rbase + ju) * D + sub * V, vf);
#pragma unroll
            for (int x = 0; x < V; ++x) acc[x] = fmaf(pu, vf[x], acc[x]);
        }
    }
    // the groups share the running max: their sums add
#pragma unroll
    for (int o = L; o < 32; o <<= 1) {
#pragma unroll
        for (int x = 0; x < V; ++x) acc[x] += __shfl_xor_sync(0xffffffffu, acc[x], o);
    }
    const float l = warp_sum(lpart);
    if (grp == 0) {
        float o_[V];
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int x = 0; x < V; ++x) o_[x] = acc[x] * inv;
        Slice<T>::store(out + (rbase + i) * D + sub * V, o_);
        if (sub == 0) lse[rbase + i] = l > 0.f ? (m + lg2(l)) * kLn2 : -INFINITY;
    }
}

// da_i (and Delta_i for the second kernel) by the forward lists.
template <typename T, int D>
__global__ void __launch_bounds__(256, 4) dist_bwd_da_kernel(
    const float *__restrict__ qa, const float *__restrict__ kc, const T *__restrict__ v,
    const T *__restrict__ o, const float *__restrict__ lse, const T *__restrict__ dout, GraphView g,
    float scale, float *__restrict__ da, float *__restrict__ delta, int64_t ntiles) {
    constexpr int V = Slice<T>::V, L = D / V, G = 32 / L;
    __shared__ int64_t s_offs[SA_MAX_OFFSETS];
    stage_offsets(g, s_offs);
    const int lane = threadIdx.x & 31, grp = lane / L, sub = lane % L;
    const int64_t bh = blockIdx.x / ntiles;
    const int64_t i = (blockIdx.x % ntiles) * kWarpsPerBlock + (threadIdx.x >> 5);
    const int64_t T_ = g.T;
    if (i >= T_) return;
    const int64_t rbase = bh * T_;
    const float nscale2 = -scale * kLog2e;
    float df[V], of[V];  // every group holds the whole dO row
    Slice<T>::load(dout + (rbase + i) * D + sub * V, df);
    Slice<T>::load(o + (rbase + i) * D + sub * V, of);
    float dl = 0.f;
#pragma unroll
    for (int x = 0; x < V; ++x) dl = fmaf(df[x], of[x], dl);
    const float Delta = group_sum<L>(dl);
    const float lse2 = lse[rbase + i] * kLog2e;
    const Coord a = load_coord(qa, rbase + i);
    const RowEdges r = row_edges(g, i);
    float gx = 0.f, gy = 0.f, gz = 0.f;  // this lane's edges' dS (a - c)
    for (int64_t e0 = 0; e0 < r.deg; e0 += 32) {
        const int64_t e = e0 + lane;
        const bool valid = e < r.deg;
        int64_t j = i;
        Coord c{0.f, 0.f, 0.f};
        float p = 0.f;
        if (valid) {
            j = fwd_key(g, r, s_offs, i, e);
            c = load_coord(kc, rbase + j);
            p = ex2(dist_score(a, c, nscale2) - lse2);
        }
        const int n = r.deg - e0 < 32 ? (int)(r.deg - e0) : 32;
        float dpt = 0.f;  // dp of this lane's edge
#pragma unroll 4
        for (int u0 = 0; u0 < n; u0 += G) {
            const int64_t ju = __shfl_sync(0xffffffffu, j, u0 + grp);
            float vf[V];
            Slice<T>::load(v + (rbase + ju) * D + sub * V, vf);
            float dp = 0.f;
#pragma unroll
            for (int x = 0; x < V; ++x) dp = fmaf(df[x], vf[x], dp);
            take_dp<L, G>(group_sum<L>(dp), u0, lane, dpt);
        }
        if (valid) {
            const float ds = p * (dpt - Delta);
            gx = fmaf(ds, a.x - c.x, gx);
            gy = fmaf(ds, a.y - c.y, gy);
            gz = fmaf(ds, a.z - c.z, gz);
        }
    }
    gx = warp_sum(gx);
    gy = warp_sum(gy);
    gz = warp_sum(gz);
    if (lane == 0) {
        const float f = -2.f * scale;
        float *dst = da + (rbase + i) * 3;
        dst[0] = f * gx;
        dst[1] = f * gy;
        dst[2] = f * gz;
        delta[rbase + i] = Delta;
    }
}

// dc_j and dv_j by the transpose lists.
template <typename T, int D>
__global__ void __launch_bounds__(256, 4) dist_bwd_dcdv_kernel(
    const float *__restrict__ qa, const float *__restrict__ kc, const float *__restrict__ lse,
    const float *__restrict__ delta, const T *__restrict__ v, const T *__restrict__ dout,
    GraphView g, float scale, float *__restrict__ dc, T *__restrict__ dv, int64_t ntiles) {
    constexpr int V = Slice<T>::V, L = D / V, G = 32 / L;
    __shared__ int64_t s_offs[SA_MAX_OFFSETS];
    stage_offsets(g, s_offs);
    const int lane = threadIdx.x & 31, grp = lane / L, sub = lane % L;
    const int64_t bh = blockIdx.x / ntiles;
    const int64_t j = (blockIdx.x % ntiles) * kWarpsPerBlock + (threadIdx.x >> 5);
    const int64_t T_ = g.T;
    if (j >= T_) return;
    const int64_t rbase = bh * T_;
    const float nscale2 = -scale * kLog2e;
    const Coord c = load_coord(kc, rbase + j);
    float vf[V];  // every group holds the whole value row
    Slice<T>::load(v + (rbase + j) * D + sub * V, vf);
    const ColEdges ce = col_edges(g, j);
    float adv[V];  // this group's edges' p dO
#pragma unroll
    for (int x = 0; x < V; ++x) adv[x] = 0.f;
    float gx = 0.f, gy = 0.f, gz = 0.f;  // this lane's edges' dS (a - c)
    for (int64_t e0 = 0; e0 < ce.deg; e0 += 32) {
        const int64_t e = e0 + lane;
        const bool valid = e < ce.deg;
        int64_t i = j;
        Coord a{0.f, 0.f, 0.f};
        float p = 0.f, Delta = 0.f;
        if (valid) {
            i = col_query(g, ce, s_offs, j, e);
            a = load_coord(qa, rbase + i);
            p = ex2(dist_score(a, c, nscale2) - __ldg(lse + rbase + i) * kLog2e);
            Delta = __ldg(delta + rbase + i);
        }
        const int n = ce.deg - e0 < 32 ? (int)(ce.deg - e0) : 32;
        float dpt = 0.f;
#pragma unroll 4
        for (int u0 = 0; u0 < n; u0 += G) {
            const int u = u0 + grp;
            const int64_t iu = __shfl_sync(0xffffffffu, i, u);
            const float pu = __shfl_sync(0xffffffffu, p, u);
            float df[V];
            Slice<T>::load(dout + (rbase + iu) * D + sub * V, df);
            float dp = 0.f;
#pragma unroll
            for (int x = 0; x < V; ++x) {
                dp = fmaf(df[x], vf[x], dp);
                adv[x] = fmaf(pu, df[x], adv[x]);
            }
            take_dp<L, G>(group_sum<L>(dp), u0, lane, dpt);
        }
        if (valid) {
            const float ds = p * (dpt - Delta);
            gx = fmaf(ds, a.x - c.x, gx);
            gy = fmaf(ds, a.y - c.y, gy);
            gz = fmaf(ds, a.z - c.z, gz);
        }
    }
#pragma unroll
    for (int off = L; off < 32; off <<= 1) {
#pragma unroll
        for (int x = 0; x < V; ++x) adv[x] += __shfl_xor_sync(0xffffffffu, adv[x], off);
    }
    gx = warp_sum(gx);
    gy = warp_sum(gy);
    gz = warp_sum(gz);
    if (grp == 0) Slice<T>::store(dv + (rbase + j) * D + sub * V, adv);
    if (lane == 0) {
        const float f = 2.f * scale;  // d s / d c = +2 scale (a - c)
        float *dst = dc + (rbase + j) * 3;
        dst[0] = f * gx;
        dst[1] = f * gy;
        dst[2] = f * gz;
    }
}

template <typename T, int D>
sa_status launch_fwd(const sa_tensor *a, const sa_tensor *c, const sa_tensor *v,
                     const GraphView &g, float scale, sa_tensor *out, float *lse, cudaStream_t s) {
    const int64_t BH = v->B * v->H;
    const int64_t ntiles = (g.T + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int64_t nblocks = ntiles * BH;
    if (nblocks > 0x7fffffffLL) return SA_ERR_UNSUPPORTED;
    SA_LAUNCH("dist_fwd", s,
              dist_fwd_kernel<T, D><<<(unsigned)nblocks, 256, 0, s>>>(
                  (const float *)a->ptr, (const float *)c->ptr, (const T *)v->ptr, g,
                  -scale * kLog2e, (T *)out->ptr, lse, ntiles));
    SA_CUDA_TRY(cudaGetLastError());
    return SA_OK;
}

template <typename T, int D>
sa_status launch_bwd(const sa_tensor *a, const sa_tensor *c, const sa_tensor *v,
                     const sa_tensor *o, const float *lse, const sa_tensor *dout,
                     const GraphView &g, float scale, sa_tensor *da, sa_tensor *dc, sa_tensor *dv,
                     float *delta, cudaStream_t s) {
    const int64_t BH = v->B * v->H;
    const int64_t ntiles = (g.T + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int64_t nblocks = ntiles * BH;
    if (nblocks > 0x7fffffffLL) return SA_ERR_UNSUPPORTED;
    SA_LAUNCH("dist_bwd_da", s,
              dist_bwd_da_kernel<T, D><<<(unsigned)nblocks, 256, 0, s>>>(
                  (const float *)a->ptr, (const float *)c->ptr, (const T *)v->ptr,
                  (const T *)o->ptr, lse, (const T *)dout->ptr, g, scale, (float *)da->ptr, delta,
                  ntiles));
    SA_LAUNCH("dist_bwd_dcdv", s,
              dist_bwd_dcdv_kernel<T, D><<<(unsigned)nblocks, 256, 0, s>>>(
                  (const float *)a->ptr, (const float *)c->ptr, lse, delta, (const T *)v->ptr,
                  (const T *)dout->ptr, g, scale, (float *)dc->ptr, (T *)dv->ptr, ntiles));
    SA_CUDA_TRY(cudaGetLastError());
    return SA_OK;
}

}  // namespace

sa_status sa_dist_fwd(const sa_tensor *a, const sa_tensor *c, const sa_tensor *v,
                      const GraphView &g, float scale, sa_tensor *out, float *lse,
                      cudaStream_t s) {
    const bool bf = v->dtype == SA_BF16;
    switch (v->D) {
        case 32:
            return bf ? launch_fwd<__nv_bfloat16, 32>(a, c, v, g, scale, out, lse, s)
                      : launch_fwd<float, 32>(a, c, v, g, scale, out, lse, s);
        case 64:
            return bf ? launch_fwd<__nv_bfloat16, 64>(a, c, v, g, scale, out, lse, s)
                      : launch_fwd<float, 64>(a, c, v, g, scale, out, lse, s);
        case 128:
            return bf ? launch_fwd<__nv_bfloat16, 128>(a, c, v, g, scale, out, lse, s)
                      : launch_fwd<float, 128>(a, c, v, g, scale, out, lse, s);
    }
    return SA_ERR_UNSUPPORTED;
}

sa_status sa_dist_bwd(const sa_tensor *a, const sa_tensor *c, const sa_tensor *v,
                      const sa_tensor *o, const float *lse, const sa_tensor *dout,
                      const GraphView &g, float scale, sa_tensor *da, sa_tensor *dc,
                      sa_tensor *dv, float *delta, cudaStream_t s) {
    const bool bf = v->dtype == SA_BF16;
#define SA_DBWD(TT, DD) launch_bwd<TT, DD>(a, c, v, o, lse, dout, g, scale, da, dc, dv, delta, s)
    switch (v->D) {
        case 32:
            return bf ? SA_DBWD(__nv_bfloat16, 32) : SA_DBWD(float, 32);
        case 64:
            return bf ? SA_DBWD(__nv_bfloat16, 64) : SA_DBWD(float, 64);
        case 128:
            return bf ? SA_DBWD(__nv_bfloat16, 128) : SA_DBWD(float, 128);
    }
#undef SA_DBWD
    return SA_ERR_UNSUPPORTED;
}
