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
#include "tc_common.cuh"

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


// ---- structured graphs: the gathered rows of a block staged in shared memory
//
// On a structured graph the lists of QB consecutive rows b0 .. b0+QB-1 read
// few distinct rows: the forward lists read the keys of one window span
// (b0 - W + 1 .. b0 + QB - 1) and, per distance o, the QB keys b0 - o ..
// b0 - o + QB - 1; the transpose lists read the queries b0 .. b0 + QB + W - 2
// and b0 + o .. b0 + o + QB - 1.  A block of 8 warps stages those rows
// (value rows and key coordinates for the forward and da; dO rows, query
// coordinates, lse and Delta for dc and dv) once with coalesced copies, then
// each warp takes rows b0 + w, b0 + w + 8, ... as above with its phase-1
// scores and phase-2 rows read from shared memory: per 32 rows about 350
// staged rows instead of ~1,300 row reads from L2 (window 32 + 9 links).

constexpr int QB = 32;                  // rows per block
constexpr int kMaxStageBytes = 52 * 1024;  // four blocks per SM

// staged rows of a block: the window span, then one QB-row block per distance
__host__ __device__ __forceinline__ int staged_rows(int W, int n_off) {
    return W + QB - 1 + QB * n_off;
}

template <typename T, int D>
__host__ __device__ __forceinline__ size_t stage_bytes(int W, int n_off, bool with_rowvals) {
    const size_t R = (size_t)staged_rows(W, n_off);
    return R * D * sizeof(T) + R * 3 * sizeof(float) + (with_rowvals ? R * 2 * sizeof(float) : 0);
}

// Stage the block's rows of src (D columns), their coordinates and, for the
// transpose lists, lse (base 2) and Delta: segment 0 is the window span (W +
// QB - 1 rows), segment 1 + x the QB rows of distance offs[x]; each segment's
// source rows are contiguous (DIR = -1: keys b0 - W + 1 .. and b0 - o ..;
// DIR = +1: queries b0 .. and b0 + o ..), so it is one flat copy.  Rows
// outside 0 .. T-1 are not written (no list reads them).  Every thread of
// the block must call it.
template <typename T, int D, int DIR>
__device__ __forceinline__ void stage_block(const GraphView &g, const int64_t *s_offs,
                                            int64_t rbase, int64_t b0, const T *src,
                                            const float *crd_src, const float *lse,
                                            const float *dl, T *rows, float *crd, float *slse,
                                            float *sdl) {
    constexpr int CPR = D * (int)sizeof(T) / 16;  // 16-byte chunks per row
    constexpr int EPC = 16 / (int)sizeof(T);      // elements per chunk
    for (int sg = 0; sg <= g.n_off; ++sg) {
        const int n = sg == 0 ? g.W + QB - 1 : QB;
        const int r0 = sg == 0 ? 0 : g.W + QB - 1 + QB * (sg - 1);
        int64_t s0 = sg == 0 ? (DIR < 0 ? b0 - g.W + 1 : b0)
                             : (DIR < 0 ? b0 - s_offs[sg - 1] : b0 + s_offs[sg - 1]);
        // the rows of the segment inside 0 .. T-1
        const int lo = s0 < 0 ? (int)(-s0 < n ? -s0 : n) : 0;
        const int hi = s0 + n > g.T ? (int)(g.T - s0 > lo ? g.T - s0 : lo) : n;
        if (hi <= lo) continue;
        const T *gsrc = src + (rbase + s0 + lo) * D;
        const uint32_t sdst = tc::smem_u32(rows + (size_t)(r0 + lo) * D);
        for (int c = threadIdx.x; c < (hi - lo) * CPR; c += blockDim.x)
            tc::cp_async16(sdst + 16 * c, gsrc + (size_t)c * EPC);
        const float *csrc = crd_src + (rbase + s0 + lo) * 3;
        float *cdst = crd + 3 * (r0 + lo);
        for (int f = threadIdx.x; f < (hi - lo) * 3; f += blockDim.x) cdst[f] = __ldg(csrc + f);
        if (slse) {
            for (int r = threadIdx.x; r < hi - lo; r += blockDim.x) {
                slse[r0 + lo + r] = __ldg(lse + rbase + s0 + lo + r) * kLog2e;
                sdl[r0 + lo + r] = __ldg(dl + rbase + s0 + lo + r);
            }
        }
    }
    tc::cp_async_commit();
    tc::cp_async_wait<0>();
    __syncthreads();
}

// Shared-memory loads by 32-bit shared address (no generic-address math).
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a));
    return v;
}

__device__ __forceinline__ Coord lds_coord(uint32_t a) {
    Coord c;
    asm volatile("ld.shared.f32 %0, [%3];\n\tld.shared.f32 %1, [%3+4];\n\tld.shared.f32 %2, [%3+8];"
                 : "=f"(c.x), "=f"(c.y), "=f"(c.z)
                 : "r"(a));
    return c;
}

// A lane's slice of a row held in registers (bf16: 4 words of bf16 pairs;
// fp32: 4 floats), with the two row operations of phase 2 against a staged
// slice: the partial dot product and p * row added to an accumulator.  bf16
// products are exact (fma.rn.f32.bf16); p is rounded to bf16 for the sum, as
// the band kernels round P for their P V products.
template <typename T>
struct StagedRow;

template <>
struct StagedRow<__nv_bfloat16> {
    uint32_t w[4];
    __device__ __forceinline__ void hold(const __nv_bfloat16 *p) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
        w[0] = u.x, w[1] = u.y, w[2] = u.z, w[3] = u.w;
    }
    __device__ __forceinline__ void stage(uint32_t a) {  // shared address
        const uint4 u = lds128(a);
        w[0] = u.x, w[1] = u.y, w[2] = u.z, w[3] = u.w;
    }
    __device__ __forceinline__ float dot(const StagedRow &o) const {
        float a = 0.f, b = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            a = tc::fma_bf_lo(w[k], o.w[k], a);
            b = tc::fma_bf_hi(w[k], o.w[k], b);
        }
        return a + b;
    }
    __device__ __forceinline__ void axpy(float p, float *acc) const {  // acc += p * this
        const uint32_t p2 = tc::pack_bf16x2(p, p);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            acc[2 * k] = tc::fma_bf_lo(p2, w[k], acc[2 * k]);
            acc[2 * k + 1] = tc::fma_bf_hi(p2, w[k], acc[2 * k + 1]);
        }
    }
};

template <>
struct StagedRow<float> {
    float f[4];
    __device__ __forceinline__ void hold(const float *p) {
        const float4 u = __ldg(reinterpret_cast<const float4 *>(p));
        f[0] = u.x, f[1] = u.y, f[2] = u.z, f[3] = u.w;
    }
    __device__ __forceinline__ void stage(uint32_t a) {  // shared address
        const uint4 u = lds128(a);
        f[0] = __uint_as_float(u.x), f[1] = __uint_as_float(u.y), f[2] = __uint_as_float(u.z),
        f[3] = __uint_as_float(u.w);
    }
    __device__ __forceinline__ float dot(const StagedRow &o) const {
        return fmaf(f[0], o.f[0], fmaf(f[1], o.f[1], fmaf(f[2], o.f[2], f[3] * o.f[3])));
    }
    __device__ __forceinline__ void axpy(float p, float *acc) const {
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] = fmaf(p, f[k], acc[k]);
    }
};

// Staged rows of a list in 32-bit arithmetic, set up once per row: edge e
// < nsplit is staged row a + sa * e, later edges row b + sb * e.  Forward list of
// query i = b0 + t: the links (row t of distance block first + e), then the
// window (key lo + e - ndil).  Transpose list of key j = b0 + t: the window
// (query j + e), then the links in ascending distance (block n_off - 1 -
// (e - nwin)).
struct StagedList {
    int deg, nsplit, a, sa, b, sb;
    __device__ __forceinline__ int row(int e) const { return e < nsplit ? a + sa * e : b + sb * e; }
};

// Number of distances (s_offs, descending) for which pred(o) holds, counted
// by the warp's lanes in two ballots (n_off <= 64).  Every lane must call it.
template <typename Pred>
__device__ __forceinline__ int count_offsets(const int64_t *s_offs, int n_off, int lane, Pred pred) {
    const unsigned b0 = __ballot_sync(0xffffffffu, lane < n_off && pred(s_offs[lane]));
    const unsigned b1 = __ballot_sync(0xffffffffu, lane + 32 < n_off && pred(s_offs[lane + 32]));
    return __popc(b0) + __popc(b1);
}

// The transpose list of key j as col_edges gives it (structured graph), its
// distances counted by the warp instead of a loop over all of them (the
// forward lists keep row_edges: its loop stops at the first distance that
// reaches the row, which for most rows is the first one).
__device__ __forceinline__ ColEdges col_edges_warp(const GraphView &g, const int64_t *s_offs,
                                                   int64_t j, int lane) {
    ColEdges c;
    c.nwin = g.T - j < g.W ? g.T - j : g.W;
    c.deg = c.nwin + count_offsets(s_offs, g.n_off, lane, [&](int64_t o) { return j + o < g.T; });
    c.start = 0;
    return c;
}

__device__ __forceinline__ StagedList fwd_list(const GraphView &g, const RowEdges &r, int64_t b0,
                                               int t) {
    StagedList l;
    l.deg = (int)r.deg;
    l.nsplit = r.ndil;
    l.a = g.W + QB - 1 + QB * r.first + t;
    l.sa = QB;
    l.b = (int)(r.lo - (b0 - g.W + 1)) - r.ndil;
    l.sb = 1;
    return l;
}

__device__ __forceinline__ StagedList col_list(const GraphView &g, const ColEdges &c, int t) {
    StagedList l;
    l.deg = (int)c.deg;
    l.nsplit = (int)c.nwin;
    l.a = t;
    l.sa = 1;
    // link e - nwin sits in block n_off - 1 - (e - nwin)
    l.b = g.W + QB - 1 + QB * (g.n_off - 1) + t + QB * l.nsplit;
    l.sb = -QB;
    return l;
}

template <typename T, int D>
__global__ void __launch_bounds__(256, 4) dist_fwd_staged_kernel(
    const float *__restrict__ qa, const float *__restrict__ kc, const T *__restrict__ v,
    GraphView g, float nscale2, T *__restrict__ out, float *__restrict__ lse, int64_t nblk) {
    constexpr int V = Slice<T>::V, L = D / V, G = 32 / L;
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ int64_t s_offs[SA_MAX_OFFSETS];
    stage_offsets(g, s_offs);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, grp = lane / L, sub = lane % L;
    const int64_t bh = blockIdx.x / nblk, b0 = (blockIdx.x % nblk) * QB, T_ = g.T;
    const int64_t rbase = bh * T_;
    const int R = staged_rows(g.W, g.n_off);
    T *rows = reinterpret_cast<T *>(dsm);
    float *crd = reinterpret_cast<float *>(dsm + (size_t)R * D * sizeof(T));
    stage_block<T, D, -1>(g, s_offs, rbase, b0, v, kc, nullptr, nullptr, rows, crd, nullptr,
                          nullptr);
    constexpr uint32_t kRowBytes = D * sizeof(T);
    const uint32_t rows_s = tc::smem_u32(rows) + 16 * sub;  // this lane's 16 bytes of row 0
    const uint32_t crd_s = tc::smem_u32(crd);
    // each warp's rows are b0 + warp + 8 u; a row's own inputs are loaded one
    // row ahead, so that their latency hides behind the previous row's work
    Coord a_nx{0.f, 0.f, 0.f};
    if (b0 + warp < T_) a_nx = load_coord(qa, rbase + b0 + warp);
    for (int t = warp; t < QB; t += kWarpsPerBlock) {
        const int64_t i = b0 + t;
        if (i >= T_) break;
        const Coord a = a_nx;
        if (t + kWarpsPerBlock < QB && i + kWarpsPerBlock < T_)
            a_nx = load_coord(qa, rbase + i + kWarpsPerBlock);
        const StagedList sl = fwd_list(g, row_edges(g, i), b0, t);
        float m = -INFINITY, lpart = 0.f, acc[V];
#pragma unroll
        for (int x = 0; x < V; ++x) acc[x] = 0.f;
        for (int e0 = 0; e0 < sl.deg; e0 += 32) {
            const int e = e0 + lane;
            int sr = t + g.W - 1;  // lanes past the list: key i's own row (written), p = 0
            float s = -INFINITY;
            if (e < sl.deg) {
                sr = sl.row(e);
                s = dist_score(a, lds_coord(crd_s + 12 * sr), nscale2);
            }
            const float mn = fmaxf(m, warp_max(s));
            const float al = ex2(m - mn);
            lpart *= al;
#pragma unroll
            for (int x = 0; x < V; ++x) acc[x] *= al;
            m = mn;
            const float p = ex2(s - mn);
            lpart += p;
            const int n = sl.deg - e0 < 32 ? sl.deg - e0 : 32;
#pragma unroll 4
            for (int u0 = 0; u0 < n; u0 += G) {
                const int u = u0 + grp;
                const int su = __shfl_sync(0xffffffffu, sr, u);
                const float pu = __shfl_sync(0xffffffffu, p, u);
                StagedRow<T> vr;
                vr.stage(rows_s + (uint32_t)su * kRowBytes);
                vr.axpy(pu, acc);
            }
        }
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
}

template <typename T, int D>
__global__ void __launch_bounds__(256, 4) dist_bwd_da_staged_kernel(
    const float *__restrict__ qa, const float *__restrict__ kc, const T *__restrict__ v,
    const T *__restrict__ o, const float *__restrict__ lse, const T *__restrict__ dout, GraphView g,
    float scale, float *__restrict__ da, float *__restrict__ delta, int64_t nblk) {
    constexpr int V = Slice<T>::V, L = D / V, G = 32 / L;
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ int64_t s_offs[SA_MAX_OFFSETS];
    stage_offsets(g, s_offs);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, grp = lane / L, sub = lane % L;
    const int64_t bh = blockIdx.x / nblk, b0 = (blockIdx.x % nblk) * QB, T_ = g.T;
    const int64_t rbase = bh * T_;
    const float nscale2 = -scale * kLog2e;
    const int R = staged_rows(g.W, g.n_off);
    T *rows = reinterpret_cast<T *>(dsm);
    float *crd = reinterpret_cast<float *>(dsm + (size_t)R * D * sizeof(T));
    stage_block<T, D, -1>(g, s_offs, rbase, b0, v, kc, nullptr, nullptr, rows, crd, nullptr,
                          nullptr);
    constexpr uint32_t kRowBytes = D * sizeof(T);
    const uint32_t rows_s = tc::smem_u32(rows) + 16 * sub;  // this lane's 16 bytes of row 0
    const uint32_t crd_s = tc::smem_u32(crd);
    // a row's own inputs one row ahead (as in the forward)
    StagedRow<T> dh_nx, oh_nx;  // this lane's slices of the next row's dO and out
    float lse_nx = 0.f;
    Coord a_nx{0.f, 0.f, 0.f};
    auto fetch = [&](int64_t ii) {
        dh_nx.hold(dout + (rbase + ii) * D + sub * V);
        oh_nx.hold(o + (rbase + ii) * D + sub * V);
        lse_nx = __ldg(lse + rbase + ii);
        a_nx = load_coord(qa, rbase + ii);
    };
    if (b0 + warp < T_) fetch(b0 + warp);
    for (int t = warp; t < QB; t += kWarpsPerBlock) {
        const int64_t i = b0 + t;
        if (i >= T_) break;
        const StagedRow<T> dh = dh_nx;
        const float Delta = group_sum<L>(dh.dot(oh_nx));
        const float lse2 = lse_nx * kLog2e;
        const Coord a = a_nx;
        if (t + kWarpsPerBlock < QB && i + kWarpsPerBlock < T_) fetch(i + kWarpsPerBlock);
        const StagedList sl = fwd_list(g, row_edges(g, i), b0, t);
        float gx = 0.f, gy = 0.f, gz = 0.f;
        for (int e0 = 0; e0 < sl.deg; e0 += 32) {
            const int e = e0 + lane;
            int sr = t + g.W - 1;  // lanes past the list: key i's own row (written), p = 0
            Coord c{0.f, 0.f, 0.f};
            float p = 0.f;
            if (e < sl.deg) {
                sr = sl.row(e);
                c = lds_coord(crd_s + 12 * sr);
                p = ex2(dist_score(a, c, nscale2) - lse2);
            }
            const int n = sl.deg - e0 < 32 ? sl.deg - e0 : 32;
            float dpt = 0.f;
#pragma unroll 4
            for (int u0 = 0; u0 < n; u0 += G) {
                const int su = __shfl_sync(0xffffffffu, sr, u0 + grp);
                StagedRow<T> vr;
                vr.stage(rows_s + (uint32_t)su * kRowBytes);
                take_dp<L, G>(group_sum<L>(dh.dot(vr)), u0, lane, dpt);
            }
            const float ds = p * (dpt - Delta);  // p = 0 past the list
            gx = fmaf(ds, a.x - c.x, gx);
            gy = fmaf(ds, a.y - c.y, gy);
            gz = fmaf(ds, a.z - c.z, gz);
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
}

template <typename T, int D>
__global__ void __launch_bounds__(256, 4) dist_bwd_dcdv_staged_kernel(
    const float *__restrict__ qa, const float *__restrict__ kc, const float *__restrict__ lse,
    const float *__restrict__ delta, const T *__restrict__ v, const T *__restrict__ dout,
    GraphView g, float scale, float *__restrict__ dc, T *__restrict__ dv, int64_t nblk) {
    constexpr int V = Slice<T>::V, L = D / V, G = 32 / L;
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ int64_t s_offs[SA_MAX_OFFSETS];
    stage_offsets(g, s_offs);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, grp = lane / L, sub = lane % L;
    const int64_t bh = blockIdx.x / nblk, b0 = (blockIdx.x % nblk) * QB, T_ = g.T;
    const int64_t rbase = bh * T_;
    const float nscale2 = -scale * kLog2e;
    const int R = staged_rows(g.W, g.n_off);
    T *rows = reinterpret_cast<T *>(dsm);
    float *crd = reinterpret_cast<float *>(dsm + (size_t)R * D * sizeof(T));
    float *slse = crd + 3 * R, *sdl = slse + R;
    stage_block<T, D, +1>(g, s_offs, rbase, b0, dout, qa, lse, delta, rows, crd, slse, sdl);
    constexpr uint32_t kRowBytes = D * sizeof(T);
    const uint32_t rows_s = tc::smem_u32(rows) + 16 * sub;  // this lane's 16 bytes of row 0
    const uint32_t crd_s = tc::smem_u32(crd);
    for (int t = warp; t < QB; t += kWarpsPerBlock) {
        const int64_t j = b0 + t;
        if (j >= T_) break;
        const Coord c = load_coord(kc, rbase + j);
        StagedRow<T> vh;  // this lane's slice of the value row
        vh.hold(v + (rbase + j) * D + sub * V);
        const StagedList sl = col_list(g, col_edges_warp(g, s_offs, j, lane), t);
        float adv[V];
#pragma unroll
        for (int x = 0; x < V; ++x) adv[x] = 0.f;
        float gx = 0.f, gy = 0.f, gz = 0.f;
        for (int e0 = 0; e0 < sl.deg; e0 += 32) {
            const int e = e0 + lane;
            int sr = t;  // lanes past the list: query j's own row (written), p = 0
            Coord a{0.f, 0.f, 0.f};
            float p = 0.f, Delta = 0.f;
            if (e < sl.deg) {
                sr = sl.row(e);
                a = lds_coord(crd_s + 12 * sr);
                p = ex2(dist_score(a, c, nscale2) - slse[sr]);
                Delta = sdl[sr];
            }
            const int n = sl.deg - e0 < 32 ? sl.deg - e0 : 32;
            float dpt = 0.f;
#pragma unroll 4
            for (int u0 = 0; u0 < n; u0 += G) {
                const int u = u0 + grp;
                const int su = __shfl_sync(0xffffffffu, sr, u);
                const float pu = __shfl_sync(0xffffffffu, p, u);
                StagedRow<T> dr;
                dr.stage(rows_s + (uint32_t)su * kRowBytes);
                dr.axpy(pu, adv);
                take_dp<L, G>(group_sum<L>(vh.dot(dr)), u0, lane, dpt);
            }
            const float ds = p * (dpt - Delta);  // p = 0 past the list
            gx = fmaf(ds, a.x - c.x, gx);
            gy = fmaf(ds, a.y - c.y, gy);
            gz = fmaf(ds, a.z - c.z, gz);
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
            const float f = 2.f * scale;
            float *dst = dc + (rbase + j) * 3;
            dst[0] = f * gx;
            dst[1] = f * gy;
            dst[2] = f * gz;
        }
    }
}

// Structured graphs whose staged rows fit kMaxStageBytes take the staged
// kernels (the window and distance spans of a block are 32-bit offsets).
// The size varies with the graph, so the kernels are opted in once for the
// largest.
template <typename T, int D>
bool use_staged(const GraphView &g, bool with_rowvals) {
    return g.kind == 0 && g.W <= (1 << 20) &&
           stage_bytes<T, D>(g.W, g.n_off, with_rowvals) <= (size_t)kMaxStageBytes;
}

template <typename T, int D>
sa_status launch_fwd(const sa_tensor *a, const sa_tensor *c, const sa_tensor *v,
                     const GraphView &g, float scale, sa_tensor *out, float *lse, cudaStream_t s) {
    const int64_t BH = v->B * v->H;
    if (use_staged<T, D>(g, false)) {
        const int64_t nblk = (g.T + QB - 1) / QB;
        if (nblk * BH > 0x7fffffffLL) return SA_ERR_UNSUPPORTED;
        const int bytes = (int)stage_bytes<T, D>(g.W, g.n_off, false);
        SA_CUDA_TRY(sa_smem_optin((const void *)dist_fwd_staged_kernel<T, D>, kMaxStageBytes));
        SA_LAUNCH("dist_fwd", s,
                  dist_fwd_staged_kernel<T, D><<<(unsigned)(nblk * BH), 256, bytes, s>>>(
                      (const float *)a->ptr, (const float *)c->ptr, (const T *)v->ptr, g,
                      -scale * kLog2e, (T *)out->ptr, lse, nblk));
        SA_CUDA_TRY(cudaGetLastError());
        return SA_OK;
    }
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
    if (use_staged<T, D>(g, true)) {
        const int64_t nblk = (g.T + QB - 1) / QB;
        if (nblk * BH > 0x7fffffffLL) return SA_ERR_UNSUPPORTED;
        const int b_da = (int)stage_bytes<T, D>(g.W, g.n_off, false);
        const int b_dc = (int)stage_bytes<T, D>(g.W, g.n_off, true);
        SA_CUDA_TRY(sa_smem_optin((const void *)dist_bwd_da_staged_kernel<T, D>, kMaxStageBytes));
        SA_CUDA_TRY(sa_smem_optin((const void *)dist_bwd_dcdv_staged_kernel<T, D>, kMaxStageBytes));
        SA_LAUNCH("dist_bwd_da", s,
                  dist_bwd_da_staged_kernel<T, D><<<(unsigned)(nblk * BH), 256, b_da, s>>>(
                      (const float *)a->ptr, (const float *)c->ptr, (const T *)v->ptr,
                      (const T *)o->ptr, lse, (const T *)dout->ptr, g, scale, (float *)da->ptr,
                      delta, nblk));
        SA_LAUNCH("dist_bwd_dcdv", s,
                  dist_bwd_dcdv_staged_kernel<T, D><<<(unsigned)(nblk * BH), 256, b_dc, s>>>(
                      (const float *)a->ptr, (const float *)c->ptr, lse, delta,
                      (const T *)v->ptr, (const T *)dout->ptr, g, scale, (float *)dc->ptr,
                      (T *)dv->ptr, nblk));
        SA_CUDA_TRY(cudaGetLastError());
        return SA_OK;
    }
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
