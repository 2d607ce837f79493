// attn_gather.cu -- every edge of the graph on CUDA cores (the gather path).
//
// A warp owns one query (forward, dQ) or one key (dK/dV).  Its 32 lanes
// split into G groups of L lanes; a group holds one neighbour row, each lane
// one 16-byte slice of it (8 bf16 or 4 fp32), so each load instruction of a
// warp fetches G whole rows and a dot product is L-1 shuffles.  Every group
// keeps its own running (max, sum, accumulator) -- the online softmax -- and
// the groups are merged at the end with the usual rescaling.  Scores are kept
// in base 2: s2 = (scale * log2 e) * q.k, so p = 2^(s2 - m2).
//
// Backward (probabilities recomputed from lse):
//   Delta_i = dO_i . out_i,  p = exp(s - lse_i),  dp = dO_i . v_j,
//   ds = p (dp - Delta_i);   dQ_i = scale sum_j ds k_j   (forward lists)
//   dV_j = sum_i p dO_i,     dK_j = scale sum_i ds q_i  (transpose lists)
// Two kernels with disjoint outputs; no float atomics, so results are
// bitwise reproducible.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sa_internal.cuh"

#include "gather_common.cuh"

namespace {

using namespace gather;

// ---- kernels ---------------------------------------------------------------

template <typename T, int D>
__global__ void __launch_bounds__(256) gather_fwd_kernel(const T *__restrict__ q,
                                                         const T *__restrict__ k,
                                                         const T *__restrict__ v, GraphView g,
                                                         float scale2, T *__restrict__ out,
                                                         float *__restrict__ lse, int64_t ntiles,
                                                         int64_t H, int64_t Hkv) {
    constexpr int V = Slice<T>::V, L = D / V, G = 32 / L;
    static_assert(L >= 1 && L <= 32 && G * L == 32, "slice layout");
    const int lane = threadIdx.x & 31, grp = lane / L, sub = lane % L;
    const int64_t bh = blockIdx.x / ntiles;
    const int64_t i = (blockIdx.x % ntiles) * kWarpsPerBlock + (threadIdx.x >> 5);
    const int64_t T_ = g.T;
    if (i >= T_) return;
    const int64_t base = bh * T_ * D, kvbase = kv_slice(bh, H, Hkv) * T_ * D;
    float qf[V];
    Slice<T>::load(q + base + i * D + sub * V, qf);
#pragma unroll
    for (int a = 0; a < V; ++a) qf[a] *= scale2;
    const RowEdges r = row_edges(g, i);
    float m = -INFINITY, l = 0.f, acc[V];
#pragma unroll
    for (int a = 0; a < V; ++a) acc[a] = 0.f;
    for (int64_t e0 = 0; e0 < r.deg; e0 += G) {
        const int64_t e = e0 + grp;
        const bool valid = e < r.deg;
        float kf[V], vf[V];
        if (valid) {
            const int64_t j = row_edge(g, r, i, e);
            Slice<T>::load(k + kvbase + j * D + sub * V, kf);
            Slice<T>::load(v + kvbase + j * D + sub * V, vf);
        } else {
#pragma unroll
            for (int a = 0; a < V; ++a) kf[a] = vf[a] = 0.f;
        }
        float s = 0.f;
#pragma unroll
        for (int a = 0; a < V; ++a) s = fmaf(qf[a], kf[a], s);
        s = group_sum<L>(s);
        if (valid) {
            const float mn = fmaxf(m, s);
            const float al = ex2(m - mn), p = ex2(s - mn);
            l = l * al + p;
#pragma unroll
            for (int a = 0; a < V; ++a) acc[a] = fmaf(p, vf[a], acc[a] * al);
            m = mn;
        }
    }
    // merge the G group states
#pragma unroll
    for (int o = L; o < 32; o <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, o);
        const float lo = __shfl_xor_sync(0xffffffffu, l, o);
        float ao[V];
#pragma unroll
        for (int a = 0; a < V; ++a) ao[a] = __shfl_xor_sync(0xffffffffu, acc[a], o);
        const float mn = fmaxf(m, mo);
        if (mn != -INFINITY) {
            const float x = ex2(m - mn), y = ex2(mo - mn);
            l = l * x + lo * y;
#pragma unroll
            for (int a = 0; a < V; ++a) acc[a] = acc[a] * x + ao[a] * y;
            m = mn;
        }
    }
    if (grp == 0) {
        float o_[V];
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int a = 0; a < V; ++a) o_[a] = acc[a] * inv;
        Slice<T>::store(out + base + i * D + sub * V, o_);
        if (sub == 0) lse[bh * T_ + i] = l > 0.f ? (m + lg2(l)) * kLn2 : -INFINITY;
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) gather_bwd_dq_kernel(
    const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
    const T *__restrict__ o, const float *__restrict__ lse, const T *__restrict__ dout, GraphView g,
    float scale, T *__restrict__ dq, float *__restrict__ delta, int64_t ntiles, int64_t H,
    int64_t Hkv) {
    constexpr int V = Slice<T>::V, L = D / V, G = 32 / L;
    const int lane = threadIdx.x & 31, grp = lane / L, sub = lane % L;
    const int64_t bh = blockIdx.x / ntiles;
    const int64_t i = (blockIdx.x % ntiles) * kWarpsPerBlock + (threadIdx.x >> 5);
    const int64_t T_ = g.T;
    if (i >= T_) return;
    const int64_t base = bh * T_ * D, kvbase = kv_slice(bh, H, Hkv) * T_ * D;
    const float scale2 = scale * kLog2e;
    float qf[V], df[V], of[V];
    Slice<T>::load(q + base + i * D + sub * V, qf);
    Slice<T>::load(dout + base + i * D + sub * V, df);
    Slice<T>::load(o + base + i * D + sub * V, of);
    float dl = 0.f;
#pragma unroll
    for (int a = 0; a < V; ++a) {
        dl = fmaf(df[a], of[a], dl);
        qf[a] *= scale2;
    }
    const float Delta = group_sum<L>(dl);
    const float lse2 = lse[bh * T_ + i] * kLog2e;
    const RowEdges r = row_edges(g, i);
    float acc[V];
#pragma unroll
    for (int a = 0; a < V; ++a) acc[a] = 0.f;
    for (int64_t e0 = 0; e0 < r.deg; e0 += G) {
        const int64_t e = e0 + grp;
        const bool valid = e < r.deg;
        float kf[V], vf[V];
        if (valid) {
            const int64_t j = row_edge(g, r, i, e);
            Slice<T>::load(k + kvbase + j * D + sub * V, kf);
            Slice<T>::load(v + kvbase + j * D + sub * V, vf);
        } else {
#pragma unroll
            for (int a = 0; a < V; ++a) kf[a] = vf[a] = 0.f;
        }
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int a = 0; a < V; ++a) {
            s = fmaf(qf[a], kf[a], s);
            dp = fmaf(df[a], vf[a], dp);
        }
        s = group_sum<L>(s);
        dp = group_sum<L>(dp);
        if (valid) {
            const float p = ex2(s - lse2);
            const float ds = p * (dp - Delta);
#pragma unroll
            for (int a = 0; a < V; ++a) acc[a] = fmaf(ds, kf[a], acc[a]);
        }
    }
#pragma unroll
    for (int off = L; off < 32; off <<= 1)
#pragma unroll
        for (int a = 0; a < V; ++a) acc[a] += __shfl_xor_sync(0xffffffffu, acc[a], off);
    if (grp == 0) {
#pragma unroll
        for (int a = 0; a < V; ++a) acc[a] *= scale;
        Slice<T>::store(dq + base + i * D + sub * V, acc);
        if (sub == 0) delta[bh * T_ + i] = Delta;
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) gather_bwd_dkdv_kernel(
    const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
    const float *__restrict__ lse, const float *__restrict__ delta, const T *__restrict__ dout,
    GraphView g, float scale, T *__restrict__ dk, T *__restrict__ dv, int64_t ntiles, int64_t H,
    int64_t Hkv) {
    constexpr int V = Slice<T>::V, L = D / V, G = 32 / L;
    const int lane = threadIdx.x & 31, grp = lane / L, sub = lane % L;
    const int64_t kvbh = blockIdx.x / ntiles;  // key/value slice
    const int64_t j = (blockIdx.x % ntiles) * kWarpsPerBlock + (threadIdx.x >> 5);
    const int64_t T_ = g.T;
    if (j >= T_) return;
    const int64_t kvbase = kvbh * T_ * D;
    // the query heads that read this key/value head: a group of H / Hkv
    const int64_t gsize = H / Hkv, qbh0 = (kvbh / Hkv) * H + (kvbh % Hkv) * gsize;
    const float scale2 = scale * kLog2e;
    float kf[V], vf[V];
    Slice<T>::load(k + kvbase + j * D + sub * V, kf);
    Slice<T>::load(v + kvbase + j * D + sub * V, vf);
#pragma unroll
    for (int a = 0; a < V; ++a) kf[a] *= scale2;
    const ColEdges c = col_edges(g, j);
    float adk[V], adv[V];
#pragma unroll
    for (int a = 0; a < V; ++a) adk[a] = adv[a] = 0.f;
    for (int64_t hq = 0; hq < gsize; ++hq) {
        const int64_t bh = qbh0 + hq, base = bh * T_ * D;
        for (int64_t e0 = 0; e0 < c.deg; e0 += G) {
            const int64_t e = e0 + grp;
            const bool valid = e < c.deg;
            float qf[V], df[V];
            float lse2 = 0.f, Delta = 0.f;
            if (valid) {
                const int64_t i = col_edge(g, c, j, e);
                Slice<T>::load(q + base + i * D + sub * V, qf);
                Slice<T>::load(dout + base + i * D + sub * V, df);
                lse2 = __ldg(lse + bh * T_ + i) * kLog2e;
                Delta = __ldg(delta + bh * T_ + i);
            } else {
#pragma unroll
                for (int a = 0; a < V; ++a) qf[a] = df[a] = 0.f;
            }
            float s = 0.f, dp = 0.f;
#pragma unroll
            for (int a = 0; a < V; ++a) {
                s = fmaf(qf[a], kf[a], s);
                dp = fmaf(df[a], vf[a], dp);
            }
            s = group_sum<L>(s);
            dp = group_sum<L>(dp);
            if (valid) {
                const float p = ex2(s - lse2);
                const float ds = p * (dp - Delta);
#pragma unroll
                for (int a = 0; a < V; ++a) {
                    adv[a] = fmaf(p, df[a], adv[a]);
                    adk[a] = fmaf(ds, qf[a], adk[a]);
                }
            }
        }
    }
#pragma unroll
    for (int off = L; off < 32; off <<= 1)
#pragma unroll
        for (int a = 0; a < V; ++a) {
            adk[a] += __shfl_xor_sync(0xffffffffu, adk[a], off);
            adv[a] += __shfl_xor_sync(0xffffffffu, adv[a], off);
        }
    if (grp == 0) {
#pragma unroll
        for (int a = 0; a < V; ++a) adk[a] *= scale;
        Slice<T>::store(dk + kvbase + j * D + sub * V, adk);
        Slice<T>::store(dv + kvbase + j * D + sub * V, adv);
    }
}

template <typename T, int D>
sa_status launch_fwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                     const GraphView &g, float scale, sa_tensor *out, float *lse, cudaStream_t s) {
    const int64_t BH = q->B * q->H;
    const int64_t ntiles = (g.T + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int64_t nblocks = ntiles * BH;
    if (nblocks <= 0) return SA_OK;
    if (nblocks > 0x7fffffffLL) return SA_ERR_UNSUPPORTED;
    SA_LAUNCH("gather_fwd", s,
              gather_fwd_kernel<T, D><<<(unsigned)nblocks, 256, 0, s>>>(
                  (const T *)q->ptr, (const T *)k->ptr, (const T *)v->ptr, g, scale * kLog2e,
                  (T *)out->ptr, lse, ntiles, q->H, k->H));
    SA_CUDA_TRY(cudaGetLastError());
    return SA_OK;
}

template <typename T, int D>
sa_status launch_bwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                     const sa_tensor *o, const float *lse, const sa_tensor *dout,
                     const GraphView &g, float scale, sa_tensor *dq, sa_tensor *dk, sa_tensor *dv,
                     float *delta, cudaStream_t s) {
    const int64_t BH = q->B * q->H;
    const int64_t ntiles = (g.T + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int64_t nblocks = ntiles * BH;
    if (nblocks <= 0) return SA_OK;
    if (nblocks > 0x7fffffffLL) return SA_ERR_UNSUPPORTED;
    SA_LAUNCH("gather_bwd_dq", s,
              gather_bwd_dq_kernel<T, D><<<(unsigned)nblocks, 256, 0, s>>>(
                  (const T *)q->ptr, (const T *)k->ptr, (const T *)v->ptr, (const T *)o->ptr, lse,
                  (const T *)dout->ptr, g, scale, (T *)dq->ptr, delta, ntiles, q->H, k->H));
    const int64_t nblocks_kv = ntiles * (k->B * k->H);
    SA_LAUNCH("gather_bwd_dkdv", s,
              gather_bwd_dkdv_kernel<T, D><<<(unsigned)nblocks_kv, 256, 0, s>>>(
                  (const T *)q->ptr, (const T *)k->ptr, (const T *)v->ptr, lse, delta,
                  (const T *)dout->ptr, g, scale, (T *)dk->ptr, (T *)dv->ptr, ntiles, q->H,
                  k->H));
    SA_CUDA_TRY(cudaGetLastError());
    return SA_OK;
}

}  // namespace

sa_status sa_gather_fwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                        const GraphView &g, float scale, sa_tensor *out, float *lse,
                        cudaStream_t s) {
    const bool bf = q->dtype == SA_BF16;
    switch (q->D) {
        case 32:
            return bf ? launch_fwd<__nv_bfloat16, 32>(q, k, v, g, scale, out, lse, s)
                      : launch_fwd<float, 32>(q, k, v, g, scale, out, lse, s);
        case 64:
            return bf ? launch_fwd<__nv_bfloat16, 64>(q, k, v, g, scale, out, lse, s)
                      : launch_fwd<float, 64>(q, k, v, g, scale, out, lse, s);
        case 128:
            return bf ? launch_fwd<__nv_bfloat16, 128>(q, k, v, g, scale, out, lse, s)
                      : launch_fwd<float, 128>(q, k, v, g, scale, out, lse, s);
    }
    return SA_ERR_UNSUPPORTED;
}

sa_status sa_gather_bwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                        const sa_tensor *o, const float *lse, const sa_tensor *dout,
                        const GraphView &g, float scale, sa_tensor *dq, sa_tensor *dk,
                        sa_tensor *dv, float *delta, cudaStream_t s) {
    const bool bf = q->dtype == SA_BF16;
#define SA_BWD(TT, DD) launch_bwd<TT, DD>(q, k, v, o, lse, dout, g, scale, dq, dk, dv, delta, s)
    switch (q->D) {
        case 32:
            return bf ? SA_BWD(__nv_bfloat16, 32) : SA_BWD(float, 32);
        case 64:
            return bf ? SA_BWD(__nv_bfloat16, 64) : SA_BWD(float, 64);
        case 128:
            return bf ? SA_BWD(__nv_bfloat16, 128) : SA_BWD(float, 128);
    }
#undef SA_BWD
    return SA_ERR_UNSUPPORTED;
}
