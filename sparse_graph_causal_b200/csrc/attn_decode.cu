// attn_decode.cu -- one new query per (batch row, head) against a KV cache,
// over the same neighbour graph.
//
// Page "SpatialLM-Mini sped up training with a 16K context by 2.47x on an RTX
// 3050", section "What to check before adopting it in your project": the
// prototype has no KV cache and its generation speed was not measured.  Here
// a token at position p (its key and value already appended at cache row p)
// attends to N(p) of the graph -- for a structured graph its W-1 cached
// predecessors, itself and the rows p - 2^k -- exactly as row p of the full
// causal computation does.  Grouped-query attention ("MiniGPT (Part 6)",
// introduction: grouped-query attention shrinks the key-value cache): query
// head h reads cache head h / (H / Hkv).
//
// Every edge is a gathered row, so this is an HBM/L2-bound gather: one CTA
// of 8 warps per (b, h); the 32 lanes of a warp form G groups of L lanes,
// each group holding one cached row (16 bytes per lane).  Group e of the CTA
// takes edges e, e + 8G, ... with its own online-softmax state; the states
// are merged in the warp by shuffles, then across the warps in shared memory.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gather_common.cuh"

namespace {

using namespace gather;

constexpr int kDecWarps = 8;

template <typename T, int D>
__global__ void __launch_bounds__(32 * kDecWarps) decode_kernel(
    const T *__restrict__ q, const T *__restrict__ kc, const T *__restrict__ vc,
    const int64_t *__restrict__ pos, GraphView g, int64_t H, int64_t Hkv, int64_t Tmax,
    float scale2, T *__restrict__ out, float *__restrict__ lse, int *err) {
    constexpr int V = Slice<T>::V, L = D / V, G = 32 / L;
    constexpr int NG = G * kDecWarps;  // groups per CTA
    __shared__ float s_m[kDecWarps], s_l[kDecWarps];
    __shared__ float s_acc[kDecWarps][D];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = lane / L, sub = lane % L;
    const int64_t bh = blockIdx.x, b = bh / H, h = bh % H;
    const int64_t kvh = b * Hkv + h / (H / Hkv);
    const int64_t p = pos[b];
    const bool in_range = p >= 0 && p < Tmax && p < g.T;
    if (!in_range) {
        // a position outside the cache or the graph: flagged, row left empty
        if (threadIdx.x == 0) atomicOr(err, SA_DEVERR_BOUNDS);
        if (warp == 0) {
            float z[V];
#pragma unroll
            for (int x = 0; x < V; ++x) z[x] = 0.f;
            if (grp == 0) Slice<T>::store(out + bh * D + sub * V, z);
            if (lane == 0) lse[bh] = -INFINITY;
        }
        return;
    }
    const T *kb = kc + kvh * Tmax * D, *vb = vc + kvh * Tmax * D;
    float qf[V];
    Slice<T>::load(q + bh * D + sub * V, qf);
#pragma unroll
    for (int x = 0; x < V; ++x) qf[x] *= scale2;
    const RowEdges r = row_edges(g, p);
    float m = -INFINITY, l = 0.f, acc[V];
#pragma unroll
    for (int x = 0; x < V; ++x) acc[x] = 0.f;
    const int gid = warp * G + grp;
    // every lane runs the same number of iterations (the group sum shuffles)
    for (int64_t e0 = 0; e0 < r.deg; e0 += NG) {
        const int64_t e = e0 + gid;
        const bool valid = e < r.deg;
        float kf[V], vf[V];
        if (valid) {
            const int64_t j = row_edge(g, r, p, e);
            Slice<T>::load(kb + j * D + sub * V, kf);
            Slice<T>::load(vb + j * D + sub * V, vf);
        } else {
#pragma unroll
            for (int x = 0; x < V; ++x) kf[x] = vf[x] = 0.f;
        }
        float s = 0.f;
#pragma unroll
        for (int x = 0; x < V; ++x) s = fmaf(qf[x], kf[x], s);
        s = group_sum<L>(s);
        if (valid) {
            const float mn = fmaxf(m, s);
            const float al = ex2(m - mn), pe = ex2(s - mn);
            l = l * al + pe;
#pragma unroll
            for (int x = 0; x < V; ++x) acc[x] = fmaf(pe, vf[x], acc[x] * al);
            m = mn;
        }
    }
    // merge the groups of the warp
#pragma unroll
    for (int o = L; o < 32; o <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, o);
        const float lo = __shfl_xor_sync(0xffffffffu, l, o);
        float ao[V];
#pragma unroll
        for (int x = 0; x < V; ++x) ao[x] = __shfl_xor_sync(0xffffffffu, acc[x], o);
        const float mn = fmaxf(m, mo);
        if (mn != -INFINITY) {
            const float w0 = ex2(m - mn), w1 = ex2(mo - mn);
            l = l * w0 + lo * w1;
#pragma unroll
            for (int x = 0; x < V; ++x) acc[x] = acc[x] * w0 + ao[x] * w1;
            m = mn;
        }
    }
    // ... then the warps of the CTA
    if (grp == 0) {
#pragma unroll
        for (int x = 0; x < V; ++x) s_acc[warp][sub * V + x] = acc[x];
        if (sub == 0) {
            s_m[warp] = m;
            s_l[warp] = l;
        }
    }
    __syncthreads();
    if (warp == 0) {
        float mt = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) mt = fmaxf(mt, s_m[w]);
        float lt = 0.f, o[V];
#pragma unroll
        for (int x = 0; x < V; ++x) o[x] = 0.f;
        if (mt != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kDecWarps; ++w) {
                const float f = s_m[w] == -INFINITY ? 0.f : ex2(s_m[w] - mt);
                lt = fmaf(s_l[w], f, lt);
#pragma unroll
                for (int x = 0; x < V; ++x) o[x] = fmaf(s_acc[w][sub * V + x], f, o[x]);
            }
        }
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
#pragma unroll
        for (int x = 0; x < V; ++x) o[x] *= inv;
        if (grp == 0) Slice<T>::store(out + bh * D + sub * V, o);
        if (lane == 0) lse[bh] = lt > 0.f ? (mt + lg2(lt)) * kLn2 : -INFINITY;
    }
}

template <typename T, int D>
sa_status launch_decode(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                        const int64_t *pos, const GraphView &g, float scale, sa_tensor *out,
                        float *lse, cudaStream_t s) {
    int *err = sa_device_error_word();
    if (!err) return SA_ERR_CUDA;
    const int64_t nblocks = q->B * q->H;
    if (nblocks > 0x7fffffffLL) return SA_ERR_UNSUPPORTED;
    SA_LAUNCH("decode", s,
              decode_kernel<T, D><<<(unsigned)nblocks, 32 * kDecWarps, 0, s>>>(
                  (const T *)q->ptr, (const T *)k->ptr, (const T *)v->ptr, pos, g, q->H, k->H,
                  k->T, scale * kLog2e, (T *)out->ptr, lse, err));
    SA_CUDA_TRY(cudaGetLastError());
    return SA_OK;
}

}  // namespace

sa_status sa_decode(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                    const int64_t *pos, const GraphView &g, float scale, sa_tensor *out,
                    float *lse, cudaStream_t s) {
    const bool bf = q->dtype == SA_BF16;
    switch (q->D) {
        case 32:
            return bf ? launch_decode<__nv_bfloat16, 32>(q, k, v, pos, g, scale, out, lse, s)
                      : launch_decode<float, 32>(q, k, v, pos, g, scale, out, lse, s);
        case 64:
            return bf ? launch_decode<__nv_bfloat16, 64>(q, k, v, pos, g, scale, out, lse, s)
                      : launch_decode<float, 64>(q, k, v, pos, g, scale, out, lse, s);
        case 128:
            return bf ? launch_decode<__nv_bfloat16, 128>(q, k, v, pos, g, scale, out, lse, s)
                      : launch_decode<float, 128>(q, k, v, pos, g, scale, out, lse, s);
    }
    return SA_ERR_UNSUPPORTED;
}
