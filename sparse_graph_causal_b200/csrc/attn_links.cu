// attn_links.cu -- the long distance links of a structured graph, as a second
// pass over the forward's result, in an order that keeps their K/V rows in L2.
//
// A distance link i -> i - o ("SpatialLM-Mini ...", section "How tokens
// choose whom to listen to": links of length 2^k) reads K and V rows that the
// sweep over the sequence touched o rows earlier.  When K and V exceed L2
// ("Longer Attention Span ...", Abstract: sequences of 160 M tokens on one
// GPU) and o is long, those rows have left L2 by then, so every long link of
// every row is a DRAM read.  The forward therefore runs in two passes:
//  1. the band kernel with the window and the links shorter than S rows, in
//     sequence order (their rows are still in L2), writing out and lse;
//  2. this kernel with the links of length >= S, all multiples of S.  With
//     C = S / 128 tiles, tile t reaches only tiles t - o/128 = t (mod C): the
//     tiles split into C classes of residue t mod C that share no K/V rows
//     between them.  Running the tiles class by class, each class's K/V rows
//     (T / C rows) stay in L2 while the class runs, so a long link is a DRAM
//     read about once per K/V row instead of once per edge.
// Pass 2 merges its edges into pass 1's row: with pass 1's (out_1, lse_1) and
// its own running max m, sum l and weighted sum acc (base 2),
//   M = max(lse_1 log2 e, m),  w_1 = 2^(lse_1 log2 e - M),  w_2 = 2^(m - M),
//   out = (out_1 w_1 + acc w_2) / (w_1 + l w_2),  lse = (M + log2(w_1 + l w_2)) ln 2,
// the online-softmax merge of two disjoint edge sets (out_1 is read back as
// stored, in the input's precision).
//
// CUDA cores only: no TMEM, no barrier between warps (layout and lane roles
// below).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sa_band.cuh"
#include "tc_common.cuh"

namespace {

constexpr int BM = 128;        // queries per tile
constexpr int kDS = 2;         // ring stages per warp
constexpr int kMinBlocks = 2;  // CTAs per SM the register budget must allow
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units, as in the band kernel

struct LinkArgs {
    int64_t T;
    int64_t H, Hkv;     // query and key/value heads (grouped-query attention)
    int64_t nt;         // tiles per slice
    int64_t C;          // classes (tiles)
    int64_t G;          // tiles per class, ceil(nt / C)
    int32_t n_off;
    int32_t offs[SA_MAX_OFFSETS];  // descending, each a multiple of 128 C
    const __nv_bfloat16 *q, *k, *v;
    __nv_bfloat16 *out;
    float *lse;
    float scale2;       // scale * log2(e)
};

// Shared memory: per warp a ring of DS stages, each the K rows and then the V
// rows of its 16 queries for one link (16 x 2D bytes each).  The 16-byte
// chunks of each 128-byte segment of a row (of the whole row when it is
// shorter) are permuted by XOR with the row's low bits, so that the lane
// pairs' 16-byte reads spread over all banks; the XOR never leaves the
// segment: kSeg chunks, a power of two.
template <int D, int DS>
struct LinkLayout {
    static constexpr int kRowBytes = 2 * D;
    static constexpr int kSeg = kRowBytes >= 128 ? 8 : kRowBytes / 16;  // chunks per segment
    static constexpr int kRows = 16;                       // queries per warp
    static constexpr int kPart = kRows * kRowBytes;        // K (or V) rows of one slot
    static constexpr int kStage = 2 * kPart;
    static constexpr int kWarpRing = DS * kStage;
    static constexpr int kWarps = 8;                       // 128 queries per CTA
    static constexpr int kAlloc = kWarps * kWarpRing;
    static_assert(kSeg == 2 || kSeg == 4 || kSeg == 8, "row segment");
    __device__ static uint32_t off(int x, int k) {         // row x, 16-byte chunk k
        return (uint32_t)(x * kRowBytes + (k / kSeg) * (16 * kSeg) +
                          (((k % kSeg) ^ (x % kSeg)) << 4));
    }
};

// One CTA of eight warps per 128-row tile; warp w owns queries 16w .. 16w+15
// and lanes 2x, 2x+1 share query x: each takes half of the columns (dot
// product halves summed by one shuffle, its half of the weighted value row
// accumulated).  A link's K and V rows for the 16 queries of a warp are 16
// contiguous rows of each tensor (keys i - o), copied with 16-byte cp.async
// copies into the warp's DS-stage ring, DS links ahead of their use.
template <int D, int DS, int MINB>
__global__ void __launch_bounds__(256, MINB) link_pass_kernel(const LinkArgs a) {
    using L = LinkLayout<D, DS>;
    constexpr int H2 = D / 2;              // columns per lane
    constexpr int NCH = H2 / 8;            // 16-byte chunks per lane and row
    constexpr int NIT = L::kPart / (32 * 16);  // copies per lane per tensor and slot
    extern __shared__ __align__(128) uint8_t smem_raw[];

    // this CTA's tile: slices in order, then class by class inside a slice
    // (32-bit: the launcher keeps the block count and T below 2^31)
    const uint32_t C = (uint32_t)a.C, G = (uint32_t)a.G, per_slice = C * G;
    const uint32_t bh = blockIdx.x / per_slice, rem = blockIdx.x - bh * per_slice;
    const uint32_t cls = rem / G, jt = rem - cls * G;
    const uint32_t t = jt * C + cls;
    if (t >= (uint32_t)a.nt) return;
    const int32_t T = (int32_t)a.T;
    const int32_t q0 = (int32_t)t * BM;
    const int32_t last = (q0 + BM - 1 < T - 1) ? q0 + BM - 1 : T - 1;
    // the links this tile's rows reach (the longest first: keys ascending)
    int nd = 0;
    for (int x = 0; x < a.n_off; ++x) nd += (a.offs[x] <= last) ? 1 : 0;
    if (nd == 0) return;  // no row of the tile has one: pass 1's result stands
    const int dfirst = a.n_off - nd;

    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int x = lane >> 1, hf = lane & 1;
    const int32_t i0 = q0 + 16 * w, i = i0 + x;
    const bool row_ok = i < T;
    const uint32_t H = (uint32_t)a.H, Hkv = (uint32_t)a.Hkv;
    const uint32_t kvbh = (bh / H) * Hkv + (bh % H) / (H / Hkv);
    const __nv_bfloat16 *kslice = a.k + (size_t)kvbh * (size_t)T * D;
    const __nv_bfloat16 *vslice = a.v + (size_t)kvbh * (size_t)T * D;
    const size_t grow = (size_t)bh * (size_t)T + (size_t)i;
    uint8_t *ring = smem_raw + w * L::kWarpRing;
    const uint32_t ring_s = tc::smem_u32(ring);

    // this lane's half of the q row
    uint32_t qw[H2 / 2];
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const uint4 w4 = row_ok ? __ldg((const uint4 *)(a.q + grow * D + hf * H2) + c)
                                : make_uint4(0, 0, 0, 0);
        qw[4 * c] = w4.x;
        qw[4 * c + 1] = w4.y;
        qw[4 * c + 2] = w4.z;
        qw[4 * c + 3] = w4.w;
    }

    // this lane's copies of a slot, the same for every slot: row xr of the
    // warp's 16, chunk kc; the destination in the stage and the source offset
    // from the slot's first key row
    int xr[NIT];
    uint32_t doff[NIT], soff[NIT];
#pragma unroll
    for (int it = 0; it < NIT; ++it) {
        const int b = (it * 32 + lane) * 16;
        xr[it] = b / L::kRowBytes;
        const int kc = (b % L::kRowBytes) / 16;
        doff[it] = L::off(xr[it], kc);
        soff[it] = (uint32_t)(xr[it] * D + 8 * kc);
    }
    // copies of slot d into stage st (nothing past the last slot, or for rows
    // before the link's reach or past the sequence); one commit group each
    auto issue = [&](int st, int d) {
        if (d < nd) {
            const int32_t kb = i0 - a.offs[dfirst + d];  // key of the warp's first query
            const int64_t kbd = (int64_t)kb * D;
            const uint32_t sk = ring_s + st * L::kStage, sv = sk + L::kPart;
#pragma unroll
            for (int it = 0; it < NIT; ++it) {
                if (kb + xr[it] >= 0 && i0 + xr[it] < T) {
                    const int64_t src = kbd + soff[it];
                    tc::cp_async16(sk + doff[it], kslice + src);
                    tc::cp_async16(sv + doff[it], vslice + src);
                }
            }
        }
        tc::cp_async_commit();
    };

    const float c2 = a.scale2;
    float m_run = -INFINITY, l_run = 0.f, acc[H2];
#pragma unroll
    for (int c = 0; c < H2; ++c) acc[c] = 0.f;
#pragma unroll
    for (int st = 0; st < DS; ++st) issue(st, st);
    for (int d = 0; d < nd; ++d) {
        const int st = d % DS;
        tc::cp_async_wait<DS - 1>();  // slot d has landed (this lane's copies)
        __syncwarp();                 // ... and every lane's
        const uint8_t *kr = ring + st * L::kStage, *vr = kr + L::kPart;
        // dot product: this lane's half, then the pair's sum
        float sp[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) sp[e] = 0.f;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const uint4 k4 = *(const uint4 *)(kr + L::off(x, hf * NCH + c));
            const uint32_t kw[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                sp[2 * e] = tc::fma_bf_lo(qw[4 * c + e], kw[e], sp[2 * e]);
                sp[2 * e + 1] = tc::fma_bf_hi(qw[4 * c + e], kw[e], sp[2 * e + 1]);
            }
        }
        float sdot = ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
        sdot += __shfl_xor_sync(0xffffffffu, sdot, 1);
        if (row_ok && i >= a.offs[dfirst + d]) {
            const float s = sdot * c2;
            if (s > m_run + kRescaleThreshold) {  // lazy rescale, as in the band kernel
                const float al = tc::ex2(m_run - s);  // 0 on the first edge
#pragma unroll
                for (int c = 0; c < H2; ++c) acc[c] *= al;
                l_run *= al;
                m_run = s;
            }
            const float pr = tc::ex2(s - m_run);
            l_run += pr;
            const uint32_t p2 = tc::pack_bf16x2(pr, pr);  // p rounded to bf16, as the band's P
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                const uint4 v4 = *(const uint4 *)(vr + L::off(x, hf * NCH + c));
                const uint32_t vw[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc[8 * c + 2 * e] = tc::fma_bf_lo(p2, vw[e], acc[8 * c + 2 * e]);
                    acc[8 * c + 2 * e + 1] = tc::fma_bf_hi(p2, vw[e], acc[8 * c + 2 * e + 1]);
                }
            }
        }
        __syncwarp();  // every lane is done with the stage: refill it
        issue(st, d + DS);
    }
    tc::cp_async_wait<0>();  // nothing stays in flight

    // merge with pass 1's row (rows without a link of this pass keep it)
    if (!row_ok || l_run == 0.f) return;
    const float l1 = a.lse[grow] * kLog2e;  // base 2; finite: every row holds itself
    const float M = fmaxf(l1, m_run);
    const float w1 = tc::ex2(l1 - M), w2 = tc::ex2(m_run - M);
    const float den = w1 + l_run * w2;
    const float inv = 1.f / den, f1 = w1 * inv, f2 = w2 * inv;
    __nv_bfloat16 *orow = a.out + grow * D + hf * H2;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const uint4 o4 = *(const uint4 *)(orow + 8 * c);
        const uint32_t ow[4] = {o4.x, o4.y, o4.z, o4.w};
        uint32_t nw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float lo = __uint_as_float(ow[e] << 16), hi = __uint_as_float(ow[e] & 0xffff0000u);
            nw[e] = tc::pack_bf16x2(fmaf(lo, f1, acc[8 * c + 2 * e] * f2),
                                    fmaf(hi, f1, acc[8 * c + 2 * e + 1] * f2));
        }
        *(uint4 *)(orow + 8 * c) = make_uint4(nw[0], nw[1], nw[2], nw[3]);
    }
    if (hf == 0) a.lse[grow] = (M + tc::lg2(den)) * kLn2;
}

template <int D, int DS, int MINB>
sa_status launch_link_pass(const LinkArgs &a, int64_t BH, cudaStream_t s) {
    using L = LinkLayout<D, DS>;
    const int64_t blocks = BH * a.C * a.G;
    if (blocks > 0x7fffffffLL || a.T >= ((int64_t)1 << 31)) return SA_ERR_UNSUPPORTED;
    SA_CUDA_TRY(sa_smem_optin((const void *)link_pass_kernel<D, DS, MINB>, L::kAlloc));
    SA_LAUNCH("link_pass", s,
              link_pass_kernel<D, DS, MINB><<<(unsigned)blocks, 32 * L::kWarps, L::kAlloc, s>>>(a));
    SA_CUDA_TRY(cudaGetLastError());
    return SA_OK;
}

}  // namespace

sa_status sa_link_pass(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                       const int64_t *offs, int n_off, int64_t span, float scale, sa_tensor *out,
                       float *lse, cudaStream_t s) {
    if (n_off < 1 || n_off > SA_MAX_OFFSETS || span < BM || span % BM != 0)
        return SA_ERR_INVALID_ARG;
    LinkArgs a{};
    a.T = q->T;
    a.H = q->H;
    a.Hkv = k->H;
    a.nt = (q->T + BM - 1) / BM;
    a.C = span / BM;
    a.G = (a.nt + a.C - 1) / a.C;
    a.n_off = n_off;
    for (int x = 0; x < n_off; ++x) {
        if (offs[x] % span != 0 || offs[x] >= q->T || (x > 0 && offs[x] >= offs[x - 1]))
            return SA_ERR_INVALID_ARG;
        a.offs[x] = (int32_t)offs[x];
    }
    a.q = (const __nv_bfloat16 *)q->ptr;
    a.k = (const __nv_bfloat16 *)k->ptr;
    a.v = (const __nv_bfloat16 *)v->ptr;
    a.out = (__nv_bfloat16 *)out->ptr;
    a.lse = lse;
    a.scale2 = scale * kLog2e;
    const int64_t BH = q->B * q->H;
    switch (q->D) {
        case 32: return launch_link_pass<32, kDS, kMinBlocks>(a, BH, s);
        case 64: return launch_link_pass<64, kDS, kMinBlocks>(a, BH, s);
        case 128: return launch_link_pass<128, kDS, 1>(a, BH, s);
    }
    return SA_ERR_UNSUPPORTED;
}
