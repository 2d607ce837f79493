// attn_band_bwd.cu -- backward on tcgen05 band tiles fused with the gathered
// edges.  Probabilities are recomputed from lse; two kernels with disjoint
// outputs and no float atomics, so results are bitwise reproducible:
//
//  band_bwd_dq   CTA = 128 queries [q0, q0+128).  Delta_i = dO_i . out_i is
//                computed per row and written for the second kernel.  Key
//                blocks of 64 from q0-W+1 (the forward's band in block
//                coordinates u = 64 b + c, row r keeps r <= u <= r+W-1):
//                S = Q K^T and dP = dO V^T in TMEM, dS = P (dP - Delta) in
//                shared memory (bf16), dQ += dS K in TMEM.
//  band_bwd_dkdv CTA = 128 keys [k0, k0+128).  Query blocks of 64 from k0
//                (v = i - k0 = 64 b + c, key row r keeps r <= v <= r+W-1):
//                S^T = K Q^T and dP^T = V dO^T in TMEM, P^T and dS^T in
//                shared memory, dV += P^T dO and dK += dS^T Q in TMEM.
//
// The other edges (2^k distance links or the non-window part of CSR lists)
// are diagonal blocks as in the forward: row r of a block belongs to query
// (or key) r; for a distance o the rows are one TMA box, for CSR lists 4-row
// TMA gathers of the row's slot.  They are accumulated on CUDA cores (fp32
// pairs) first and initialise the TMEM accumulators, which the band MMAs then
// add to.
//
// Warp roles (256 threads): 0 TMA producer, 1 TMEM allocator + MMA issuer,
// 2 diagonal-block producer (3 idle), 4-7 compute warpgroup (thread = owned
// row = TMEM lane).  Waits are bounded as in the forward.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "sa_band.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace {

constexpr int BM = 128;  // rows a CTA owns
constexpr int BB = 64;   // streamed block
constexpr float kLog2e = 1.4426950408889634f;

struct BwdArgs {
    int64_t T;
    int32_t W;
    int32_t kind;
    int32_t n_off;
    int64_t offs[SA_MAX_OFFSETS];  // descending
    const int64_t *rowptr;
    const int32_t *colidx;
    const int64_t *rev_rowptr;
    const int32_t *rev_colidx;
    const __nv_bfloat16 *q, *k, *v, *o, *dout;
    const float *lse;
    float *delta;
    __nv_bfloat16 *dq, *dk, *dv;
    float scale;
    float scale2;  // scale * log2(e)
    int *err;
};

__host__ __device__ constexpr int align1k(int x) { return (x + 1023) & ~1023; }

// ---------------------------------------------------------------- helpers

// Load a 128-row tile (two 64-row boxes per 64-column half) with a box-64 map.
template <int D>
__device__ __forceinline__ void tma_tile128(uint32_t dst, const void *map, int64_t row, int64_t bh,
                                            uint32_t bar) {
#pragma unroll
    for (int x = 0; x < D / 64; ++x)
#pragma unroll
        for (int h = 0; h < 2; ++h)
            tc::tma_load_3d(dst + x * (BM * 128) + h * (64 * 128), map, x * 64,
                            (int32_t)(row + 64 * h), (int32_t)bh, bar);
}

template <int D>
__device__ __forceinline__ void tma_block64(uint32_t dst, const void *map, int64_t row, int64_t bh,
                                            uint32_t bar) {
#pragma unroll
    for (int x = 0; x < D / 64; ++x)
        tc::tma_load_3d(dst + x * (BB * 128), map, x * 64, (int32_t)row, (int32_t)bh, bar);
}

// 16-byte chunk c of row r in a tile of `rows` rows (64-column halves stacked).
__device__ __forceinline__ uint32_t tile_off(int rows, int r, int c) {
    return (uint32_t)((c >> 3) * (rows * 128)) + tc::sw128_off((uint32_t)r, (uint32_t)(c & 7));
}

template <int D>
__device__ __forceinline__ void load_row_packed(const uint8_t *tile, int rows, int r, uint32_t *w) {
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        const uint4 x = *(const uint4 *)(tile + tile_off(rows, r, c));
        w[4 * c] = x.x;
        w[4 * c + 1] = x.y;
        w[4 * c + 2] = x.z;
        w[4 * c + 3] = x.w;
    }
}

// ---- fp32-pair versions (f32x2 FMA): a row of D values as D/2 pairs
// (elements 2e, 2e+1), four independent partial sums in the dot products.

__device__ __forceinline__ float sum4_f2(uint64_t s0, uint64_t s1, uint64_t s2, uint64_t s3) {
    return ((tc::f2lo(s0) + tc::f2hi(s0)) + (tc::f2lo(s1) + tc::f2hi(s1))) +
           ((tc::f2lo(s2) + tc::f2hi(s2)) + (tc::f2lo(s3) + tc::f2hi(s3)));
}

// a . b, both rows of swizzled tiles in shared memory (row r of each).
template <int D>
__device__ __forceinline__ float dot2_smem_smem(const uint8_t *ta, const uint8_t *tb, int rows,
                                                int r) {
    uint64_t s0 = 0ull, s1 = 0ull, s2 = 0ull, s3 = 0ull;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        const uint4 x = *(const uint4 *)(ta + tile_off(rows, r, c));
        const uint4 y = *(const uint4 *)(tb + tile_off(rows, r, c));
        s0 = tc::ffma2(tc::bf2_to_f2(x.x), tc::bf2_to_f2(y.x), s0);
        s1 = tc::ffma2(tc::bf2_to_f2(x.y), tc::bf2_to_f2(y.y), s1);
        s2 = tc::ffma2(tc::bf2_to_f2(x.z), tc::bf2_to_f2(y.z), s2);
        s3 = tc::ffma2(tc::bf2_to_f2(x.w), tc::bf2_to_f2(y.w), s3);
    }
    return sum4_f2(s0, s1, s2, s3);
}

// a . b, a = row r of a swizzled tile read in physical chunk order, b = row r
// of an unswizzled gathered tile read at the swizzled address.
template <int D>
__device__ __forceinline__ float dot2_phys_gathered(const uint8_t *ta, const uint8_t *tb, int rows,
                                                    int r) {
    uint64_t s0 = 0ull, s1 = 0ull, s2 = 0ull, s3 = 0ull;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        const uint4 x = *(const uint4 *)(ta + (c >> 3) * (rows * 128) + r * 128 + ((c & 7) << 4));
        const uint4 y = *(const uint4 *)(tb + tile_off(rows, r, c));
        s0 = tc::ffma2(tc::bf2_to_f2(x.x), tc::bf2_to_f2(y.x), s0);
        s1 = tc::ffma2(tc::bf2_to_f2(x.y), tc::bf2_to_f2(y.y), s1);
        s2 = tc::ffma2(tc::bf2_to_f2(x.z), tc::bf2_to_f2(y.z), s2);
        s3 = tc::ffma2(tc::bf2_to_f2(x.w), tc::bf2_to_f2(y.w), s3);
    }
    return sum4_f2(s0, s1, s2, s3);
}

// a . b, a already unpacked to pairs (chunk c in a2[4c .. 4c+3]), b row r of
// a tile read at the swizzled address.
template <int D>
__device__ __forceinline__ float dot2_reg_smem(const uint64_t *a2, const uint8_t *tile, int rows,
                                               int r) {
    uint64_t s0 = 0ull, s1 = 0ull, s2 = 0ull, s3 = 0ull;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        const uint4 y = *(const uint4 *)(tile + tile_off(rows, r, c));
        s0 = tc::ffma2(a2[4 * c], tc::bf2_to_f2(y.x), s0);
        s1 = tc::ffma2(a2[4 * c + 1], tc::bf2_to_f2(y.y), s1);
        s2 = tc::ffma2(a2[4 * c + 2], tc::bf2_to_f2(y.z), s2);
        s3 = tc::ffma2(a2[4 * c + 3], tc::bf2_to_f2(y.w), s3);
    }
    return sum4_f2(s0, s1, s2, s3);
}

// a . b, a packed bf16 pairs in registers, b row r of a tile.
template <int D>
__device__ __forceinline__ float dot2_packed_smem(const uint32_t *a, const uint8_t *tile, int rows,
                                                  int r) {
    uint64_t s0 = 0ull, s1 = 0ull, s2 = 0ull, s3 = 0ull;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        const uint4 y = *(const uint4 *)(tile + tile_off(rows, r, c));
        s0 = tc::ffma2(tc::bf2_to_f2(a[4 * c]), tc::bf2_to_f2(y.x), s0);
        s1 = tc::ffma2(tc::bf2_to_f2(a[4 * c + 1]), tc::bf2_to_f2(y.y), s1);
        s2 = tc::ffma2(tc::bf2_to_f2(a[4 * c + 2]), tc::bf2_to_f2(y.z), s2);
        s3 = tc::ffma2(tc::bf2_to_f2(a[4 * c + 3]), tc::bf2_to_f2(y.w), s3);
    }
    return sum4_f2(s0, s1, s2, s3);
}

// acc2 += a * (row r of a tile), pairs.
template <int D>
__device__ __forceinline__ void axpy2_smem(uint64_t *acc2, float a, const uint8_t *tile, int rows,
                                           int r) {
    const uint64_t a2 = tc::f2pack(a, a);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        const uint4 y = *(const uint4 *)(tile + tile_off(rows, r, c));
        acc2[4 * c] = tc::ffma2(a2, tc::bf2_to_f2(y.x), acc2[4 * c]);
        acc2[4 * c + 1] = tc::ffma2(a2, tc::bf2_to_f2(y.y), acc2[4 * c + 1]);
        acc2[4 * c + 2] = tc::ffma2(a2, tc::bf2_to_f2(y.z), acc2[4 * c + 2]);
        acc2[4 * c + 3] = tc::ffma2(a2, tc::bf2_to_f2(y.w), acc2[4 * c + 3]);
    }
}

// acc2 holds chunk t at logical chunk t ^ (r & 7) (per 64-column half): put it
// back in logical order through a D-float scratch row in shared memory.
template <int D>
__device__ __forceinline__ void unpermute_row2(uint64_t *acc2, float *scr_row, int r) {
    uint64_t *scr = (uint64_t *)scr_row;
#pragma unroll
    for (int t = 0; t < D / 8; ++t) {
        const int lc = (t & ~7) | ((t & 7) ^ (r & 7));
        *(ulonglong2 *)(scr + 4 * lc) = make_ulonglong2(acc2[4 * t], acc2[4 * t + 1]);
        *(ulonglong2 *)(scr + 4 * lc + 2) = make_ulonglong2(acc2[4 * t + 2], acc2[4 * t + 3]);
    }
    __syncwarp();
#pragma unroll
    for (int t = 0; t < D / 4; ++t) {
        const ulonglong2 f = *(const ulonglong2 *)(scr + 2 * t);
        acc2[2 * t] = f.x;
        acc2[2 * t + 1] = f.y;
    }
}

template <int D>
__device__ __forceinline__ void tmem_store_row2(uint32_t taddr, const uint64_t *acc2) {
#pragma unroll
    for (int c = 0; c < D; c += 32) {
        uint32_t w[32];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
            w[2 * x] = __float_as_uint(tc::f2lo(acc2[c / 2 + x]));
            w[2 * x + 1] = __float_as_uint(tc::f2hi(acc2[c / 2 + x]));
        }
        tc::tmem_st32(taddr + c, w);
    }
}

// TMEM row (D fp32 columns) * mul -> bf16 row in global memory.
template <int D>
__device__ __forceinline__ void tmem_row_to_global(uint32_t taddr, float mul, __nv_bfloat16 *dst,
                                                   bool store) {
#pragma unroll
    for (int c = 0; c < D; c += 32) {
        uint32_t w[32];
        tc::tmem_ld32(taddr + c, w);
        tc::tmem_ld_wait();
        if (store) {
#pragma unroll
            for (int x = 0; x < 32; x += 8) {
                uint4 o4;
                o4.x = tc::pack_bf16x2(__uint_as_float(w[x]) * mul, __uint_as_float(w[x + 1]) * mul);
                o4.y = tc::pack_bf16x2(__uint_as_float(w[x + 2]) * mul,
                                       __uint_as_float(w[x + 3]) * mul);
                o4.z = tc::pack_bf16x2(__uint_as_float(w[x + 4]) * mul,
                                       __uint_as_float(w[x + 5]) * mul);
                o4.w = tc::pack_bf16x2(__uint_as_float(w[x + 6]) * mul,
                                       __uint_as_float(w[x + 7]) * mul);
                *(uint4 *)(dst + c + x) = o4;
            }
        }
    }
}

// Write 64 bf16 values (from fp32) as row r of a 128 x 64 K-major SW128 tile.
__device__ __forceinline__ void store_row64_bf16(uint8_t *tile, int r, const float *x) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 w;
        w.x = tc::pack_bf16x2(x[8 * c], x[8 * c + 1]);
        w.y = tc::pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
        w.z = tc::pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
        w.w = tc::pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
        *(uint4 *)(tile + tc::sw128_off((uint32_t)r, (uint32_t)c)) = w;
    }
}

#define WAIT_OR(bar_, par_, action_)                                                   \
    if (!tc::mbar_wait((bar_), (par_), abort, a.err, SA_DEVERR_TIMEOUT)) {              \
        action_;                                                                       \
    }

// =================================================================== dQ

template <int D, int BS, int DS, int PB>
struct LayoutDQ {
    static constexpr int kRow = BM * D * 2, kBlk = BB * D * 2, kDSTile = BM * BB * 2;
    static constexpr int kQ = 0, kDO = kRow, kK = 2 * kRow, kV = kK + BS * kBlk;
    static constexpr int kDS = kV + BS * kBlk;
    static constexpr int kDiagK = kDS + PB * kDSTile;
    static constexpr int kDiagV = kDiagK + DS * kRow;
    static constexpr int kBars = kDiagV + DS * kRow;
    static constexpr int DSX = DS > 0 ? DS : 1;
    static constexpr int bQFull = 0, bBandFull = 1, bBandEmpty = bBandFull + BS;
    static constexpr int bSFull = bBandEmpty + BS, bSFree = bSFull + 2;
    static constexpr int bDSFull = bSFree + 2, bDSDone = bDSFull + PB;
    static constexpr int bInit = bDSDone + PB, bDiagFull = bInit + 1;
    static constexpr int bDiagEmpty = bDiagFull + DSX, bGroup = bDiagEmpty + DSX;
    static constexpr int nBars = bGroup + 1;
    static constexpr int kMisc = kBars + nBars * 8;
    static constexpr int kAlloc = kMisc + 16 + 1024;
    static constexpr uint32_t tS = 0, tDP = 128, tDQ = 256, kTmemCols = 512;
};

template <int D, int BS, int DS, int PB>
__global__ void __launch_bounds__(256, 1)
band_bwd_dq_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv,
                   const __grid_constant__ CUtensorMap tdo,
                   const __grid_constant__ CUtensorMap tkr,
                   const __grid_constant__ CUtensorMap tvr, const BwdArgs a) {
    using L = LayoutDQ<D, BS, DS, PB>;
    constexpr int DSX = L::DSX;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = tc::smem_u32(sm);
    uint32_t *tmem_slot = (uint32_t *)(sm + L::kMisc);
    volatile int *abort = (volatile int *)(sm + L::kMisc + 4);
    int *n_diag_s = (int *)(sm + L::kMisc + 8);
    auto bar = [&](int b) { return sbase + L::kBars + 8u * (uint32_t)b; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bh = blockIdx.y, q0 = (int64_t)blockIdx.x * BM, T = a.T;
    const int32_t W = a.W;
    const int64_t kb0 = q0 - W + 1;
    const int64_t last_key = (q0 + BM - 1 < T - 1) ? q0 + BM - 1 : T - 1;
    const int64_t nblk = (last_key - kb0) / BB + 1;
    const int64_t need0 = (int64_t)W - 1 - q0;
    const int64_t b_first = need0 > 0 ? need0 / BB : 0;
    const int n_band = (int)(nblk - b_first);

    if (tid == 0) {
        tc::mbar_init(bar(L::bQFull), 1);
        for (int s = 0; s < BS; ++s) {
            tc::mbar_init(bar(L::bBandFull + s), 1);
            tc::mbar_init(bar(L::bBandEmpty + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(bar(L::bSFull + s), 1);
            tc::mbar_init(bar(L::bSFree + s), 4);
        }
        for (int s = 0; s < PB; ++s) {
            tc::mbar_init(bar(L::bDSFull + s), 4);
            tc::mbar_init(bar(L::bDSDone + s), 1);
        }
        tc::mbar_init(bar(L::bInit), 4);
        tc::mbar_init(bar(L::bGroup), 128);  // 128-thread compute barrier (bounded)
        for (int s = 0; s < DSX; ++s) {
            tc::mbar_init(bar(L::bDiagFull + s), 1);
            tc::mbar_init(bar(L::bDiagEmpty + s), 4);
        }
        *abort = 0;
        *n_diag_s = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) tc::tmem_alloc(tc::smem_u32(tmem_slot), L::kTmemCols);
    __syncthreads();
    if (DS > 0 && warp >= 4) {
        int nd = 0;
        const int64_t i = q0 + (tid - 128);
        if (a.kind == 0) {
            for (int x = 0; x < a.n_off; ++x) nd += (a.offs[x] <= last_key) ? 1 : 0;
        } else if (i < T) {
            const int64_t deg = a.rowptr[i + 1] - a.rowptr[i];
            nd = (int)(deg - ((i + 1 < W) ? i + 1 : W));
        }
        atomicMax(n_diag_s, nd);
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_diag = DS > 0 ? *n_diag_s : 0;

    if (warp == 0) {
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(bar(L::bQFull), 2 * L::kRow);
            tma_tile128<D>(sbase + L::kQ, &tq, q0, bh, bar(L::bQFull));
            tma_tile128<D>(sbase + L::kDO, &tdo, q0, bh, bar(L::bQFull));
            for (int bl = 0; bl < n_band; ++bl) {
                const int st = bl % BS, use = bl / BS;
                if (use > 0) WAIT_OR(bar(L::bBandEmpty + st), (use - 1) & 1, break);
                const int64_t krow = kb0 + (b_first + bl) * BB;
                tc::mbar_arrive_expect_tx(bar(L::bBandFull + st), 2 * L::kBlk);
                tma_block64<D>(sbase + L::kK + st * L::kBlk, &tk, krow, bh, bar(L::bBandFull + st));
                tma_block64<D>(sbase + L::kV + st * L::kBlk, &tv, krow, bh, bar(L::bBandFull + st));
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idS = tc::idesc_bf16(BM, BB, false, false);
            const uint32_t idQ = tc::idesc_bf16(BM, D, false, true);
            bool ok = tc::mbar_wait(bar(L::bQFull), 0, abort, a.err, SA_DEVERR_TIMEOUT);
            auto issue = [&](int bl) -> bool {
                const int st = bl % BS, sb = bl & 1;
                if (!tc::mbar_wait(bar(L::bBandFull + st), (bl / BS) & 1, abort, a.err,
                                   SA_DEVERR_TIMEOUT))
                    return false;
                if (bl >= 2 && !tc::mbar_wait(bar(L::bSFree + sb), ((bl >> 1) - 1) & 1, abort,
                                              a.err, SA_DEVERR_TIMEOUT))
                    return false;
                tc::tc_fence_after();
                const uint32_t ka = sbase + L::kK + st * L::kBlk, va = sbase + L::kV + st * L::kBlk;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t offr = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                    const uint32_t offb = (kk >> 2) * (BB * 128) + (kk & 3) * 32;
                    tc::mma_bf16_ss(tmem + L::tS + sb * BB,
                                    tc::sdesc_sw128(sbase + L::kQ + offr, 16, 1024),
                                    tc::sdesc_sw128(ka + offb, 16, 1024), idS, kk > 0);
                    tc::mma_bf16_ss(tmem + L::tDP + sb * BB,
                                    tc::sdesc_sw128(sbase + L::kDO + offr, 16, 1024),
                                    tc::sdesc_sw128(va + offb, 16, 1024), idS, kk > 0);
                }
                tc::mma_commit(bar(L::bSFull + sb));
                return true;
            };
            if (ok && n_band > 0) ok = issue(0);
            for (int bl = 0; ok && bl < n_band; ++bl) {
                if (BS >= 2 && bl + 1 < n_band && !issue(bl + 1)) break;
                const int pb = bl % PB, st = bl % BS;
                if (bl == 0) WAIT_OR(bar(L::bInit), 0, break);
                WAIT_OR(bar(L::bDSFull + pb), (bl / PB) & 1, break);
                tc::tc_fence_after();
                const uint32_t dsa = sbase + L::kDS + pb * L::kDSTile;
                const uint32_t ka = sbase + L::kK + st * L::kBlk;
#pragma unroll
                for (int kk = 0; kk < BB / 16; ++kk)
                    tc::mma_bf16_ss(tmem + L::tDQ, tc::sdesc_sw128(dsa + kk * 32, 16, 1024),
                                    tc::sdesc_sw128(ka + kk * 16 * 128, BB * 128, 1024), idQ, 1u);
                tc::mma_commit(bar(L::bBandEmpty + st));
                tc::mma_commit(bar(L::bDSDone + pb));
                if (BS == 1 && bl + 1 < n_band && !issue(bl + 1)) break;
            }
        }
    } else if (warp == 2 || warp == 3) {
        // warp 2 stages the diagonal blocks; warp 3 has no role
        if (warp == 2 && DS > 0) {
            // CSR: lane l owns rows 4l .. 4l+3 (list start, residual count, next key)
            int64_t cstart[4] = {0, 0, 0, 0}, cres[4] = {0, 0, 0, 0};
            int32_t cj[4] = {0, 0, 0, 0};
            if (a.kind == 1) {
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int64_t i = q0 + 4 * lane + h;
                    if (i < T) {
                        cstart[h] = a.rowptr[i];
                        cres[h] = a.rowptr[i + 1] - cstart[h] - ((i + 1 < W) ? i + 1 : W);
                        if (cres[h] > 0) cj[h] = a.colidx[cstart[h]];
                    }
                }
            }
            for (int d = 0; d < n_diag; ++d) {
                const int st = d % DSX, use = d / DSX;
                const uint32_t kdst = sbase + L::kDiagK + st * L::kRow;
                const uint32_t vdst = sbase + L::kDiagV + st * L::kRow;
                if (use > 0) WAIT_OR(bar(L::bDiagEmpty + st), (use - 1) & 1, break);
                if (lane == 0) tc::mbar_arrive_expect_tx(bar(L::bDiagFull + st), 2 * L::kRow);
                if (a.kind == 0) {
                    if (lane == 0) {
                        const int64_t krow = q0 - a.offs[a.n_off - n_diag + d];
                        tma_tile128<D>(kdst, &tk, krow, bh, bar(L::bDiagFull + st));
                        tma_tile128<D>(vdst, &tv, krow, bh, bar(L::bDiagFull + st));
                    }
                } else {
                    int32_t rr[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const int64_t i = q0 + 4 * lane + h;
                        const int64_t j = d < cres[h] ? (int64_t)cj[h] : (i < T ? i : 0);
                        rr[h] = (int32_t)(bh * T + j);
                    }
#pragma unroll
                    for (int x = 0; x < D / 64; ++x) {
                        const uint32_t off = x * (BM * 128) + 4 * lane * 128;
                        tc::tma_gather4(kdst + off, &tkr, x * 64, rr[0], rr[1], rr[2], rr[3],
                                        bar(L::bDiagFull + st));
                        tc::tma_gather4(vdst + off, &tvr, x * 64, rr[0], rr[1], rr[2], rr[3],
                                        bar(L::bDiagFull + st));
                    }
#pragma unroll
                    for (int h = 0; h < 4; ++h)
                        if (d + 1 < cres[h]) cj[h] = a.colidx[cstart[h] + d + 1];
                }
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // compute warpgroup: thread r = owned row r = TMEM lane r
        const int r = tid - 128;
        const int64_t i = q0 + r;
        const bool row_ok = i < T;
        const size_t grow = (size_t)bh * (size_t)T + (size_t)i;
        const uint32_t lane_off = (uint32_t)((warp - 4) * 32) << 16;
        const uint32_t tS = tmem + lane_off + L::tS, tDP = tmem + lane_off + L::tDP;
        const uint32_t tDQ = tmem + lane_off + L::tDQ;
        const float c2 = a.scale2;
        const float lse2 = row_ok ? a.lse[grow] * kLog2e : 0.f;
        // the out row for Delta is fetched while Q and dO arrive
        uint4 orow4[D / 8];
#pragma unroll
        for (int c = 0; c < D / 8; ++c)
            orow4[c] = row_ok ? __ldg((const uint4 *)(a.o + grow * D) + c) : make_uint4(0, 0, 0, 0);
        bool ok = tc::mbar_wait(bar(L::bQFull), 0, abort, a.err, SA_DEVERR_TIMEOUT);
        float Delta = 0.f;
        if (ok) {
            // Delta_i = dO_i . out_i
            uint32_t dor[D / 2];
            load_row_packed<D>(sm + L::kDO, BM, r, dor);
            if (row_ok) {
                uint64_t d0 = 0ull, d1 = 0ull, d2 = 0ull, d3 = 0ull;
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    d0 = tc::ffma2(tc::bf2_to_f2(dor[4 * c]), tc::bf2_to_f2(orow4[c].x), d0);
                    d1 = tc::ffma2(tc::bf2_to_f2(dor[4 * c + 1]), tc::bf2_to_f2(orow4[c].y), d1);
                    d2 = tc::ffma2(tc::bf2_to_f2(dor[4 * c + 2]), tc::bf2_to_f2(orow4[c].z), d2);
                    d3 = tc::ffma2(tc::bf2_to_f2(dor[4 * c + 3]), tc::bf2_to_f2(orow4[c].w), d3);
                }
                Delta = sum4_f2(d0, d1, d2, d3);
                a.delta[grow] = Delta;
            }
            // diagonal blocks (fp32 pairs)
            uint64_t acc2[D / 2];
#pragma unroll
            for (int x = 0; x < D / 2; ++x) acc2[x] = 0ull;
            if (DS > 0 && n_diag > 0) {
                if (a.kind == 0) {
                    // distance links: swizzled tiles, q in logical chunk order
                    uint64_t q2[D / 2];
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) {
                        const uint4 x = *(const uint4 *)(sm + L::kQ + tile_off(BM, r, c));
                        q2[4 * c] = tc::bf2_to_f2(x.x);
                        q2[4 * c + 1] = tc::bf2_to_f2(x.y);
                        q2[4 * c + 2] = tc::bf2_to_f2(x.z);
                        q2[4 * c + 3] = tc::bf2_to_f2(x.w);
                    }
                    for (int d = 0; d < n_diag; ++d) {
                        const int st = d % DSX;
                        WAIT_OR(bar(L::bDiagFull + st), (d / DSX) & 1, ok = false; break);
                        if (row_ok && i >= a.offs[a.n_off - n_diag + d]) {
                            const uint8_t *kt = sm + L::kDiagK + st * L::kRow;
                            const uint8_t *vt = sm + L::kDiagV + st * L::kRow;
                            const float p =
                                tc::ex2(fmaf(dot2_reg_smem<D>(q2, kt, BM, r), c2, -lse2));
                            const float ds = p * (dot2_packed_smem<D>(dor, vt, BM, r) - Delta);
                            axpy2_smem<D>(acc2, ds, kt, BM, r);
                        }
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(bar(L::bDiagEmpty + st));
                    }
                } else {
                    // CSR gathers are unswizzled: pair them with the physical
                    // chunk order of the swizzled q and dO rows (see the forward)
                    int64_t resid = 0;
                    if (row_ok)
                        resid = (a.rowptr[i + 1] - a.rowptr[i]) - ((i + 1 < W) ? i + 1 : W);
                    for (int d = 0; d < n_diag; ++d) {
                        const int st = d % DSX;
                        WAIT_OR(bar(L::bDiagFull + st), (d / DSX) & 1, ok = false; break);
                        if (row_ok && d < resid) {
                            const uint8_t *kt = sm + L::kDiagK + st * L::kRow;
                            const uint8_t *vt = sm + L::kDiagV + st * L::kRow;
                            const float p = tc::ex2(
                                fmaf(dot2_phys_gathered<D>(sm + L::kQ, kt, BM, r), c2, -lse2));
                            const float ds =
                                p * (dot2_phys_gathered<D>(sm + L::kDO, vt, BM, r) - Delta);
                            axpy2_smem<D>(acc2, ds, kt, BM, r);
                        }
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(bar(L::bDiagEmpty + st));
                    }
                    tc::mbar_arrive(bar(L::bGroup));
                    if (!tc::mbar_wait(bar(L::bGroup), 0, abort, a.err, SA_DEVERR_TIMEOUT)) ok = false;
                    unpermute_row2<D>(acc2, (float *)(sm + L::kDiagK) + (size_t)r * D, r);
                }
            }
            tmem_store_row2<D>(tDQ, acc2);
            tc::tmem_st_wait();
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar(L::bInit));

        // band blocks
        for (int bl = 0; ok && bl < n_band; ++bl) {
            const int sb = bl & 1, pb = bl % PB;
            const int64_t u0 = (b_first + bl) * BB;
            WAIT_OR(bar(L::bSFull + sb), (bl >> 1) & 1, ok = false; break);
            tc::tc_fence_after();
            float s[BB], dp[BB];
            tc::tmem_ld32(tS + sb * BB, (uint32_t *)s);
            tc::tmem_ld32(tS + sb * BB + 32, (uint32_t *)(s + 32));
            tc::tmem_ld32(tDP + sb * BB, (uint32_t *)dp);
            tc::tmem_ld32(tDP + sb * BB + 32, (uint32_t *)(dp + 32));
            tc::tmem_ld_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(L::bSFree + sb));
            const bool need_mask = (u0 < BM - 1) || (u0 + BB - 1 > (int64_t)W - 1) ||
                                   (u0 + q0 < (int64_t)W - 1);
            if (need_mask) {
                // keep columns [c_lo, c_hi]: r <= u <= r+W-1 and key >= 0
                const int64_t lo = ((int64_t)r > (int64_t)W - 1 - q0) ? r : (int64_t)W - 1 - q0;
                const int64_t hi = (int64_t)r + W - 1;
                const int c_lo = (int)(lo - u0 < 0 ? 0 : (lo - u0 > BB ? BB : lo - u0));
                const int c_hi = (int)(hi - u0 > BB - 1 ? BB - 1 : (hi - u0 < -1 ? -1 : hi - u0));
                // 16-column chunks outside every kept range of this warp: dS = 0
#pragma unroll
                for (int c16 = 0; c16 < BB / 16; ++c16) {
                    if (__any_sync(0xffffffffu, c_lo <= 16 * c16 + 15 && c_hi >= 16 * c16)) {
#pragma unroll
                        for (int c = 16 * c16; c < 16 * c16 + 16; ++c) {
                            const float p =
                                (c >= c_lo && c <= c_hi) ? tc::ex2(fmaf(s[c], c2, -lse2)) : 0.f;
                            s[c] = p * (dp[c] - Delta);  // dS
                        }
                    } else {
#pragma unroll
                        for (int c = 16 * c16; c < 16 * c16 + 16; ++c) s[c] = 0.f;
                    }
                }
            } else {
#pragma unroll
                for (int c = 0; c < BB; ++c) s[c] = tc::ex2(fmaf(s[c], c2, -lse2)) * (dp[c] - Delta);
            }
            if (bl >= PB) WAIT_OR(bar(L::bDSDone + pb), ((bl - PB) / PB) & 1, ok = false; break);
            store_row64_bf16(sm + L::kDS + pb * L::kDSTile, r, s);
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(L::bDSFull + pb));
        }
        if (ok && n_band > 0) {
            const int lb = n_band - 1;
            ok = tc::mbar_wait(bar(L::bDSDone + lb % PB), (lb / PB) & 1, abort, a.err,
                               SA_DEVERR_TIMEOUT);
        }
        if (ok) {
            tc::tc_fence_after();
            tmem_row_to_global<D>(tDQ, a.scale, a.dq + grow * D, row_ok);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, L::kTmemCols);
    }
}

// ================================================================= dK/dV

template <int D, int BS, int DS, int PB>
struct LayoutDKV {
    static constexpr int kRow = BM * D * 2, kBlk = BB * D * 2, kPTile = BM * BB * 2;
    static constexpr int kK = 0, kV = kRow, kQ = 2 * kRow, kDO = kQ + BS * kBlk;
    static constexpr int kLse = kDO + BS * kBlk, kDel = kLse + BS * 256;
    static constexpr int kP = align1k(kDel + BS * 256), kDS = kP + PB * kPTile;
    static constexpr int kDiagQ = kDS + PB * kPTile, kDiagDO = kDiagQ + DS * kRow;
    static constexpr int kBars = kDiagDO + DS * kRow;
    static constexpr int DSX = DS > 0 ? DS : 1;
    static constexpr int bKVFull = 0, bBandFull = 1, bBandEmpty = bBandFull + BS;
    static constexpr int bSFull = bBandEmpty + BS, bSFree = bSFull + 2;
    static constexpr int bPFull = bSFree + 2, bPDone = bPFull + PB;
    static constexpr int bInit = bPDone + PB, bDiagFull = bInit + 1;
    static constexpr int bDiagEmpty = bDiagFull + DSX, bGroup = bDiagEmpty + DSX;
    static constexpr int nBars = bGroup + 1;
    static constexpr int kMisc = kBars + nBars * 8;
    static constexpr int kAlloc = kMisc + 16 + 1024;
    static constexpr uint32_t tS = 0, tDP = 128, tDV = 256, tDK = 256 + D, kTmemCols = 512;
};

template <int D, int BS, int DS, int PB>
__global__ void __launch_bounds__(256, 1)
band_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv,
                     const __grid_constant__ CUtensorMap tdo,
                     const __grid_constant__ CUtensorMap tqr,
                     const __grid_constant__ CUtensorMap tdor, const BwdArgs a) {
    using L = LayoutDKV<D, BS, DS, PB>;
    constexpr int DSX = L::DSX;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = tc::smem_u32(sm);
    uint32_t *tmem_slot = (uint32_t *)(sm + L::kMisc);
    volatile int *abort = (volatile int *)(sm + L::kMisc + 4);
    int *n_diag_s = (int *)(sm + L::kMisc + 8);
    auto bar = [&](int b) { return sbase + L::kBars + 8u * (uint32_t)b; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bh = blockIdx.y, k0 = (int64_t)blockIdx.x * BM, T = a.T;
    const int32_t W = a.W;
    // queries k0 .. min(T-1, k0+127+W-1) in blocks of 64 from k0
    const int64_t vmax_w = (int64_t)BM - 1 + W - 1, vmax_t = T - 1 - k0;
    const int64_t vmax = vmax_w < vmax_t ? vmax_w : vmax_t;
    const int n_band = (int)(vmax / BB + 1);

    if (tid == 0) {
        tc::mbar_init(bar(L::bKVFull), 1);
        for (int s = 0; s < BS; ++s) {
            // TMA bytes + the 32 producer lanes that stage lse and Delta
            tc::mbar_init(bar(L::bBandFull + s), 33);
            tc::mbar_init(bar(L::bBandEmpty + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(bar(L::bSFull + s), 1);
            tc::mbar_init(bar(L::bSFree + s), 4);
        }
        for (int s = 0; s < PB; ++s) {
            tc::mbar_init(bar(L::bPFull + s), 4);
            tc::mbar_init(bar(L::bPDone + s), 1);
        }
        tc::mbar_init(bar(L::bInit), 4);
        tc::mbar_init(bar(L::bGroup), 128);  // 128-thread compute barrier (bounded)
        for (int s = 0; s < DSX; ++s) {
            tc::mbar_init(bar(L::bDiagFull + s), 1);
            tc::mbar_init(bar(L::bDiagEmpty + s), 4);
        }
        *abort = 0;
        *n_diag_s = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) tc::tmem_alloc(tc::smem_u32(tmem_slot), L::kTmemCols);
    __syncthreads();
    if (DS > 0 && warp >= 4) {
        int nd = 0;
        const int64_t j = k0 + (tid - 128);
        if (a.kind == 0) {
            for (int x = 0; x < a.n_off; ++x) nd += (k0 + a.offs[x] <= T - 1) ? 1 : 0;
        } else if (j < T) {
            const int64_t deg = a.rev_rowptr[j + 1] - a.rev_rowptr[j];
            nd = (int)(deg - ((T - j < W) ? T - j : W));
        }
        atomicMax(n_diag_s, nd);
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_diag = DS > 0 ? *n_diag_s : 0;
    // distance list of this tile: the n_diag smallest offsets with k0 + o <= T-1,
    // taken in descending order (as stored)
    const int off_first = a.n_off - n_diag;

    if (warp == 0) {
        // lane 0 issues the TMA copies; all 32 lanes stage lse (base 2) and
        // Delta of the block's 64 queries (zero past the end of the sequence)
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(bar(L::bKVFull), 2 * L::kRow);
            tma_tile128<D>(sbase + L::kK, &tk, k0, bh, bar(L::bKVFull));
            tma_tile128<D>(sbase + L::kV, &tv, k0, bh, bar(L::bKVFull));
        }
        for (int bl = 0; bl < n_band; ++bl) {
            const int st = bl % BS, use = bl / BS;
            if (use > 0) WAIT_OR(bar(L::bBandEmpty + st), (use - 1) & 1, break);
            const int64_t qrow = k0 + (int64_t)bl * BB;
            if (lane == 0) {
                tc::mbar_arrive_expect_tx(bar(L::bBandFull + st), 2 * L::kBlk);
                tma_block64<D>(sbase + L::kQ + st * L::kBlk, &tq, qrow, bh, bar(L::bBandFull + st));
                tma_block64<D>(sbase + L::kDO + st * L::kBlk, &tdo, qrow, bh,
                               bar(L::bBandFull + st));
            }
            float *ls = (float *)(sm + L::kLse + st * 256), *dl = (float *)(sm + L::kDel + st * 256);
            for (int c = lane; c < BB; c += 32) {
                const int64_t i = qrow + c;
                const size_t gi = (size_t)bh * (size_t)T + (size_t)i;
                ls[c] = i < T ? a.lse[gi] * kLog2e : 0.f;
                dl[c] = i < T ? a.delta[gi] : 0.f;
            }
            tc::mbar_arrive(bar(L::bBandFull + st));
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idS = tc::idesc_bf16(BM, BB, false, false);
            const uint32_t idG = tc::idesc_bf16(BM, D, false, true);
            bool ok = tc::mbar_wait(bar(L::bKVFull), 0, abort, a.err, SA_DEVERR_TIMEOUT);
            auto issue = [&](int bl) -> bool {
                const int st = bl % BS, sb = bl & 1;
                if (!tc::mbar_wait(bar(L::bBandFull + st), (bl / BS) & 1, abort, a.err,
                                   SA_DEVERR_TIMEOUT))
                    return false;
                if (bl >= 2 && !tc::mbar_wait(bar(L::bSFree + sb), ((bl >> 1) - 1) & 1, abort,
                                              a.err, SA_DEVERR_TIMEOUT))
                    return false;
                tc::tc_fence_after();
                const uint32_t qa = sbase + L::kQ + st * L::kBlk, da = sbase + L::kDO + st * L::kBlk;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t offr = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                    const uint32_t offb = (kk >> 2) * (BB * 128) + (kk & 3) * 32;
                    tc::mma_bf16_ss(tmem + L::tS + sb * BB,
                                    tc::sdesc_sw128(sbase + L::kK + offr, 16, 1024),
                                    tc::sdesc_sw128(qa + offb, 16, 1024), idS, kk > 0);
                    tc::mma_bf16_ss(tmem + L::tDP + sb * BB,
                                    tc::sdesc_sw128(sbase + L::kV + offr, 16, 1024),
                                    tc::sdesc_sw128(da + offb, 16, 1024), idS, kk > 0);
                }
                tc::mma_commit(bar(L::bSFull + sb));
                return true;
            };
            if (ok && n_band > 0) ok = issue(0);
            for (int bl = 0; ok && bl < n_band; ++bl) {
                if (BS >= 2 && bl + 1 < n_band && !issue(bl + 1)) break;
                const int pb = bl % PB, st = bl % BS;
                if (bl == 0) WAIT_OR(bar(L::bInit), 0, break);
                WAIT_OR(bar(L::bPFull + pb), (bl / PB) & 1, break);
                tc::tc_fence_after();
                const uint32_t pa = sbase + L::kP + pb * L::kPTile;
                const uint32_t dsa = sbase + L::kDS + pb * L::kPTile;
                const uint32_t qa = sbase + L::kQ + st * L::kBlk, da = sbase + L::kDO + st * L::kBlk;
#pragma unroll
                for (int kk = 0; kk < BB / 16; ++kk) {
                    tc::mma_bf16_ss(tmem + L::tDV, tc::sdesc_sw128(pa + kk * 32, 16, 1024),
                                    tc::sdesc_sw128(da + kk * 16 * 128, BB * 128, 1024), idG, 1u);
                    tc::mma_bf16_ss(tmem + L::tDK, tc::sdesc_sw128(dsa + kk * 32, 16, 1024),
                                    tc::sdesc_sw128(qa + kk * 16 * 128, BB * 128, 1024), idG, 1u);
                }
                tc::mma_commit(bar(L::bBandEmpty + st));
                tc::mma_commit(bar(L::bPDone + pb));
                if (BS == 1 && bl + 1 < n_band && !issue(bl + 1)) break;
            }
        }
    } else if (warp == 2 || warp == 3) {
        // warp 2 stages the diagonal blocks; warp 3 has no role
        if (warp == 2 && DS > 0) {
            // CSR: lane l owns key rows 4l .. 4l+3: start of the residual part of
            // their transpose lists (after the band queries j .. j+W-1), its
            // length, and the next query
            int64_t cstart[4] = {0, 0, 0, 0}, cres[4] = {0, 0, 0, 0};
            int32_t cj[4] = {0, 0, 0, 0};
            if (a.kind == 1) {
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int64_t j = k0 + 4 * lane + h;
                    if (j < T) {
                        const int64_t nb = (T - j < W) ? T - j : W;
                        cstart[h] = a.rev_rowptr[j] + nb;
                        cres[h] = a.rev_rowptr[j + 1] - cstart[h];
                        if (cres[h] > 0) cj[h] = a.rev_colidx[cstart[h]];
                    }
                }
            }
            for (int d = 0; d < n_diag; ++d) {
                const int st = d % DSX, use = d / DSX;
                const uint32_t qdst = sbase + L::kDiagQ + st * L::kRow;
                const uint32_t ddst = sbase + L::kDiagDO + st * L::kRow;
                if (use > 0) WAIT_OR(bar(L::bDiagEmpty + st), (use - 1) & 1, break);
                if (lane == 0) tc::mbar_arrive_expect_tx(bar(L::bDiagFull + st), 2 * L::kRow);
                if (a.kind == 0) {
                    if (lane == 0) {
                        const int64_t qrow = k0 + a.offs[off_first + d];
                        tma_tile128<D>(qdst, &tq, qrow, bh, bar(L::bDiagFull + st));
                        tma_tile128<D>(ddst, &tdo, qrow, bh, bar(L::bDiagFull + st));
                    }
                } else {
                    int32_t rr[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const int64_t j = k0 + 4 * lane + h;
                        const int64_t i = d < cres[h] ? (int64_t)cj[h] : (j < T ? j : 0);
                        rr[h] = (int32_t)(bh * T + i);
                    }
#pragma unroll
                    for (int x = 0; x < D / 64; ++x) {
                        const uint32_t off = x * (BM * 128) + 4 * lane * 128;
                        tc::tma_gather4(qdst + off, &tqr, x * 64, rr[0], rr[1], rr[2], rr[3],
                                        bar(L::bDiagFull + st));
                        tc::tma_gather4(ddst + off, &tdor, x * 64, rr[0], rr[1], rr[2], rr[3],
                                        bar(L::bDiagFull + st));
                    }
#pragma unroll
                    for (int h = 0; h < 4; ++h)
                        if (d + 1 < cres[h]) cj[h] = a.rev_colidx[cstart[h] + d + 1];
                }
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // compute warpgroup: thread r = owned row r = TMEM lane r
        const int r = tid - 128;
        const int64_t j = k0 + r;
        const bool row_ok = j < T;
        const size_t grow = (size_t)bh * (size_t)T + (size_t)j;
        const uint32_t lane_off = (uint32_t)((warp - 4) * 32) << 16;
        const uint32_t tS = tmem + lane_off + L::tS, tDP = tmem + lane_off + L::tDP;
        const uint32_t tDV = tmem + lane_off + L::tDV, tDK = tmem + lane_off + L::tDK;
        const float c2 = a.scale2;
        bool ok = tc::mbar_wait(bar(L::bKVFull), 0, abort, a.err, SA_DEVERR_TIMEOUT);
        if (ok) {
            // diagonal blocks (fp32 pairs); lse and Delta of the linked query
            // are loaded one block ahead
            uint64_t adk2[D / 2], adv2[D / 2];
#pragma unroll
            for (int x = 0; x < D / 2; ++x) adk2[x] = adv2[x] = 0ull;
            const size_t gbh = (size_t)bh * (size_t)T;
            if (DS > 0 && n_diag > 0) {
                if (a.kind == 0) {
                    // distance links: query j + o, swizzled tiles read in logical order
                    auto query_of = [&](int d) -> int64_t {
                        if (!row_ok || d >= n_diag) return -1;
                        const int64_t cand = j + a.offs[off_first + d];
                        return cand < T ? cand : -1;
                    };
                    int64_t i_cur = query_of(0);
                    float lse_cur = i_cur >= 0 ? a.lse[gbh + i_cur] : 0.f;
                    float del_cur = i_cur >= 0 ? a.delta[gbh + i_cur] : 0.f;
                    for (int d = 0; d < n_diag; ++d) {
                        const int64_t i_nxt = query_of(d + 1);
                        const float lse_nxt = i_nxt >= 0 ? a.lse[gbh + i_nxt] : 0.f;
                        const float del_nxt = i_nxt >= 0 ? a.delta[gbh + i_nxt] : 0.f;
                        const int st = d % DSX;
                        WAIT_OR(bar(L::bDiagFull + st), (d / DSX) & 1, ok = false; break);
                        if (i_cur >= 0) {
                            const uint8_t *qt = sm + L::kDiagQ + st * L::kRow;
                            const uint8_t *dt = sm + L::kDiagDO + st * L::kRow;
                            const float sdot = dot2_smem_smem<D>(qt, sm + L::kK, BM, r);
                            const float dpdot = dot2_smem_smem<D>(dt, sm + L::kV, BM, r);
                            const float p = tc::ex2(fmaf(sdot, c2, -lse_cur * kLog2e));
                            const float ds = p * (dpdot - del_cur);
                            axpy2_smem<D>(adv2, p, dt, BM, r);
                            axpy2_smem<D>(adk2, ds, qt, BM, r);
                        }
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(bar(L::bDiagEmpty + st));
                        i_cur = i_nxt;
                        lse_cur = lse_nxt;
                        del_cur = del_nxt;
                    }
                } else {
                    // CSR gathers are unswizzled: the key's k and v rows read in
                    // physical chunk order pair with them (see the forward)
                    int64_t rs = 0, nb = 0, resid = 0;
                    if (row_ok) {
                        rs = a.rev_rowptr[j];
                        nb = (T - j < W) ? T - j : W;
                        resid = a.rev_rowptr[j + 1] - rs - nb;
                    }
                    // query of slot d (-1 if none): the list entry two slots
                    // ahead, lse and Delta one slot ahead
                    auto query_of = [&](int d) -> int64_t {
                        return (row_ok && d < resid) ? (int64_t)a.rev_colidx[rs + nb + d] : -1;
                    };
                    int64_t i_cur = query_of(0), i_nxt = query_of(1);
                    float lse_cur = i_cur >= 0 ? a.lse[gbh + i_cur] : 0.f;
                    float del_cur = i_cur >= 0 ? a.delta[gbh + i_cur] : 0.f;
                    for (int d = 0; d < n_diag; ++d) {
                        const int64_t i_n2 = query_of(d + 2);
                        const float lse_nxt = i_nxt >= 0 ? a.lse[gbh + i_nxt] : 0.f;
                        const float del_nxt = i_nxt >= 0 ? a.delta[gbh + i_nxt] : 0.f;
                        const int st = d % DSX;
                        WAIT_OR(bar(L::bDiagFull + st), (d / DSX) & 1, ok = false; break);
                        if (i_cur >= 0) {
                            const uint8_t *qt = sm + L::kDiagQ + st * L::kRow;
                            const uint8_t *dt = sm + L::kDiagDO + st * L::kRow;
                            const float sdot = dot2_phys_gathered<D>(sm + L::kK, qt, BM, r);
                            const float dpdot = dot2_phys_gathered<D>(sm + L::kV, dt, BM, r);
                            const float p = tc::ex2(fmaf(sdot, c2, -lse_cur * kLog2e));
                            const float ds = p * (dpdot - del_cur);
                            axpy2_smem<D>(adv2, p, dt, BM, r);
                            axpy2_smem<D>(adk2, ds, qt, BM, r);
                        }
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(bar(L::bDiagEmpty + st));
                        i_cur = i_nxt;
                        i_nxt = i_n2;
                        lse_cur = lse_nxt;
                        del_cur = del_nxt;
                    }
                    tc::mbar_arrive(bar(L::bGroup));
                    if (!tc::mbar_wait(bar(L::bGroup), 0, abort, a.err, SA_DEVERR_TIMEOUT)) ok = false;
                    float *scr = (float *)(sm + L::kDiagQ);
                    unpermute_row2<D>(adv2, scr + (size_t)r * D, r);
                    unpermute_row2<D>(adk2, scr + (size_t)(BM + r) * D, r);
                }
            }
            tmem_store_row2<D>(tDV, adv2);
            tmem_store_row2<D>(tDK, adk2);
            tc::tmem_st_wait();
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar(L::bInit));

        for (int bl = 0; ok && bl < n_band; ++bl) {
            const int sb = bl & 1, pb = bl % PB, st = bl % BS;
            const int64_t v0 = (int64_t)bl * BB;
            WAIT_OR(bar(L::bSFull + sb), (bl >> 1) & 1, ok = false; break);
            tc::tc_fence_after();
            float s[BB], dp[BB];
            tc::tmem_ld32(tS + sb * BB, (uint32_t *)s);
            tc::tmem_ld32(tS + sb * BB + 32, (uint32_t *)(s + 32));
            tc::tmem_ld32(tDP + sb * BB, (uint32_t *)dp);
            tc::tmem_ld32(tDP + sb * BB + 32, (uint32_t *)(dp + 32));
            tc::tmem_ld_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(L::bSFree + sb));
            const float *lse_s = (const float *)(sm + L::kLse + st * 256);
            const float *del_s = (const float *)(sm + L::kDel + st * 256);
            const bool need_mask = (v0 < BM - 1) || (v0 + BB - 1 > (int64_t)W - 1) ||
                                   (k0 + v0 + BB - 1 > T - 1);
            if (need_mask) {
                // keep columns [c_lo, c_hi]: r <= v <= r+W-1 and query < T
                const int64_t vlim = T - 1 - k0;
                int64_t hi = (int64_t)r + W - 1;
                if (hi > vlim) hi = vlim;
                const int64_t lo = r;
                const int c_lo = (int)(lo - v0 < 0 ? 0 : (lo - v0 > BB ? BB : lo - v0));
                const int c_hi = (int)(hi - v0 > BB - 1 ? BB - 1 : (hi - v0 < -1 ? -1 : hi - v0));
                // 16-column chunks outside every kept range of this warp: P = dS = 0
#pragma unroll
                for (int c16 = 0; c16 < BB / 16; ++c16) {
                    if (__any_sync(0xffffffffu, c_lo <= 16 * c16 + 15 && c_hi >= 16 * c16)) {
#pragma unroll
                        for (int c = 16 * c16; c < 16 * c16 + 16; ++c) {
                            const float p = (c >= c_lo && c <= c_hi)
                                                ? tc::ex2(fmaf(s[c], c2, -lse_s[c]))
                                                : 0.f;
                            s[c] = p;
                            dp[c] = p * (dp[c] - del_s[c]);
                        }
                    } else {
#pragma unroll
                        for (int c = 16 * c16; c < 16 * c16 + 16; ++c) s[c] = dp[c] = 0.f;
                    }
                }
            } else {
#pragma unroll
                for (int c = 0; c < BB; ++c) {
                    const float p = tc::ex2(fmaf(s[c], c2, -lse_s[c]));
                    s[c] = p;
                    dp[c] = p * (dp[c] - del_s[c]);
                }
            }
            if (bl >= PB) WAIT_OR(bar(L::bPDone + pb), ((bl - PB) / PB) & 1, ok = false; break);
            store_row64_bf16(sm + L::kP + pb * L::kPTile, r, s);
            store_row64_bf16(sm + L::kDS + pb * L::kPTile, r, dp);
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(L::bPFull + pb));
        }
        if (ok && n_band > 0) {
            const int lb = n_band - 1;
            ok = tc::mbar_wait(bar(L::bPDone + lb % PB), (lb / PB) & 1, abort, a.err,
                               SA_DEVERR_TIMEOUT);
        }
        if (ok) {
            tc::tc_fence_after();
            tmem_row_to_global<D>(tDV, 1.f, a.dv + grow * D, row_ok);
            tmem_row_to_global<D>(tDK, a.scale, a.dk + grow * D, row_ok);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, L::kTmemCols);
    }
}

template <int D, int BSQ, int BSK, int DS, int PBQ, int PBK>
sa_status launch_band_bwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                          const sa_tensor *o, const float *lse, const sa_tensor *dout,
                          const sa_graph_s *g, float scale, sa_tensor *dq, sa_tensor *dk,
                          sa_tensor *dv, float *delta, cudaStream_t s) {
    using LQ = LayoutDQ<D, BSQ, DS, PBQ>;
    using LK = LayoutDKV<D, BSK, DS, PBK>;
    static_assert(LQ::kAlloc <= 232448 && LK::kAlloc <= 232448, "shared memory budget");
    const int64_t BH = q->B * q->H, T = q->T;
    CUtensorMap mq, mk, mv, mdo, mqr, mkr, mvr, mdor;
    const uint64_t rows = (uint64_t)(BH * T);
    if (!sa_tmap_bf16_3d(&mq, q->ptr, D, T, BH, BB) || !sa_tmap_bf16_3d(&mk, k->ptr, D, T, BH, BB) ||
        !sa_tmap_bf16_3d(&mv, v->ptr, D, T, BH, BB) ||
        !sa_tmap_bf16_3d(&mdo, dout->ptr, D, T, BH, BB) ||
        !sa_tmap_bf16_rows(&mqr, q->ptr, D, rows) || !sa_tmap_bf16_rows(&mkr, k->ptr, D, rows) ||
        !sa_tmap_bf16_rows(&mvr, v->ptr, D, rows) || !sa_tmap_bf16_rows(&mdor, dout->ptr, D, rows))
    {
        sa_record_cuda_error(cudaErrorInvalidValue, "band_bwd: tensor map encoding");
        return SA_ERR_CUDA;
    }
    BwdArgs a{};
    a.T = T;
    a.W = g->W;
    a.kind = g->kind;
    a.n_off = g->kind == 0 ? g->n_off : 0;
    for (int x = 0; x < SA_MAX_OFFSETS; ++x) a.offs[x] = x < a.n_off ? g->offs[x] : 0;
    a.rowptr = g->rowptr;
    a.colidx = g->colidx;
    a.rev_rowptr = g->rev_rowptr;
    a.rev_colidx = g->rev_colidx;
    a.q = (const __nv_bfloat16 *)q->ptr;
    a.k = (const __nv_bfloat16 *)k->ptr;
    a.v = (const __nv_bfloat16 *)v->ptr;
    a.o = (const __nv_bfloat16 *)o->ptr;
    a.dout = (const __nv_bfloat16 *)dout->ptr;
    a.lse = lse;
    a.delta = delta;
    a.dq = (__nv_bfloat16 *)dq->ptr;
    a.dk = (__nv_bfloat16 *)dk->ptr;
    a.dv = (__nv_bfloat16 *)dv->ptr;
    a.scale = scale;
    a.scale2 = scale * kLog2e;
    a.err = sa_device_error_word();
    if (!a.err) return SA_ERR_CUDA;
    auto kq = band_bwd_dq_kernel<D, BSQ, DS, PBQ>;
    auto kkv = band_bwd_dkdv_kernel<D, BSK, DS, PBK>;
    SA_CUDA_TRY(sa_smem_optin((const void *)kq, LQ::kAlloc));
    SA_CUDA_TRY(sa_smem_optin((const void *)kkv, LK::kAlloc));
    dim3 grid((unsigned)((T + BM - 1) / BM), (unsigned)BH);
    SA_LAUNCH("band_bwd_dq", s, kq<<<grid, 256, LQ::kAlloc, s>>>(mq, mk, mv, mdo, mkr, mvr, a));
    SA_LAUNCH("band_bwd_dkdv", s,
              kkv<<<grid, 256, LK::kAlloc, s>>>(mq, mk, mv, mdo, mqr, mdor, a));
    SA_CUDA_TRY(cudaGetLastError());
    return SA_OK;
}

}  // namespace

bool sa_band_bwd_supported(const sa_tensor *q, const sa_graph_s *g) {
    if (q->dtype != SA_BF16 || (q->D != 64 && q->D != 128)) return false;
    if (g->W < 1) return false;
    if (q->B * q->H > 65535 || q->T >= ((int64_t)1 << 31)) return false;
    const bool diag = (g->kind == 0) ? g->n_off > 0 : (g->max_resid > 0 || g->max_resid_rev > 0);
    if (g->kind == 1 && (!g->rowptr || !g->rev_rowptr)) return false;
    // distance / CSR edges with D = 128 stay on the gather kernels (register budget)
    if (diag && q->D == 128) return false;
    return true;
}

sa_status sa_band_bwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                      const sa_tensor *out, const float *lse, const sa_tensor *dout,
                      const sa_graph_s *g, const GraphView &, float scale, sa_tensor *dq,
                      sa_tensor *dk, sa_tensor *dv, float *delta, cudaStream_t s) {
    const bool diag = (g->kind == 0) ? g->n_off > 0 : (g->max_resid > 0 || g->max_resid_rev > 0);
    // <D, dQ ring stages, dK/dV ring stages, diagonal stages, dS buffers,
    //  P^T/dS^T buffers>, sized to the 227 KB of shared memory
    if (q->D == 64)
        return diag ? launch_band_bwd<64, 4, 3, 2, 2, 2>(q, k, v, out, lse, dout, g, scale, dq,
                                                         dk, dv, delta, s)
                    : launch_band_bwd<64, 4, 3, 0, 2, 2>(q, k, v, out, lse, dout, g, scale, dq,
                                                         dk, dv, delta, s);
    return launch_band_bwd<128, 4, 3, 0, 2, 1>(q, k, v, out, lse, dout, g, scale, dq, dk, dv,
                                               delta, s);
}
