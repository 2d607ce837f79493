// attn_band_bwd.cu -- backward on tcgen05 band tiles fused with the gathered
// edges.  Probabilities are recomputed from lse; two kernels with disjoint
// outputs and no float atomics, so results are bitwise reproducible:
//
//  band_bwd_dq   tile = 128 queries [q0, q0+128).  Delta_i = dO_i . out_i is
//                computed per row and written for the second kernel.  Key
//                blocks of BB from q0-W+1 (the forward's band in block
//                coordinates u = BB b + c, row r keeps r <= u <= r+W-1):
//                S = Q K^T and dP = dO V^T in TMEM, dS = P (dP - Delta)
//                written back over S in TMEM (bf16), dQ += dS K in TMEM with
//                dS read from TMEM by the MMA.
//  band_bwd_dkdv tile = 128 keys [k0, k0+128).  Query blocks of BB from k0
//                (v = i - k0 = BB b + c, key row r keeps r <= v <= r+W-1):
//                S^T = K Q^T and dP^T = V dO^T in TMEM, P^T and dS^T written
//                back over them (bf16), dV += P^T dO and dK += dS^T Q in TMEM.
//
// The other edges (2^k distance links or the non-window part of CSR lists)
// are diagonal blocks as in the forward: row r of a block belongs to query
// (or key) r; for a distance o the rows are one TMA box loaded by the
// producer, for CSR lists each compute warp copies its own rows with
// cp.async (sa_rows.cuh).  They are accumulated on the CUDA cores first
// (in registers at D = 64, directly in TMEM at D = 128) and initialise the
// TMEM accumulators, which the band MMAs then add to.  On a structured graph
// band_bwd_dq stores (p, dS) of every distance edge in a cache that
// band_bwd_dkdv reads instead of recomputing them.  With grouped-query
// attention a dK/dV tile covers one key/value head and loops over the query
// heads of its group.
//
// Both kernels are persistent and run NP (1 or 2) independent tile pipelines
// per CTA, each with its own shared-memory rings, TMEM columns and barriers.
// Warp roles: warp 2p is the TMA producer of pipeline p (its tile, the band
// ring, the diagonal blocks), warp 2p+1 its MMA issuer (warp 1 also allocates
// TMEM), warps 4+4p .. 7+4p its compute warpgroup (thread = owned row = TMEM
// lane).  Waits are bounded as in the forward.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sa_band.cuh"
#include "sa_rows.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace {

constexpr int BM = 128;  // rows a tile owns
constexpr float kLog2e = 1.4426950408889634f;

// Distance links inside the key span the band blocks of a tile cover anyway
// are folded into the band blocks (at most kMaxFold; sa_fold_links).
constexpr int kMaxFold = 4;

struct BwdArgs {
    int64_t T;
    int64_t BH;          // query slices B*H
    int64_t H, Hkv;      // query and key/value heads (grouped-query attention)
    int32_t W;
    int32_t We;          // span of the band blocks: W, or the longest folded link + 1
    int32_t nf;          // folded links
    int32_t fold[kMaxFold];
    int32_t kind;
    int32_t n_off;
    int32_t l2pf;        // prefetch diagonal rows into L2 (they do not fit in it)
    int64_t offs[SA_MAX_OFFSETS];  // descending
    const int64_t *rowptr;
    const int32_t *colidx;
    const int64_t *rev_rowptr;
    const int32_t *rev_colidx;
    const __nv_bfloat16 *o;        // forward output (Delta)
    // diagonal rows are copied from these: k, v (dQ pass), q, dout (dK/dV pass)
    const __nv_bfloat16 *k, *v, *q, *dout;
    const float *lse;
    float *delta;
    // Optional cache of (p, dS) per distance edge, written by dQ, read by
    // dK/dV: [distance index][b*h][query], fp32 pairs; null to recompute
    float2 *pds;
    __nv_bfloat16 *dq, *dk, *dv;
    float scale;
    float scale2;  // scale * log2(e)
    int *err;
};

// Register budgets with two pipelines (384 threads launched at 168 each).
struct BwdRegs {
    static constexpr int producer = 56, compute = 224;
    static_assert(128 * producer + 256 * compute <= 384 * 168, "register split");
};

// ---------------------------------------------------------------- helpers

// ROWS rows of a [B*H, T, D] tensor (all D/64 column chunks) with a map whose
// box is ROWS x 64; chunk x lands ROWS * 128 bytes after chunk x-1.
template <int D, int ROWS>
__device__ __forceinline__ void tma_rows(uint32_t dst, const void *map, int32_t row, int32_t bh,
                                         uint32_t bar) {
#pragma unroll
    for (int x = 0; x < D / 64; ++x)
        tc::tma_load_3d(dst + x * (ROWS * 128), map, x * 64, row, bh, bar);
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

// ---- bf16 x bf16 -> fp32 FMAs (exact products, one rounding per add):
// dot products with eight independent partial sums, axpys with the scalar
// rounded to bf16 (as the band path rounds P and dS for its MMAs).

__device__ __forceinline__ float sum8(const float *s) {
    return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}

// a . b, both rows of swizzled tiles in shared memory (row r of each).
template <int D>
__device__ __forceinline__ float dot_bf_smem_smem(const uint8_t *ta, const uint8_t *tb, int rows,
                                                  int r) {
    float sp[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) sp[x] = 0.f;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        const uint4 x = *(const uint4 *)(ta + tile_off(rows, r, c));
        const uint4 y = *(const uint4 *)(tb + tile_off(rows, r, c));
        const uint32_t xa[4] = {x.x, x.y, x.z, x.w}, yb[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            sp[2 * e] = tc::fma_bf_lo(xa[e], yb[e], sp[2 * e]);
            sp[2 * e + 1] = tc::fma_bf_hi(xa[e], yb[e], sp[2 * e + 1]);
        }
    }
    return sum8(sp);
}

// a . b, a packed bf16 pairs in registers (chunk c in a[4c .. 4c+3]), b row r
// of a tile read at the swizzled address.
template <int D>
__device__ __forceinline__ float dot_bf_reg_smem(const uint32_t *a, const uint8_t *tile, int rows,
                                                 int r) {
    float sp[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) sp[x] = 0.f;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        const uint4 y = *(const uint4 *)(tile + tile_off(rows, r, c));
        const uint32_t yb[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            sp[2 * e] = tc::fma_bf_lo(a[4 * c + e], yb[e], sp[2 * e]);
            sp[2 * e + 1] = tc::fma_bf_hi(a[4 * c + e], yb[e], sp[2 * e + 1]);
        }
    }
    return sum8(sp);
}

// acc += bf16(a) * (row r of a tile).
template <int D>
__device__ __forceinline__ void axpy_bf_smem(float *acc, float a, const uint8_t *tile, int rows,
                                             int r) {
    const uint32_t a2 = tc::pack_bf16x2(a, a);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        const uint4 y = *(const uint4 *)(tile + tile_off(rows, r, c));
        const uint32_t yb[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc[8 * c + 2 * e] = tc::fma_bf_lo(a2, yb[e], acc[8 * c + 2 * e]);
            acc[8 * c + 2 * e + 1] = tc::fma_bf_hi(a2, yb[e], acc[8 * c + 2 * e + 1]);
        }
    }
}

// TMEM row (D fp32 columns) += bf16(a) * (row r of a tile) where `on`, 32
// columns at a time (for D = 128, whose two accumulators do not fit in
// registers).  Every lane of the warp must call it (the TMEM loads and stores
// are warp-collective); a lane with on == false stores its row back unchanged.
template <int D>
__device__ __forceinline__ void tmem_axpy_row(uint32_t taddr, float a, bool on,
                                              const uint8_t *tile, int rows, int r) {
    const uint32_t a2 = tc::pack_bf16x2(a, a);
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t w[32];
        tc::tmem_ld32(taddr + c0, w);
        tc::tmem_ld_wait();
#pragma unroll
        for (int c = c0 / 8; c < c0 / 8 + 4; ++c) {
            const uint4 y = *(const uint4 *)(tile + tile_off(rows, r, c));
            const uint32_t yb[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int x = 8 * c - c0 + 2 * e;
                const float lo = tc::fma_bf_lo(a2, yb[e], __uint_as_float(w[x]));
                const float hi = tc::fma_bf_hi(a2, yb[e], __uint_as_float(w[x + 1]));
                w[x] = on ? __float_as_uint(lo) : w[x];
                w[x + 1] = on ? __float_as_uint(hi) : w[x + 1];
            }
        }
        tc::tmem_st32(taddr + c0, w);
        tc::tmem_st_wait();
    }
}

// D fp32 values (zeros for acc == nullptr) -> TMEM row.
template <int D>
__device__ __forceinline__ void tmem_store_row(uint32_t taddr, const float *acc) {
#pragma unroll
    for (int c = 0; c < D; c += 32) {
        uint32_t w[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) w[x] = acc ? __float_as_uint(acc[c + x]) : 0u;
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

// Pack n fp32 values as n/2 bf16 pairs (round to nearest even).
// TMEM rows (D fp32 columns, this warp's 32 lanes from taddr) times `mul` as
// bf16 to global memory, DG columns per row: in whole sectors through the
// accumulator's own first columns (tc::tmem_rows_store) when DG is a multiple
// of 64, else row by row.  dst: the warp's row 0; rows >= nrows not written.
template <int DG>
__device__ __forceinline__ void tmem_rows_to_global(uint32_t taddr, float mul, __nv_bfloat16 *dst,
                                                    int64_t nrows_in, int lane) {
    const int nrows = nrows_in < 0 ? 0 : (nrows_in > 32 ? 32 : (int)nrows_in);
    if constexpr (DG % 64 == 0) {
        uint32_t pk[DG / 2];
#pragma unroll
        for (int c = 0; c < DG; c += 32) {
            uint32_t w[32];
            tc::tmem_ld32(taddr + c, w);
            tc::tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 32; x += 2)
                pk[(c + x) / 2] =
                    tc::pack_bf16x2(__uint_as_float(w[x]) * mul, __uint_as_float(w[x + 1]) * mul);
        }
        tc::tmem_rows_store<DG / 2>(taddr, pk, dst, DG, nrows, lane);
    } else {
        tmem_row_to_global<DG>(taddr, mul, dst + (size_t)lane * DG, lane < nrows);
    }
}

template <int N>
__device__ __forceinline__ void pack_bf16_row(const float *x, uint32_t *w) {
#pragma unroll
    for (int c = 0; c < N / 2; ++c) w[c] = tc::pack_bf16x2(x[2 * c], x[2 * c + 1]);
}

// 64 fp32 values as bf16, row r of a 128-row K-major tile with 128-byte
// swizzle (the layout TMA writes), for a shared-memory MMA operand.
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

// Tile t of a pipeline: (b*h slice, first row).
struct TileId {
    int32_t bh, r0;
};
__device__ __forceinline__ TileId tile_id(int64_t t, int64_t ntr) {
    TileId id;
    const int64_t bh = t / ntr;
    id.bh = (int32_t)bh;
    id.r0 = (int32_t)((t - bh * ntr) * BM);
    return id;
}

#define WAIT_OR(bar_, par_, action_)                                                   \
    if (!tc::mbar_wait((bar_), (par_), abort, a.err, SA_DEVERR_TIMEOUT)) {              \
        action_;                                                                       \
    }

// =================================================================== dQ

// PS = 0: dS (bf16) is written over S in TMEM and read from there by the dQ
// MMA.  PS > 0: dS goes to PS shared-memory tiles instead, which frees the S
// buffer as soon as the compute warps have read it (for one pipeline).
template <int D, int NP, int BB, int SB, int BS, int DS, int PS>
struct LayoutDQ {
    static constexpr int kRow = BM * D * 2, kBlk = BB * D * 2, kDSTile = BM * BB * 2;
    static constexpr int pQ = 0, pDO = kRow, pK = 2 * kRow, pV = pK + BS * kBlk;
    static constexpr int pDK = pV + BS * kBlk, pDV = pDK + DS * kRow;
    static constexpr int pDS = pDV + DS * kRow;
    static constexpr int kPipe = pDS + PS * kDSTile;
    static constexpr int kBars = NP * kPipe;
    // barriers of one pipeline (S and dP share a buffer index sb; dS is
    // written over S, so a buffer is free once its dQ MMA is done)
    static constexpr int bQFull = 0, bQEmpty = 1;
    static constexpr int bKVFull = 2, bKVEmpty = bKVFull + BS;
    static constexpr int bSFull = bKVEmpty + BS, bSFree = bSFull + SB;
    static constexpr int bDSFull = bSFree + SB, bDQDone = bDSFull + SB;
    static constexpr int bInit = bDQDone + SB;
    static constexpr int bPSDone = bInit + 1;              // dS tile consumed by its MMA
    // distance blocks loaded by the producer with TMA (structured graphs)
    static constexpr int DSX = DS > 0 ? DS : 1;
    static constexpr int bDiagFull = bPSDone + (PS > 0 ? PS : 1), bDiagEmpty = bDiagFull + DSX;
    static constexpr int bInfoFull = bDiagEmpty + DSX, bInfoEmpty = bInfoFull + 2;
    static constexpr int nBarsPipe = bInfoEmpty + 2;
    static constexpr int kMisc = kBars + NP * nBarsPipe * 8;  // tmem slot, abort, info[NP][2]
    static constexpr int kTotal = kMisc + 8 + 8 * NP;
    static constexpr int kAlloc = kTotal + 1024;
    static_assert(PS == 0 || BB == 64, "shared-memory dS tiles are 64 keys wide");
    // TMEM columns of pipeline p start at tPipe p: S buffers, dP buffers, dQ
    static constexpr uint32_t tPipe = 512 / NP, tS = 0, tDP = SB * BB, tDQ = 2 * SB * BB;
    static constexpr uint32_t kTmemCols = 512;
    static_assert(2 * SB * BB + D <= (int)tPipe, "TMEM columns of a pipeline");
    static_assert(kRow % 1024 == 0 && kBlk % 1024 == 0, "swizzle atoms");
};

// Band geometry of a query tile: key blocks of BB from q0-W+1 up to the last key.
template <int BB>
struct DQBand {
    int32_t kb0, b_first, n_band;
    __device__ __forceinline__ DQBand(int32_t q0, int64_t T, int32_t W) {
        kb0 = q0 - W + 1;
        const int32_t last_key = (q0 + BM - 1 < T - 1) ? q0 + BM - 1 : (int32_t)(T - 1);
        const int32_t nblk = (last_key - kb0) / BB + 1;
        const int32_t need = W - 1 - q0;
        b_first = need > 0 ? need / BB : 0;
        n_band = nblk - b_first;
    }
};

// LDW: the diagonal slots are copied by each compute warp (CSR lists); else
// the producer loads each distance block as TMA boxes (structured graphs).
template <int D, int NP, int BB, int SB, int BS, int DS, int PS, bool LDW, int DG>
__global__ void __launch_bounds__(128 + 128 * NP, 1)
band_bwd_dq_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
                   const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                   const __grid_constant__ CUtensorMap tkd,
                   const __grid_constant__ CUtensorMap tvd, const BwdArgs a) {
    using L = LayoutDQ<D, NP, BB, SB, BS, DS, PS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = tc::smem_u32(sm);
    uint32_t *tmem_slot = (uint32_t *)(sm + L::kMisc);
    volatile int *abort = (volatile int *)(sm + L::kMisc + 4);
    auto bar = [&](int p, int b) {
        return sbase + L::kBars + 8u * (uint32_t)(p * L::nBarsPipe + b);
    };
    auto wait = [&](int p, int b, uint32_t parity) {
        return tc::mbar_wait(bar(p, b), parity, abort, a.err, SA_DEVERR_TIMEOUT);
    };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t T = a.T;
    const int32_t W = a.W;
    const int64_t ntr = (T + BM - 1) / BM, ntiles = ntr * a.BH;
    const int64_t stride = (int64_t)gridDim.x * NP;

    if (tid == 0) {
        for (int p = 0; p < NP; ++p) {
            tc::mbar_init(bar(p, L::bQFull), 1);
            tc::mbar_init(bar(p, L::bQEmpty), 5);  // last S/dP MMA commit + 4 compute warps
            for (int s = 0; s < BS; ++s) {
                tc::mbar_init(bar(p, L::bKVFull + s), 1);
                tc::mbar_init(bar(p, L::bKVEmpty + s), 1);
            }
            for (int s = 0; s < SB; ++s) {
                tc::mbar_init(bar(p, L::bSFull + s), 1);
                // freed by the dQ MMA (dS in TMEM) or by the compute warps
                tc::mbar_init(bar(p, L::bSFree + s), PS > 0 ? 4 : 1);
                tc::mbar_init(bar(p, L::bDSFull + s), 4);
                tc::mbar_init(bar(p, L::bDQDone + s), 1);
            }
            tc::mbar_init(bar(p, L::bInit), 4);
            for (int s = 0; s < PS; ++s) tc::mbar_init(bar(p, L::bPSDone + s), 1);
            for (int s = 0; s < L::DSX; ++s) {
                tc::mbar_init(bar(p, L::bDiagFull + s), 1);
                tc::mbar_init(bar(p, L::bDiagEmpty + s), 4);
            }
            for (int s = 0; s < 2; ++s) {
                tc::mbar_init(bar(p, L::bInfoFull + s), 1);
                tc::mbar_init(bar(p, L::bInfoEmpty + s), 4);
            }
        }
        *abort = 0;
        tc::fence_barrier_init();
    }
    if constexpr (LDW && DG < D) {
        // the per-warp copies fill DG columns of each diagonal row: the rest
        // of the rings stays zero
        for (int p = 0; p < NP; ++p)
            for (int o = L::pDK + 16 * tid; o < L::pDS; o += 16 * blockDim.x)
                *(uint4 *)(sm + p * L::kPipe + o) = make_uint4(0, 0, 0, 0);
    }
    if (warp == 1) tc::tmem_alloc(tc::smem_u32(tmem_slot), L::kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 4) {
        if (NP == 2) tc::regs_dec<BwdRegs::producer>();
      if ((warp >> 1) < NP && (warp & 1) == 0) {
        // ---------------- producer of pipeline p (lane 0): Q and dO of the
        // tile, the band K/V blocks through their ring and, for a structured
        // graph, the distance blocks (the count first, to the compute warps)
        // after the band blocks that fit the ring
        const int p = warp >> 1;
        const uint32_t pb = sbase + (uint32_t)(p * L::kPipe);
        volatile int *info = (volatile int *)(sm + L::kMisc + 8) + 2 * p;
        if (lane == 0) {
            uint32_t kvc = 0, dc = 0;
            bool ok = true;
            int64_t lt = 0;
            for (int64_t t = (int64_t)blockIdx.x * NP + p; ok && t < ntiles; t += stride, ++lt) {
                const TileId id = tile_id(t, ntr);
                const int32_t q0 = id.r0, bh = id.bh;
                const int32_t kvbh = (int32_t)((bh / a.H) * a.Hkv + (bh % a.H) / (a.H / a.Hkv));
                const DQBand<BB> g(q0, T, a.We);
                constexpr bool kTmaDiag = DS > 0 && !LDW;
                int nd = 0;
                if constexpr (kTmaDiag) {
                    const int64_t last = (q0 + BM - 1 < T - 1) ? q0 + BM - 1 : T - 1;
                    for (int x = 0; x < a.n_off; ++x) nd += (a.offs[x] <= last) ? 1 : 0;
                    const int slot = (int)(lt & 1);
                    if (lt >= 2 && !wait(p, L::bInfoEmpty + slot, (uint32_t)(((lt >> 1) - 1) & 1)))
                        break;
                    info[slot] = nd;
                    tc::mbar_arrive(bar(p, L::bInfoFull + slot));
                }
                if (lt >= 1 && !wait(p, L::bQEmpty, (uint32_t)((lt - 1) & 1))) break;
                tc::mbar_arrive_expect_tx(bar(p, L::bQFull), 2 * L::kRow);
                tma_rows<D, BM>(pb + L::pQ, &tq, q0, bh, bar(p, L::bQFull));
                tma_rows<D, BM>(pb + L::pDO, &tdo, q0, bh, bar(p, L::bQFull));
                auto load_kv = [&](int bl) -> bool {
                    const int st = (int)(kvc % BS);
                    const uint32_t use = kvc / BS;
                    if (use > 0 && !wait(p, L::bKVEmpty + st, (use - 1) & 1)) return false;
                    const int32_t krow = g.kb0 + (g.b_first + bl) * BB;
                    tc::mbar_arrive_expect_tx(bar(p, L::bKVFull + st), 2 * L::kBlk);
                    tma_rows<D, BB>(pb + L::pK + st * L::kBlk, &tk, krow, kvbh,
                                    bar(p, L::bKVFull + st));
                    tma_rows<D, BB>(pb + L::pV + st * L::kBlk, &tv, krow, kvbh,
                                    bar(p, L::bKVFull + st));
                    ++kvc;
                    return true;
                };
                int bl = 0;
                if constexpr (kTmaDiag) {
                    const int n_pre = g.n_band < BS ? g.n_band : BS;
                    for (; ok && bl < n_pre; ++bl) ok = load_kv(bl);
                    // distance o: keys q0-o .. q0+127-o
                    for (int d = 0; ok && d < nd; ++d) {
                        const int st = (int)(dc % DS);
                        const uint32_t use = dc / DS;
                        if (use > 0 && !wait(p, L::bDiagEmpty + st, (use - 1) & 1)) {
                            ok = false;
                            break;
                        }
                        const int32_t krow = (int32_t)(q0 - a.offs[a.n_off - nd + d]);
                        tc::mbar_arrive_expect_tx(bar(p, L::bDiagFull + st), 2 * L::kRow);
                        tma_rows<D, BM>(pb + L::pDK + st * L::kRow, &tkd, krow, kvbh,
                                        bar(p, L::bDiagFull + st));
                        tma_rows<D, BM>(pb + L::pDV + st * L::kRow, &tvd, krow, kvbh,
                                        bar(p, L::bDiagFull + st));
                        ++dc;
                    }
                }
                for (; ok && bl < g.n_band; ++bl) ok = load_kv(bl);
            }
        }
      } else if ((warp >> 1) < NP) {
        // ---------------- MMA issuer of pipeline p: S and dP of block g, then
        // dQ += dS K of block g-1
        const int p = warp >> 1;
        const uint32_t pb = sbase + (uint32_t)(p * L::kPipe);
        const uint32_t tp = tmem + p * L::tPipe;
        if (lane == 0) {
            const uint32_t idS = tc::idesc_bf16(BM, BB, false, false);
            const uint32_t idQ = tc::idesc_bf16(BM, D, false, true);
            uint32_t gb = 0;  // band blocks issued (all tiles)
            bool have = false, first = false, ok = true;
            uint32_t pg = 0;
            int64_t plt = 0;
            auto do_dq = [&]() -> bool {
                const int sb = (int)(pg % SB), st = (int)(pg % BS);
                if (first && !wait(p, L::bInit, (uint32_t)(plt & 1))) return false;
                if (!wait(p, L::bDSFull + sb, (pg / SB) & 1)) return false;
                tc::tc_fence_after();
                const uint32_t ka = pb + L::pK + st * L::kBlk;
                if constexpr (PS > 0) {
                    const int ps = (int)(pg % PS);
                    const uint32_t dsa = pb + L::pDS + ps * L::kDSTile;
#pragma unroll
                    for (int kk = 0; kk < BB / 16; ++kk)
                        tc::mma_bf16_ss(tp + L::tDQ, tc::sdesc_sw128(dsa + kk * 32, 16, 1024),
                                        tc::sdesc_sw128(ka + kk * 16 * 128, BB * 128, 1024), idQ,
                                        1u);
                    tc::mma_commit(bar(p, L::bKVEmpty + st));
                    tc::mma_commit(bar(p, L::bPSDone + ps));
                } else {
#pragma unroll
                    for (int kk = 0; kk < BB / 16; ++kk)
                        tc::mma_bf16_ts(tp + L::tDQ, tp + L::tS + sb * BB + kk * 8,
                                        tc::sdesc_sw128(ka + kk * 16 * 128, BB * 128, 1024), idQ,
                                        1u);
                    tc::mma_commit(bar(p, L::bKVEmpty + st));
                    tc::mma_commit(bar(p, L::bSFree + sb));
                }
                tc::mma_commit(bar(p, L::bDQDone + sb));
                return true;
            };
            int64_t lt = 0;
            for (int64_t t = (int64_t)blockIdx.x * NP + p; ok && t < ntiles; t += stride, ++lt) {
                const TileId id = tile_id(t, ntr);
                const DQBand<BB> g(id.r0, T, a.We);
                if (!wait(p, L::bQFull, (uint32_t)(lt & 1))) break;
                const uint32_t qa = pb + L::pQ, da = pb + L::pDO;
                for (int bl = 0; bl < g.n_band; ++bl) {
                    const int st = (int)(gb % BS), sb = (int)(gb % SB);
                    // one S buffer: dQ of the previous block frees it first
                    if (SB == 1 && have) {
                        if (!do_dq()) {
                            ok = false;
                            break;
                        }
                        have = false;
                    }
                    if (!wait(p, L::bKVFull + st, (gb / BS) & 1) ||
                        (gb >= SB && !wait(p, L::bSFree + sb, ((gb / SB) - 1) & 1))) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t ka = pb + L::pK + st * L::kBlk, va = pb + L::pV + st * L::kBlk;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t offr = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                        const uint32_t offb = (kk >> 2) * (BB * 128) + (kk & 3) * 32;
                        tc::mma_bf16_ss(tp + L::tS + sb * BB, tc::sdesc_sw128(qa + offr, 16, 1024),
                                        tc::sdesc_sw128(ka + offb, 16, 1024), idS, kk > 0);
                        tc::mma_bf16_ss(tp + L::tDP + sb * BB,
                                        tc::sdesc_sw128(da + offr, 16, 1024),
                                        tc::sdesc_sw128(va + offb, 16, 1024), idS, kk > 0);
                    }
                    tc::mma_commit(bar(p, L::bSFull + sb));
                    if (bl == g.n_band - 1) tc::mma_commit(bar(p, L::bQEmpty));
                    // dS of this block is computed while dQ of the previous one runs
                    if (SB > 1 && have && !do_dq()) {
                        ok = false;
                        break;
                    }
                    have = true;
                    pg = gb;
                    first = (bl == 0);
                    plt = lt;
                    ++gb;
                }
                // the tile's last dQ MMA goes now: its epilogue waits for it
                if (ok && have) {
                    ok = do_dq();
                    have = false;
                }
            }
        }
      }
    } else {
        // ---------------- compute warpgroup of pipeline p: thread r = query
        // row r = TMEM lane r
        if (NP == 2) tc::regs_inc<BwdRegs::compute>();
        const int p = (warp - 4) >> 2;
        const int r = tid - 128 - 128 * p;
        uint8_t *pm = sm + p * L::kPipe;
        const uint32_t lane_off = (uint32_t)(((warp - 4) & 3) * 32) << 16;
        const uint32_t tS = tmem + p * L::tPipe + lane_off + L::tS;
        const uint32_t tDP = tmem + p * L::tPipe + lane_off + L::tDP;
        const uint32_t tDQ = tmem + p * L::tPipe + lane_off + L::tDQ;
        const float c2 = a.scale2;
        const int wq = r >> 5;  // warp within the group: rows 32 wq .. 32 wq + 31
        volatile int *info = (volatile int *)(sm + L::kMisc + 8) + 2 * p;
        uint32_t gb = 0, dc = 0;
        bool ok = true;
        int64_t lt = 0;
        for (int64_t t = (int64_t)blockIdx.x * NP + p; ok && t < ntiles; t += stride, ++lt) {
            const TileId id = tile_id(t, ntr);
            const int32_t q0 = id.r0, bh = id.bh;
            const int64_t kvbh = (bh / a.H) * a.Hkv + (bh % a.H) / (a.H / a.Hkv);
            const DQBand<BB> g(q0, T, a.We);
            const int64_t i = q0 + r;
            const bool row_ok = i < T;
            const size_t grow = (size_t)bh * (size_t)T + (size_t)i;
            const float lse2 = row_ok ? a.lse[grow] * kLog2e : 0.f;
            // the out row for Delta is fetched while Q and dO arrive
            uint4 orow4[DG / 8];
#pragma unroll
            for (int c = 0; c < DG / 8; ++c)
                orow4[c] = row_ok ? __ldg((const uint4 *)(a.o + grow * DG) + c) : make_uint4(0, 0, 0, 0);
            if (!__all_sync(0xffffffffu, wait(p, L::bQFull, (uint32_t)(lt & 1)))) break;
            // Delta_i = dO_i . out_i
            float Delta = 0.f;
            {
                uint32_t dor[DG / 2];
                load_row_packed<DG>(pm + L::pDO, BM, r, dor);
                float sp[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) sp[x] = 0.f;
#pragma unroll
                for (int c = 0; c < DG / 8; ++c) {
                    const uint32_t ow[4] = {orow4[c].x, orow4[c].y, orow4[c].z, orow4[c].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        sp[2 * e] = tc::fma_bf_lo(dor[4 * c + e], ow[e], sp[2 * e]);
                        sp[2 * e + 1] = tc::fma_bf_hi(dor[4 * c + e], ow[e], sp[2 * e + 1]);
                    }
                }
                Delta = sum8(sp);
            }
            if (row_ok) a.delta[grow] = Delta;
            // diagonal slots: the K and V rows of this row's distance links (or
            // CSR residual entries), fetched by this warp itself; their sum is
            // kept in registers (D = 64) or in the TMEM accumulator (D = 128)
            constexpr bool kRegAcc = D == 64;
            float acc[kRegAcc ? D : 1];
#pragma unroll
            for (int x = 0; x < (kRegAcc ? D : 1); ++x) acc[x] = 0.f;
            if constexpr (!kRegAcc) {
                tmem_store_row<D>(tDQ, nullptr);
                tc::tmem_st_wait();
            }
            if constexpr (DS > 0) {
                // slots: the tile's distance blocks (count from the producer),
                // or, for CSR lists, the longest residual list of this warp's rows
                int nd = 0;
                int64_t cst = 0;
                int32_t resid = 0;
                if constexpr (!LDW) {
                    const int slot = (int)(lt & 1);
                    ok = __all_sync(0xffffffffu,
                                    wait(p, L::bInfoFull + slot, (uint32_t)((lt >> 1) & 1)));
                    nd = ok ? info[slot] : 0;
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar(p, L::bInfoEmpty + slot));
                } else {
                    if (row_ok) {
                        cst = a.rowptr[i];
                        resid = (int32_t)(a.rowptr[i + 1] - cst - ((i + 1 < W) ? i + 1 : W));
                    }
                    nd = (int)__reduce_max_sync(0xffffffffu, (unsigned)resid);
                }
                const int dfirst = a.n_off - nd;  // distance index of slot 0 (keys ascending)
                auto key_of = [&](int d) -> int32_t {  // (CSR slots)
                    return d < resid ? __ldg(a.colidx + cst + d) : -1;
                };
                // the q row in registers (D = 64) or read from the Q tile (D = 128,
                // whose accumulator already takes 128 registers)
                uint32_t qw[D == 64 ? DG / 2 : 1];
                if constexpr (D == 64) load_row_packed<DG>(pm + L::pQ, BM, r, qw);
                auto body = [&](int d, int st) {
                    const bool valid = LDW ? (d < resid) : (row_ok && i >= a.offs[dfirst + d]);
                    const uint8_t *kt = pm + L::pDK + st * L::kRow;
                    const uint8_t *vt = pm + L::pDV + st * L::kRow;
                    float ds = 0.f;
                    if (valid) {
                        float qk;
                        if constexpr (D == 64)
                            qk = dot_bf_reg_smem<DG>(qw, kt, BM, r);
                        else
                            qk = dot_bf_smem_smem<DG>(pm + L::pQ, kt, BM, r);
                        const float pr = tc::ex2(fmaf(qk, c2, -lse2));
                        ds = pr * (dot_bf_smem_smem<DG>(pm + L::pDO, vt, BM, r) - Delta);
                        if (a.pds)
                            a.pds[((size_t)(dfirst + d) * (size_t)a.BH + (size_t)bh) *
                                      (size_t)T +
                                  (size_t)i] = make_float2(pr, ds);
                        if constexpr (kRegAcc) axpy_bf_smem<DG>(acc, ds, kt, BM, r);
                    }
                    // (warp-collective: every lane, whether or not its row has the slot)
                    if constexpr (!kRegAcc) tmem_axpy_row<D>(tDQ, ds, valid, kt, BM, r);
                };
                if constexpr (LDW) {
                    rows::warp_slots<DG, DS>(
                        nd, sbase + (uint32_t)(p * L::kPipe + L::pDK),
                        sbase + (uint32_t)(p * L::kPipe + L::pDV), (uint32_t)L::kRow, a.k, a.v,
                        a.l2pf != 0, lane, wq,
                        [&](int) { return (size_t)kvbh * (size_t)T * DG; }, key_of, body);
                } else {
                    for (int d = 0; ok && d < nd; ++d) {
                        const int st = (int)(dc % DS);
                        if (!__all_sync(0xffffffffu, wait(p, L::bDiagFull + st, (dc / DS) & 1))) {
                            ok = false;
                            break;
                        }
                        body(d, st);
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(bar(p, L::bDiagEmpty + st));
                        ++dc;
                    }
                }
            }
            if (!ok) break;
            // this warp is done reading Q and dO of the tile
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(p, L::bQEmpty));
            if constexpr (kRegAcc) tmem_store_row<D>(tDQ, acc);
            tc::tmem_st_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(p, L::bInit));

            // band blocks: dS = P (dP - Delta), bf16 over S
            uint32_t gb_last = gb;
            for (int bl = 0; ok && bl < g.n_band; ++bl, ++gb) {
                const int sb = (int)(gb % SB);
                const int32_t u0 = (g.b_first + bl) * BB;
                gb_last = gb;
                if (!wait(p, L::bSFull + sb, (gb / SB) & 1)) {
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                float s[BB], dp[BB];
                tc::tmem_ld_n<BB>(tS + sb * BB, (uint32_t *)s);
                tc::tmem_ld_n<BB>(tDP + sb * BB, (uint32_t *)dp);
                tc::tmem_ld_wait();
                if (PS > 0) {  // S and dP are in registers: the buffer is free
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar(p, L::bSFree + sb));
                }
                const int32_t We = a.We;
                const bool need_mask = a.nf > 0 || (u0 < BM - 1) || (u0 + BB - 1 > We - 1) ||
                                       (u0 + q0 < We - 1);
                if (need_mask) {
                    // keep columns [c_lo, c_hi]: r + We - W <= u <= r + We - 1
                    // and key >= 0, plus the folded links u = r + We - 1 - o
                    const int32_t kmin = We - 1 - q0;  // u of key 0
                    const int32_t lo = (r + We - W > kmin) ? r + We - W : kmin;
                    const int32_t hi = r + We - 1;
                    const int c_lo = lo - u0 < 0 ? 0 : (lo - u0 > BB ? BB : lo - u0);
                    const int c_hi = hi - u0 > BB - 1 ? BB - 1 : (hi - u0 < -1 ? -1 : hi - u0);
                    uint64_t keep = tc::bits_range(c_lo, c_hi);  // bit c: column c kept
                    if (a.nf > 0) {
#pragma unroll
                        for (int x = 0; x < kMaxFold; ++x) {
                            const int32_t u = r + We - 1 - a.fold[x];
                            if (x < a.nf && u >= kmin && u >= u0 && u < u0 + BB)
                                keep |= 1ull << (u - u0);
                        }
                    }
                    // 16-column chunks outside every kept range of this warp: dS = 0
#pragma unroll
                    for (int c16 = 0; c16 < BB / 16; ++c16) {
                        if (__any_sync(0xffffffffu, ((keep >> (16 * c16)) & 0xffffull) != 0ull)) {
#pragma unroll
                            for (int c = 16 * c16; c < 16 * c16 + 16; ++c) {
                                const float pr =
                                    ((keep >> c) & 1ull) ? tc::ex2(fmaf(s[c], c2, -lse2)) : 0.f;
                                s[c] = pr * (dp[c] - Delta);
                            }
                        } else {
#pragma unroll
                            for (int c = 16 * c16; c < 16 * c16 + 16; ++c) s[c] = 0.f;
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < BB; ++c)
                        s[c] = tc::ex2(fmaf(s[c], c2, -lse2)) * (dp[c] - Delta);
                }
                if constexpr (PS > 0) {
                    const int ps = (int)(gb % PS);
                    if (gb >= PS && !wait(p, L::bPSDone + ps, ((gb / PS) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    store_row64_bf16(pm + L::pDS + ps * L::kDSTile, r, s);
                    tc::fence_proxy_async_smem();
                } else {
                    uint32_t w[BB / 2];
                    pack_bf16_row<BB>(s, w);
                    tc::tmem_st_n<BB / 2>(tS + sb * BB, w);
                    tc::tmem_st_wait();
                    tc::tc_fence_before();
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar(p, L::bDSFull + sb));
            }
            if (!ok) break;
            if (!wait(p, L::bDQDone + (int)(gb_last % SB), (gb_last / SB) & 1)) break;
            tc::tc_fence_after();
            tmem_rows_to_global<DG>(tDQ, a.scale,
                                    a.dq + ((size_t)bh * (size_t)T + (size_t)(q0 + 32 * wq)) * DG,
                                    T - (q0 + 32 * wq), lane);
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

// PS = 0: P^T and dS^T (bf16) are written over S^T and dP^T in TMEM.  PS > 0:
// they go to PS pairs of shared-memory tiles, which frees the S^T/dP^T buffer
// as soon as the compute warps have read it (for one pipeline).
template <int D, int NP, int BB, int SB, int BS, int DS, int PS>
struct LayoutDKV {
    static constexpr int kRow = BM * D * 2, kBlk = BB * D * 2, kPTile = BM * BB * 2;
    static constexpr int pK = 0, pV = kRow, pQ = 2 * kRow, pDO = pQ + BS * kBlk;
    static constexpr int pDQ = pDO + BS * kBlk, pDDO = pDQ + DS * kRow;
    static constexpr int pP = pDDO + DS * kRow, pDS = pP + PS * kPTile;
    static constexpr int kPipe = pDS + PS * kPTile;
    // lse (base 2) and Delta of each band stage's BB queries, after the pipelines
    static constexpr int kStage = 2 * BB * 4;
    static constexpr int kLse = NP * kPipe;
    static constexpr int kBars = kLse + NP * BS * kStage;
    // barriers of one pipeline (S^T and dP^T share a buffer index sb; P^T and
    // dS^T are written over them, so a buffer is free once its dV/dK MMAs are
    // done)
    static constexpr int bKVFull = 0, bKVEmpty = 1;
    static constexpr int bBFull = 2, bBEmpty = bBFull + BS;
    static constexpr int bSFull = bBEmpty + BS, bSFree = bSFull + SB;
    static constexpr int bPFull = bSFree + SB, bDKVDone = bPFull + SB;
    static constexpr int bInit = bDKVDone + SB;
    static constexpr int bPSDone = bInit + 1;              // P^T/dS^T tiles consumed
    // distance blocks loaded by the producer with TMA (structured graphs)
    static constexpr int DSX = DS > 0 ? DS : 1;
    static constexpr int bDiagFull = bPSDone + (PS > 0 ? PS : 1), bDiagEmpty = bDiagFull + DSX;
    static constexpr int bInfoFull = bDiagEmpty + DSX, bInfoEmpty = bInfoFull + 2;
    static constexpr int nBarsPipe = bInfoEmpty + 2;
    static constexpr int kMisc = kBars + NP * nBarsPipe * 8;  // tmem slot, abort, info[NP][2]
    static constexpr int kTotal = kMisc + 8 + 8 * NP;
    static constexpr int kAlloc = kTotal + 1024;
    static_assert(PS == 0 || BB == 64, "shared-memory P tiles are 64 queries wide");
    static constexpr uint32_t tPipe = 512 / NP, tS = 0, tDP = SB * BB, tDV = 2 * SB * BB,
                              tDK = 2 * SB * BB + D;
    static constexpr uint32_t kTmemCols = 512;
    static_assert(2 * SB * BB + 2 * D <= (int)tPipe, "TMEM columns of a pipeline");
    static_assert(kRow % 1024 == 0 && kBlk % 1024 == 0, "swizzle atoms");
};

// Query blocks of a key tile: BB queries from k0 up to min(k0+127+W-1, T-1).
template <int BB>
__device__ __forceinline__ int dkv_n_band(int32_t k0, int64_t T, int32_t W) {
    const int64_t vmax_w = (int64_t)BM - 1 + W - 1, vmax_t = T - 1 - k0;
    const int64_t vmax = vmax_w < vmax_t ? vmax_w : vmax_t;
    return (int)(vmax / BB + 1);
}

// LDW: the diagonal slots are copied by each compute warp (CSR lists); else
// the producer loads each distance block as TMA boxes (structured graphs).
template <int D, int NP, int BB, int SB, int BS, int DS, int PS, bool LDW, int DG>
__global__ void __launch_bounds__(128 + 128 * NP, 1)
band_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tkt,
                     const __grid_constant__ CUtensorMap tvt,
                     const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
                     const __grid_constant__ CUtensorMap tqd,
                     const __grid_constant__ CUtensorMap tdod, const BwdArgs a) {
    using L = LayoutDKV<D, NP, BB, SB, BS, DS, PS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = tc::smem_u32(sm);
    uint32_t *tmem_slot = (uint32_t *)(sm + L::kMisc);
    volatile int *abort = (volatile int *)(sm + L::kMisc + 4);
    auto bar = [&](int p, int b) {
        return sbase + L::kBars + 8u * (uint32_t)(p * L::nBarsPipe + b);
    };
    auto wait = [&](int p, int b, uint32_t parity) {
        return tc::mbar_wait(bar(p, b), parity, abort, a.err, SA_DEVERR_TIMEOUT);
    };
    auto stage_lse = [&](int p, int st) {
        return (float *)(sm + L::kLse + (p * BS + st) * L::kStage);
    };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t T = a.T;
    const int32_t W = a.W;
    // tiles run over key/value slices; each takes the blocks of every query
    // head of its group (grouped-query attention: GQ = H / Hkv heads)
    const int64_t BHkv = a.BH / (a.H / a.Hkv);
    const int GQ = (int)(a.H / a.Hkv);
    const int64_t ntr = (T + BM - 1) / BM, ntiles = ntr * BHkv;
    const int64_t stride = (int64_t)gridDim.x * NP;
    auto qslice0 = [&](int32_t kvbh) -> int64_t {  // first query slice of the group
        return ((int64_t)kvbh / a.Hkv) * a.H + ((int64_t)kvbh % a.Hkv) * GQ;
    };

    if (tid == 0) {
        for (int p = 0; p < NP; ++p) {
            tc::mbar_init(bar(p, L::bKVFull), 1);
            tc::mbar_init(bar(p, L::bKVEmpty), 5);  // last S^T/dP^T MMA commit + 4 compute warps
            for (int s = 0; s < BS; ++s) {
                // TMA bytes + the 32 producer lanes that stage lse and Delta
                tc::mbar_init(bar(p, L::bBFull + s), 33);
                tc::mbar_init(bar(p, L::bBEmpty + s), 1);
            }
            for (int s = 0; s < SB; ++s) {
                tc::mbar_init(bar(p, L::bSFull + s), 1);
                // freed by the dV/dK MMAs (P^T in TMEM) or by the compute warps
                tc::mbar_init(bar(p, L::bSFree + s), PS > 0 ? 4 : 1);
                tc::mbar_init(bar(p, L::bPFull + s), 4);
                tc::mbar_init(bar(p, L::bDKVDone + s), 1);
            }
            tc::mbar_init(bar(p, L::bInit), 4);
            for (int s = 0; s < PS; ++s) tc::mbar_init(bar(p, L::bPSDone + s), 1);
            for (int s = 0; s < L::DSX; ++s) {
                tc::mbar_init(bar(p, L::bDiagFull + s), 1);
                tc::mbar_init(bar(p, L::bDiagEmpty + s), 4);
            }
            for (int s = 0; s < 2; ++s) {
                tc::mbar_init(bar(p, L::bInfoFull + s), 1);
                tc::mbar_init(bar(p, L::bInfoEmpty + s), 4);
            }
        }
        *abort = 0;
        tc::fence_barrier_init();
    }
    if constexpr (LDW && DG < D) {
        // the per-warp copies fill DG columns of each diagonal row: the rest
        // of the rings stays zero
        for (int p = 0; p < NP; ++p)
            for (int o = L::pDQ + 16 * tid; o < L::pP; o += 16 * blockDim.x)
                *(uint4 *)(sm + p * L::kPipe + o) = make_uint4(0, 0, 0, 0);
    }
    if (warp == 1) tc::tmem_alloc(tc::smem_u32(tmem_slot), L::kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 4) {
        if (NP == 2) tc::regs_dec<BwdRegs::producer>();
      if ((warp >> 1) < NP && (warp & 1) == 0) {
        // ---------------- producer of pipeline p: K and V of the tile, then
        // the band Q/dO blocks of every query head of the group (with lse and
        // Delta) through their ring and, for a structured graph, the distance
        // blocks of every head (the count first, to the compute warps) after
        // the band blocks that fit the ring
        const int p = warp >> 1;
        const uint32_t pb = sbase + (uint32_t)(p * L::kPipe);
        volatile int *info = (volatile int *)(sm + L::kMisc + 8) + 2 * p;
        constexpr bool kTmaDiag = DS > 0 && !LDW;
        uint32_t bc = 0, dc = 0;
        bool ok = true;
        int64_t lt = 0;
        for (int64_t t = (int64_t)blockIdx.x * NP + p; ok && t < ntiles; t += stride, ++lt) {
            const TileId id = tile_id(t, ntr);
            const int32_t k0 = id.r0, kvbh = id.bh;
            const int64_t qbh0 = qslice0(kvbh);
            const int n_band = dkv_n_band<BB>(k0, T, a.We);
            const int NB = GQ * n_band;  // band blocks of all heads of the group
            int nd = 0;  // distance blocks of one head
            if constexpr (kTmaDiag) {
                for (int x = 0; x < a.n_off; ++x) nd += (k0 + a.offs[x] <= T - 1) ? 1 : 0;
                const int slot = (int)(lt & 1);
                if (lt >= 2 && !wait(p, L::bInfoEmpty + slot, (uint32_t)(((lt >> 1) - 1) & 1)))
                    break;
                if (lane == 0) {
                    info[slot] = nd;
                    tc::mbar_arrive(bar(p, L::bInfoFull + slot));
                }
            }
            // band block bl (all lanes): lane 0 the TMA copies, every lane a
            // share of lse (base 2) and Delta, zero past the end of the
            // sequence; block bl+1's values are fetched into registers while
            // the producer waits for the next free stage
            constexpr int PL = BB / 32;  // values per lane
            float pf_l[PL], pf_d[PL];
            auto fetch_vals = [&](int bl) {
                const int hq = bl / n_band, b = bl - hq * n_band;
#pragma unroll
                for (int x = 0; x < PL; ++x) {
                    const int64_t i = (int64_t)k0 + b * BB + lane + 32 * x;
                    const size_t gi = (size_t)(qbh0 + hq) * (size_t)T + (size_t)i;
                    const bool in = bl < NB && i < T;
                    pf_l[x] = in ? a.lse[gi] : 0.f;
                    pf_d[x] = in ? a.delta[gi] : 0.f;
                }
            };
            fetch_vals(0);
            auto load_blk = [&](int bl) -> bool {
                const int st = (int)(bc % BS);
                const uint32_t use = bc / BS;
                if (use > 0 && !wait(p, L::bBEmpty + st, (use - 1) & 1)) return false;
                const int hq = bl / n_band;
                const int32_t qrow = k0 + (bl - hq * n_band) * BB;
                const int32_t qz = (int32_t)(qbh0 + hq);
                if (lane == 0) {
                    tc::mbar_arrive_expect_tx(bar(p, L::bBFull + st), 2 * L::kBlk);
                    tma_rows<D, BB>(pb + L::pQ + st * L::kBlk, &tq, qrow, qz, bar(p, L::bBFull + st));
                    tma_rows<D, BB>(pb + L::pDO + st * L::kBlk, &tdo, qrow, qz,
                                    bar(p, L::bBFull + st));
                }
                float *ls = stage_lse(p, st), *dl = ls + BB;
#pragma unroll
                for (int x = 0; x < PL; ++x) {
                    ls[lane + 32 * x] = pf_l[x] * kLog2e;
                    dl[lane + 32 * x] = pf_d[x];
                }
                tc::mbar_arrive(bar(p, L::bBFull + st));
                ++bc;
                fetch_vals(bl + 1);
                return true;
            };
            const int n_pre = NB < BS ? NB : BS;
            int okl = 1;
            if (lane == 0) {
                if (lt >= 1 && !wait(p, L::bKVEmpty, (uint32_t)((lt - 1) & 1))) okl = 0;
                if (okl) {
                    tc::mbar_arrive_expect_tx(bar(p, L::bKVFull), 2 * L::kRow);
                    tma_rows<D, BM>(pb + L::pK, &tkt, k0, kvbh, bar(p, L::bKVFull));
                    tma_rows<D, BM>(pb + L::pV, &tvt, k0, kvbh, bar(p, L::bKVFull));
                }
            }
            ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
            for (int bl = 0; ok && bl < n_pre; ++bl) ok = load_blk(bl);
            if constexpr (kTmaDiag) {
                // distance o of head hq: queries k0+o .. k0+127+o of its slice
                for (int d = 0; ok && d < GQ * nd; ++d) {
                    const int hq = d / nd, dd = d - hq * nd;
                    const int st = (int)(dc % DS);
                    const uint32_t use = dc / DS;
                    if (use > 0 && !wait(p, L::bDiagEmpty + st, (use - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        const int32_t qrow = (int32_t)(k0 + a.offs[a.n_off - nd + dd]);
                        const int32_t qz = (int32_t)(qbh0 + hq);
                        tc::mbar_arrive_expect_tx(bar(p, L::bDiagFull + st), 2 * L::kRow);
                        tma_rows<D, BM>(pb + L::pDQ + st * L::kRow, &tqd, qrow, qz,
                                        bar(p, L::bDiagFull + st));
                        tma_rows<D, BM>(pb + L::pDDO + st * L::kRow, &tdod, qrow, qz,
                                        bar(p, L::bDiagFull + st));
                    }
                    ++dc;
                }
            }
            for (int bl = n_pre; ok && bl < NB; ++bl) ok = load_blk(bl);
        }
      } else if ((warp >> 1) < NP) {
        // ---------------- MMA issuer of pipeline p: S^T and dP^T of block g,
        // then dV += P^T dO and dK += dS^T Q of block g-1
        const int p = warp >> 1;
        const uint32_t pb = sbase + (uint32_t)(p * L::kPipe);
        const uint32_t tp = tmem + p * L::tPipe;
        if (lane == 0) {
            const uint32_t idS = tc::idesc_bf16(BM, BB, false, false);
            const uint32_t idG = tc::idesc_bf16(BM, D, false, true);
            uint32_t gb = 0;
            bool have = false, first = false, ok = true;
            uint32_t pg = 0;
            int64_t plt = 0;
            auto do_dkv = [&]() -> bool {
                const int sb = (int)(pg % SB), st = (int)(pg % BS);
                if (first && !wait(p, L::bInit, (uint32_t)(plt & 1))) return false;
                if (!wait(p, L::bPFull + sb, (pg / SB) & 1)) return false;
                tc::tc_fence_after();
                const uint32_t qa = pb + L::pQ + st * L::kBlk, da = pb + L::pDO + st * L::kBlk;
                if constexpr (PS > 0) {
                    const int ps = (int)(pg % PS);
                    const uint32_t pa = pb + L::pP + ps * L::kPTile;
                    const uint32_t dsa = pb + L::pDS + ps * L::kPTile;
#pragma unroll
                    for (int kk = 0; kk < BB / 16; ++kk) {
                        tc::mma_bf16_ss(tp + L::tDV, tc::sdesc_sw128(pa + kk * 32, 16, 1024),
                                        tc::sdesc_sw128(da + kk * 16 * 128, BB * 128, 1024), idG,
                                        1u);
                        tc::mma_bf16_ss(tp + L::tDK, tc::sdesc_sw128(dsa + kk * 32, 16, 1024),
                                        tc::sdesc_sw128(qa + kk * 16 * 128, BB * 128, 1024), idG,
                                        1u);
                    }
                    tc::mma_commit(bar(p, L::bBEmpty + st));
                    tc::mma_commit(bar(p, L::bPSDone + ps));
                } else {
#pragma unroll
                    for (int kk = 0; kk < BB / 16; ++kk) {
                        tc::mma_bf16_ts(tp + L::tDV, tp + L::tS + sb * BB + kk * 8,
                                        tc::sdesc_sw128(da + kk * 16 * 128, BB * 128, 1024), idG,
                                        1u);
                        tc::mma_bf16_ts(tp + L::tDK, tp + L::tDP + sb * BB + kk * 8,
                                        tc::sdesc_sw128(qa + kk * 16 * 128, BB * 128, 1024), idG,
                                        1u);
                    }
                    tc::mma_commit(bar(p, L::bBEmpty + st));
                    tc::mma_commit(bar(p, L::bSFree + sb));
                }
                tc::mma_commit(bar(p, L::bDKVDone + sb));
                return true;
            };
            int64_t lt = 0;
            for (int64_t t = (int64_t)blockIdx.x * NP + p; ok && t < ntiles; t += stride, ++lt) {
                const TileId id = tile_id(t, ntr);
                const int NB = GQ * dkv_n_band<BB>(id.r0, T, a.We);
                if (!wait(p, L::bKVFull, (uint32_t)(lt & 1))) break;
                const uint32_t ka = pb + L::pK, va = pb + L::pV;
                for (int bl = 0; bl < NB; ++bl) {
                    const int st = (int)(gb % BS), sb = (int)(gb % SB);
                    // one S^T buffer: dV/dK of the previous block free it first
                    if (SB == 1 && have) {
                        if (!do_dkv()) {
                            ok = false;
                            break;
                        }
                        have = false;
                    }
                    if (!wait(p, L::bBFull + st, (gb / BS) & 1) ||
                        (gb >= SB && !wait(p, L::bSFree + sb, ((gb / SB) - 1) & 1))) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t qa = pb + L::pQ + st * L::kBlk, da = pb + L::pDO + st * L::kBlk;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t offr = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                        const uint32_t offb = (kk >> 2) * (BB * 128) + (kk & 3) * 32;
                        tc::mma_bf16_ss(tp + L::tS + sb * BB, tc::sdesc_sw128(ka + offr, 16, 1024),
                                        tc::sdesc_sw128(qa + offb, 16, 1024), idS, kk > 0);
                        tc::mma_bf16_ss(tp + L::tDP + sb * BB,
                                        tc::sdesc_sw128(va + offr, 16, 1024),
                                        tc::sdesc_sw128(da + offb, 16, 1024), idS, kk > 0);
                    }
                    tc::mma_commit(bar(p, L::bSFull + sb));
                    if (bl == NB - 1) tc::mma_commit(bar(p, L::bKVEmpty));
                    if (SB > 1 && have && !do_dkv()) {
                        ok = false;
                        break;
                    }
                    have = true;
                    pg = gb;
                    first = (bl == 0);
                    plt = lt;
                    ++gb;
                }
                // the tile's last dV/dK MMAs go now: its epilogue waits for them
                if (ok && have) {
                    ok = do_dkv();
                    have = false;
                }
            }
        }
      }
    } else {
        // ---------------- compute warpgroup of pipeline p: thread r = key row
        // r = TMEM lane r
        if (NP == 2) tc::regs_inc<BwdRegs::compute>();
        const int p = (warp - 4) >> 2;
        const int r = tid - 128 - 128 * p;
        uint8_t *pm = sm + p * L::kPipe;
        const uint32_t lane_off = (uint32_t)(((warp - 4) & 3) * 32) << 16;
        const uint32_t tbase = tmem + p * L::tPipe + lane_off;
        const uint32_t tS = tbase + L::tS, tDP = tbase + L::tDP;
        const uint32_t tDV = tbase + L::tDV, tDK = tbase + L::tDK;
        const float c2 = a.scale2;
        const int wq = r >> 5;  // warp within the group: key rows 32 wq .. 32 wq + 31
        volatile int *info = (volatile int *)(sm + L::kMisc + 8) + 2 * p;
        uint32_t gb = 0, dc = 0;
        bool ok = true;
        int64_t lt = 0;
        for (int64_t t = (int64_t)blockIdx.x * NP + p; ok && t < ntiles; t += stride, ++lt) {
            const TileId id = tile_id(t, ntr);
            const int32_t k0 = id.r0, kvbh = id.bh;
            const int64_t qbh0 = qslice0(kvbh);
            const int n_band = dkv_n_band<BB>(k0, T, a.We);
            const int NB = GQ * n_band;
            const int64_t j = k0 + r;
            const bool row_ok = j < T;
            if (!__all_sync(0xffffffffu, wait(p, L::bKVFull, (uint32_t)(lt & 1)))) break;
            // diagonal slots: the Q and dO rows of the queries that reach this
            // key by a distance link (or by a CSR residual entry), for every
            // query head of the group, fetched by this warp itself; (p, dS) of
            // each edge comes from the dQ kernel's cache, or is recomputed from
            // lse and Delta of the query, loaded three slots ahead
            // D = 64: diagonal sums in registers, stored to TMEM after the
            // slots; D = 128: summed in TMEM directly (zeroed first)
            constexpr bool kRegAcc = D == 64;
            float adk[kRegAcc ? D : 1], adv[kRegAcc ? D : 1];
#pragma unroll
            for (int x = 0; x < (kRegAcc ? D : 1); ++x) adk[x] = adv[x] = 0.f;
            if constexpr (!kRegAcc) {
                tmem_store_row<D>(tDV, nullptr);
                tmem_store_row<D>(tDK, nullptr);
                tc::tmem_st_wait();
            }
            if constexpr (DS > 0) {
                // slots per head: the tile's distance blocks (count from the
                // producer), or, for CSR lists, the longest residual transpose
                // list of this warp's keys
                int nd = 0;
                int64_t rs = 0, nb = 0, resid = 0;
                if constexpr (!LDW) {
                    const int slot = (int)(lt & 1);
                    ok = __all_sync(0xffffffffu,
                                    wait(p, L::bInfoFull + slot, (uint32_t)((lt >> 1) & 1)));
                    nd = ok ? info[slot] : 0;
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar(p, L::bInfoEmpty + slot));
                } else {
                    if (row_ok) {
                        rs = a.rev_rowptr[j];
                        nb = (T - j < W) ? T - j : W;
                        resid = a.rev_rowptr[j + 1] - rs - nb;
                    }
                    nd = (int)__reduce_max_sync(0xffffffffu, (unsigned)resid);
                }
                const int off_first = a.n_off - nd;
                // slot d: link (or residual position) d % nd of query head
                // d / nd; its query row, -1 if none
                const int nds = GQ * nd;
                // slot d -> (query head d / nd, link d % nd); no division
                // without grouped heads
                auto link_of = [&](int d) { return GQ == 1 ? d : d % nd; };
                auto head_of = [&](int d) { return GQ == 1 ? 0 : d / nd; };
                auto key_of = [&](int d) -> int32_t {
                    if (!row_ok || d >= nds) return -1;
                    const int dd = link_of(d);
                    if constexpr (!LDW) {
                        const int64_t cand = j + a.offs[off_first + dd];
                        return cand < T ? (int32_t)cand : -1;
                    }
                    return dd < resid ? __ldg(a.rev_colidx + rs + nb + dd) : -1;
                };
                const bool cached = a.kind == 0 && a.pds != nullptr;
                auto edge_vals = [&](int d, int64_t i) -> float2 {
                    if (i < 0) return make_float2(0.f, 0.f);
                    const size_t qbh = (size_t)(qbh0 + head_of(d));
                    if (cached)
                        return a.pds[((size_t)(off_first + link_of(d)) * (size_t)a.BH + qbh) *
                                         (size_t)T +
                                     (size_t)i];
                    return make_float2(a.lse[qbh * (size_t)T + i], a.delta[qbh * (size_t)T + i]);
                };
                int64_t i_cur = key_of(0), i_nxt = key_of(1), i_n2 = key_of(2), i_n3 = key_of(3);
                float2 v_cur = edge_vals(0, i_cur), v_nxt = edge_vals(1, i_nxt), v_n2 = edge_vals(2, i_n2);
                auto body = [&](int d, int st) {
                    const int64_t i_n4 = key_of(d + 4);
                    const float2 v_n3 = edge_vals(d + 3, i_n3);
                    const uint8_t *qt = pm + L::pDQ + st * L::kRow;
                    const uint8_t *dt = pm + L::pDDO + st * L::kRow;
                    float pr = 0.f, ds = 0.f;
                    if (i_cur >= 0) {
                        if (cached) {
                            pr = v_cur.x;
                            ds = v_cur.y;
                        } else {
                            const float sdot = dot_bf_smem_smem<DG>(qt, pm + L::pK, BM, r);
                            const float dpdot = dot_bf_smem_smem<DG>(dt, pm + L::pV, BM, r);
                            pr = tc::ex2(fmaf(sdot, c2, -v_cur.x * kLog2e));
                            ds = pr * (dpdot - v_cur.y);
                        }
                        if constexpr (kRegAcc) {
                            axpy_bf_smem<DG>(adv, pr, dt, BM, r);
                            axpy_bf_smem<DG>(adk, ds, qt, BM, r);
                        }
                    }
                    // (warp-collective: every lane, whether or not its key has the slot)
                    if constexpr (!kRegAcc) {
                        tmem_axpy_row<D>(tDV, pr, i_cur >= 0, dt, BM, r);
                        tmem_axpy_row<D>(tDK, ds, i_cur >= 0, qt, BM, r);
                    }
                    i_cur = i_nxt;
                    i_nxt = i_n2;
                    i_n2 = i_n3;
                    i_n3 = i_n4;
                    v_cur = v_nxt;
                    v_nxt = v_n2;
                    v_n2 = v_n3;
                };
                if constexpr (LDW) {
                    rows::warp_slots<DG, DS>(
                        nds, sbase + (uint32_t)(p * L::kPipe + L::pDQ),
                        sbase + (uint32_t)(p * L::kPipe + L::pDDO), (uint32_t)L::kRow, a.q,
                        a.dout, a.l2pf != 0, lane, wq,
                        [&](int d) {
                            return (size_t)(qbh0 + (nd > 0 ? head_of(d) : 0)) * (size_t)T * DG;
                        },
                        key_of, body);
                } else {
                    for (int d = 0; ok && d < nds; ++d) {
                        const int st = (int)(dc % DS);
                        if (!__all_sync(0xffffffffu, wait(p, L::bDiagFull + st, (dc / DS) & 1))) {
                            ok = false;
                            break;
                        }
                        body(d, st);
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(bar(p, L::bDiagEmpty + st));
                        ++dc;
                    }
                }
            }
            if (!ok) break;
            // this warp is done reading K and V of the tile
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(p, L::bKVEmpty));
            if constexpr (kRegAcc) {
                tmem_store_row<D>(tDV, adv);
                tmem_store_row<D>(tDK, adk);
            }
            tc::tmem_st_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(p, L::bInit));

            // band blocks of every head of the group: P^T and dS^T (bf16) over
            // S^T and dP^T
            uint32_t gb_last = gb;
            for (int bl = 0; ok && bl < NB; ++bl, ++gb) {
                const int sb = (int)(gb % SB), st = (int)(gb % BS);
                const int32_t v0 = (GQ == 1 ? bl : bl % n_band) * BB;
                gb_last = gb;
                if (!wait(p, L::bSFull + sb, (gb / SB) & 1) ||
                    !wait(p, L::bBFull + st, (gb / BS) & 1)) {  // lse / Delta staged
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                float s[BB], dp[BB];
                tc::tmem_ld_n<BB>(tS + sb * BB, (uint32_t *)s);
                tc::tmem_ld_n<BB>(tDP + sb * BB, (uint32_t *)dp);
                tc::tmem_ld_wait();
                if (PS > 0) {  // S^T and dP^T are in registers: the buffer is free
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar(p, L::bSFree + sb));
                }
                const float *lse_s = stage_lse(p, st), *del_s = lse_s + BB;
                const bool need_mask = a.nf > 0 || (v0 < BM - 1) || (v0 + BB - 1 > a.We - 1) ||
                                       ((int64_t)k0 + v0 + BB - 1 > T - 1);
                if (need_mask) {
                    // keep columns [c_lo, c_hi]: r <= v <= r+W-1 and query < T,
                    // plus the folded links v = r + o
                    const int64_t vlim = T - 1 - k0;
                    int64_t hi = (int64_t)r + W - 1;
                    if (hi > vlim) hi = vlim;
                    const int64_t lo = r;
                    const int c_lo = (int)(lo - v0 < 0 ? 0 : (lo - v0 > BB ? BB : lo - v0));
                    const int c_hi =
                        (int)(hi - v0 > BB - 1 ? BB - 1 : (hi - v0 < -1 ? -1 : hi - v0));
                    uint64_t keep = tc::bits_range(c_lo, c_hi);  // bit c: column c kept
                    if (a.nf > 0) {
#pragma unroll
                        for (int x = 0; x < kMaxFold; ++x) {
                            const int64_t v = (int64_t)r + a.fold[x];
                            if (x < a.nf && v <= vlim && v >= v0 && v < v0 + BB)
                                keep |= 1ull << (int)(v - v0);
                        }
                    }
                    // 16-column chunks outside every kept range of this warp: P = dS = 0
#pragma unroll
                    for (int c16 = 0; c16 < BB / 16; ++c16) {
                        if (__any_sync(0xffffffffu, ((keep >> (16 * c16)) & 0xffffull) != 0ull)) {
#pragma unroll
                            for (int c = 16 * c16; c < 16 * c16 + 16; ++c) {
                                const float pr =
                                    ((keep >> c) & 1ull) ? tc::ex2(fmaf(s[c], c2, -lse_s[c])) : 0.f;
                                s[c] = pr;
                                dp[c] = pr * (dp[c] - del_s[c]);
                            }
                        } else {
#pragma unroll
                            for (int c = 16 * c16; c < 16 * c16 + 16; ++c) s[c] = dp[c] = 0.f;
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < BB; ++c) {
                        const float pr = tc::ex2(fmaf(s[c], c2, -lse_s[c]));
                        s[c] = pr;
                        dp[c] = pr * (dp[c] - del_s[c]);
                    }
                }
                if constexpr (PS > 0) {
                    const int ps = (int)(gb % PS);
                    if (gb >= PS && !wait(p, L::bPSDone + ps, ((gb / PS) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    store_row64_bf16(pm + L::pP + ps * L::kPTile, r, s);
                    store_row64_bf16(pm + L::pDS + ps * L::kPTile, r, dp);
                    tc::fence_proxy_async_smem();
                } else {
                    uint32_t w[BB / 2];
                    pack_bf16_row<BB>(s, w);
                    tc::tmem_st_n<BB / 2>(tS + sb * BB, w);
                    pack_bf16_row<BB>(dp, w);
                    tc::tmem_st_n<BB / 2>(tDP + sb * BB, w);
                    tc::tmem_st_wait();
                    tc::tc_fence_before();
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar(p, L::bPFull + sb));
            }
            if (!ok) break;
            if (!wait(p, L::bDKVDone + (int)(gb_last % SB), (gb_last / SB) & 1)) break;
            tc::tc_fence_after();
            const size_t wrow = (size_t)kvbh * (size_t)T + (size_t)(k0 + 32 * wq);
            tmem_rows_to_global<DG>(tDV, 1.f, a.dv + wrow * DG, T - (k0 + 32 * wq), lane);
            tmem_rows_to_global<DG>(tDK, a.scale, a.dk + wrow * DG, T - (k0 + 32 * wq), lane);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, L::kTmemCols);
    }
}

template <int NP>
inline bool regs_cover(const void *kern) {
    // setmaxnreg.inc waits until the CTA's pool holds what it asks for: the
    // launch must provide the whole warpgroup split
    if (NP != 2) return true;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return false;
    return fa.numRegs * (128 + 128 * NP) >= 128 * BwdRegs::producer + 128 * NP * BwdRegs::compute;
}

template <int D, int NP, int BB, int SB, int BSQ, int BSK, int DS, int PS, bool LDW, int DG>
sa_status launch_band_bwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                          const sa_tensor *o, const float *lse, const sa_tensor *dout,
                          const sa_graph_s *g, float scale, sa_tensor *dq, sa_tensor *dk,
                          sa_tensor *dv, float *delta, void *pds, cudaStream_t s) {
    using LQ = LayoutDQ<D, NP, BB, SB, BSQ, DS, PS>;
    using LK = LayoutDKV<D, NP, BB, SB, BSK, DS, PS>;
    static_assert(LQ::kAlloc <= 232448 && LK::kAlloc <= 232448, "shared memory budget");
    constexpr int kThreads = 128 + 128 * NP;
    static_assert(DG == D || (D == 64 && DG == 32), "row length");
    auto kq = band_bwd_dq_kernel<D, NP, BB, SB, BSQ, DS, PS, LDW, DG>;
    auto kkv = band_bwd_dkdv_kernel<D, NP, BB, SB, BSK, DS, PS, LDW, DG>;
    static int regs_ok = -1;
    if (regs_ok < 0)
        regs_ok = regs_cover<NP>((const void *)kq) && regs_cover<NP>((const void *)kkv);
    if (!regs_ok) {
        sa_record_cuda_error(cudaErrorInvalidConfiguration,
                             "band_bwd: launch registers below the warpgroup split");
        return SA_ERR_CUDA;
    }
    const int64_t BH = q->B * q->H, BHkv = k->B * k->H, T = q->T;
    // 128-row boxes for the tiles, BB-row boxes for the band rings
    CUtensorMap mq, mdo, mk, mv, mqb, mdob, mkb, mvb;
    if (!sa_tmap_bf16_3d(&mq, q->ptr, DG, T, BH, BM) ||
        !sa_tmap_bf16_3d(&mdo, dout->ptr, DG, T, BH, BM) ||
        !sa_tmap_bf16_3d(&mk, k->ptr, DG, T, BHkv, BM) ||
        !sa_tmap_bf16_3d(&mv, v->ptr, DG, T, BHkv, BM) ||
        !sa_tmap_bf16_3d(&mqb, q->ptr, DG, T, BH, BB) ||
        !sa_tmap_bf16_3d(&mdob, dout->ptr, DG, T, BH, BB) ||
        !sa_tmap_bf16_3d(&mkb, k->ptr, DG, T, BHkv, BB) ||
        !sa_tmap_bf16_3d(&mvb, v->ptr, DG, T, BHkv, BB)) {
        sa_record_cuda_error(cudaErrorInvalidValue, "band_bwd: tensor map encoding");
        return SA_ERR_CUDA;
    }
    BwdArgs a{};
    a.T = T;
    a.BH = BH;
    a.H = q->H;
    a.Hkv = k->H;
    a.l2pf = (double)BH * (double)T * DG * 2 * 2 > 64.0 * 1024 * 1024 ? 1 : 0;
    a.W = g->W;
    a.kind = g->kind;
    a.We = sa_fold_links(g, BB, kMaxFold, a.fold, &a.nf, a.offs, &a.n_off);
    a.rowptr = g->rowptr;
    a.colidx = g->colidx;
    a.rev_rowptr = g->rev_rowptr;
    a.rev_colidx = g->rev_colidx;
    a.o = (const __nv_bfloat16 *)o->ptr;
    a.k = (const __nv_bfloat16 *)k->ptr;
    a.v = (const __nv_bfloat16 *)v->ptr;
    a.q = (const __nv_bfloat16 *)q->ptr;
    a.dout = (const __nv_bfloat16 *)dout->ptr;
    a.lse = lse;
    a.delta = delta;
    a.pds = (g->kind == 0 && g->n_off > 0) ? (float2 *)pds : nullptr;
    a.dq = (__nv_bfloat16 *)dq->ptr;
    a.dk = (__nv_bfloat16 *)dk->ptr;
    a.dv = (__nv_bfloat16 *)dv->ptr;
    a.scale = scale;
    a.scale2 = scale * kLog2e;
    a.err = sa_device_error_word();
    if (!a.err) return SA_ERR_CUDA;
    SA_CUDA_TRY(sa_smem_optin((const void *)kq, LQ::kAlloc));
    SA_CUDA_TRY(sa_smem_optin((const void *)kkv, LK::kAlloc));
    // persistent: one CTA per SM, NP tiles in flight in each; dQ tiles run
    // over query slices, dK/dV tiles over key/value slices
    int sms = 0;
    SA_CUDA_TRY(sa_sm_count(&sms));
    auto grid_for = [&](int64_t slices) {
        const int64_t nctas = (((T + BM - 1) / BM) * slices + NP - 1) / NP;
        return (unsigned)(nctas < sms ? nctas : sms);
    };
    SA_LAUNCH("band_bwd_dq", s,
              kq<<<grid_for(BH), kThreads, LQ::kAlloc, s>>>(mq, mdo, mkb, mvb, mk, mv, a));
    SA_LAUNCH("band_bwd_dkdv", s,
              kkv<<<grid_for(BHkv), kThreads, LK::kAlloc, s>>>(mk, mv, mqb, mdob, mq, mdo, a));
    SA_CUDA_TRY(cudaGetLastError());
    return SA_OK;
}

}  // namespace

bool sa_band_bwd_supported(const sa_tensor *q, const sa_tensor *k, const sa_graph_s *g) {
    if (q->dtype != SA_BF16 || (q->D != 32 && q->D != 64 && q->D != 128)) return false;
    if (g->W < 1) return false;
    // 32-bit tile coordinates; the CSR gathers address rows of all slices
    // (slice * T + row) as one int32 coordinate
    if (q->B * q->H >= ((int64_t)1 << 31) || q->T >= ((int64_t)1 << 31)) return false;
    if (g->kind == 1 && q->B * q->H * q->T >= ((int64_t)1 << 31)) return false;
    if (g->kind == 1 && (!g->rowptr || !g->rev_rowptr)) return false;
    return true;
}

sa_status sa_band_bwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                      const sa_tensor *out, const float *lse, const sa_tensor *dout,
                      const sa_graph_s *g, const GraphView &, float scale, sa_tensor *dq,
                      sa_tensor *dk, sa_tensor *dv, float *delta, void *pds, cudaStream_t s) {
    const bool diag = (g->kind == 0) ? g->n_off > 0 : (g->max_resid > 0 || g->max_resid_rev > 0);
    // <D, pipelines, band block, S buffers, dQ ring stages, dK/dV ring stages,
    //  diagonal stages, shared-memory P/dS tiles>, sized to the 227 KB of
    // shared memory and 512 TMEM columns
    const bool csr = g->kind == 1;
#define SA_BWD_ARGS q, k, v, out, lse, dout, g, scale, dq, dk, dv, delta, pds, s
    // (D = 32 runs on the D = 64 tiles, its rows zero-extended)
    if (q->D == 32) {
        if (!diag) return launch_band_bwd<64, 2, 32, 2, 4, 4, 0, 0, false, 32>(SA_BWD_ARGS);
        return csr ? launch_band_bwd<64, 2, 32, 2, 2, 2, 2, 0, true, 32>(SA_BWD_ARGS)
                   : launch_band_bwd<64, 2, 32, 2, 2, 2, 2, 0, false, 32>(SA_BWD_ARGS);
    }
    if (q->D == 64) {
        if (!diag) return launch_band_bwd<64, 2, 32, 2, 4, 4, 0, 0, false, 64>(SA_BWD_ARGS);
        return csr ? launch_band_bwd<64, 2, 32, 2, 2, 2, 2, 0, true, 64>(SA_BWD_ARGS)
                   : launch_band_bwd<64, 2, 32, 2, 2, 2, 2, 0, false, 64>(SA_BWD_ARGS);
    }
    // D = 128: one pipeline, P^T / dS^T and dS in shared memory; with
    // diagonal edges a one-stage diagonal ring and two-stage band rings
    if (!diag) return launch_band_bwd<128, 1, 64, 2, 3, 3, 0, 1, false, 128>(SA_BWD_ARGS);
    return csr ? launch_band_bwd<128, 1, 64, 2, 2, 2, 1, 1, true, 128>(SA_BWD_ARGS)
               : launch_band_bwd<128, 1, 64, 2, 2, 2, 1, 1, false, 128>(SA_BWD_ARGS);
#undef SA_BWD_ARGS
}
