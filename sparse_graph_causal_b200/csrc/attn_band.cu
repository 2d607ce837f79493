// attn_band.cu -- forward on tcgen05 band tiles fused with the gathered edges.
//
// A tile is 128 consecutive queries [q0, q0+128) of one (b, h) slice.
//  * Window edges (the band of "MiniGPT (Part 6)", section "A mask is not
//    enough": keys j <= i with i - j < W) run as dense 128 x 64 blocks on the
//    tensor cores: keys [q0-W+1, q0+127] are cut into blocks of 64 starting at
//    q0-W+1, so in block coordinates u = 64 b + c a query row r keeps exactly
//    r <= u <= r+W-1 (and j >= 0).  S = Q K^T lands in TMEM, the softmax
//    warpgroup turns it into P (bf16, written back over S in TMEM), and
//    O += P V accumulates in TMEM with P read from TMEM by the MMA.
//  * Every other edge -- the 2^k distance links of "SpatialLM-Mini ...",
//    section "How tokens choose whom to listen to", or the non-window part of
//    a CSR list ("Longer Attention Span ...", Abstract) -- is a "diagonal"
//    block: 128 key rows, row r belonging to query r (for a distance o the
//    keys q0-o .. q0+127-o; for CSR lists slot s of every row's residual
//    list).  For a distance link the block is 128 contiguous rows: the
//    producer loads it as TMA boxes into a DS-stage ring (with an L2
//    prefetch a few blocks ahead when K and V exceed L2).  For CSR lists
//    each softmax warp copies the K and V rows of its own 32 queries itself
//    with 16-byte cp.async copies, DS slots ahead, into the same swizzled
//    layout (sa_rows.cuh).  Thread r then takes the dot product of its own
//    row on the CUDA cores.
//  * Links short enough to fall inside the key span that the band blocks
//    cover anyway (at most kMaxFold) are folded into the band blocks as
//    extra kept columns; a CSR graph whose rows all start with the same key
//    prefix (global tokens) gets one more band block holding keys 0 .. 63.
//    Each row's kept columns of a block are one 64-bit mask.
//  * One online softmax (running max m and sum l per row, base 2) covers both
//    classes: the diagonal blocks go first, their weighted sum initialises O
//    in TMEM, then the band blocks rescale O only when a row's max grows by
//    more than 2^8 (the stale max keeps every p <= 256, exact in fp32).
//  * Epilogue: out = O / l (bf16, round to nearest even), lse = (m + log2 l) ln 2.
//
// The kernel is persistent and runs NP (1 or 2) independent tile pipelines
// per CTA, each with its own shared-memory rings, TMEM columns (two S
// buffers and O) and barriers, so that the softmax of one tile overlaps the
// loads, MMAs and softmax of the other.  Warp roles: warp 2p is the TMA
// producer of pipeline p (Q, the band K/V ring and the distance blocks),
// warp 2p+1 its
// MMA issuer (warp 1 also allocates TMEM), warps 4+4p .. 7+4p its softmax
// warpgroup (thread = query row = TMEM lane).  With two pipelines the
// producer warpgroup hands registers to the softmax warpgroups (setmaxnreg).
// Every mbarrier wait is bounded (2 s); on expiry the CTA records
// SA_DEVERR_TIMEOUT in the device error word, all roles leave their loops,
// TMEM is freed and the kernel returns.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sa_band.cuh"
#include "sa_rows.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace {

constexpr int BM = 128;             // queries per tile
constexpr int BN = 64;              // keys per band block
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Diagonal rows are prefetched into L2 ahead of their copies when K and V do
// not fit in L2 (long links and random CSR keys then miss it, and the copy
// ring alone keeps too few DRAM reads in flight); with L2-resident K and V
// the prefetches are pure overhead and are skipped.
constexpr double kL2ResidentBytes = 64.0 * 1024 * 1024;
// Distance blocks (TMA boxes) are prefetched into L2 this many blocks ahead
// of their loads under the same condition.
constexpr int kPrefetchBlocks = 4;
// Register budgets with two pipelines (384 threads launched at 168 each):
// the producer warpgroup keeps 56, the softmax warpgroups take the rest.
template <int DS>
struct Regs {
    static constexpr int producer = 56;
    static constexpr int softmax = 224;
    static_assert(128 * producer + 256 * softmax <= 384 * 168, "register split");
};

// Distance links short enough to fall inside the span of key blocks that a
// tile covers anyway are folded into the band blocks: row r keeps, besides its
// window, the single key i - o of each folded link o (at most kMaxFold).
constexpr int kMaxFold = 4;

struct FwdArgs {
    int64_t T;
    int64_t BH;
    int64_t H, Hkv;                // query and key/value heads (grouped-query attention)
    int32_t W;          // band width (structured window or verified CSR band)
    int32_t We;         // span of the band blocks: W, or the longest folded link + 1
    int32_t nf;         // folded links
    int32_t fold[kMaxFold];
    int32_t kind;       // 0 structured, 1 CSR
    int32_t gp;         // CSR: every row i holds keys 0 .. min(gp, i + 1) - 1 (0: none)
    int32_t n_off;
    int32_t l2pf;                  // diagonal rows prefetched into L2 ahead of their copies
    int64_t offs[SA_MAX_OFFSETS];  // distances (structured), descending
    const int64_t *rowptr;         // CSR
    const int32_t *colidx;
    const __nv_bfloat16 *k, *v;    // diagonal rows are copied from here
    __nv_bfloat16 *out;
    float *lse;
    float scale2;                  // scale * log2(e)
    int *err;
};

// Shared memory: NP pipeline regions, then barriers.  All tiles are K-major
// with 128-byte swizzle, 64 columns (128 bytes) per row and chunk.
template <int D, int NP, int KS, int VS, int DS>
struct Layout {
    static constexpr int kQTile = BM * D * 2;          // 128 rows x D
    static constexpr int kBlk = BN * D * 2;            // 64 rows x D
    static constexpr int pQ = 0;
    static constexpr int pK = pQ + kQTile;              // band K ring
    static constexpr int pV = pK + KS * kBlk;           // band V ring
    static constexpr int pDK = pV + VS * kBlk;          // diagonal K ring
    static constexpr int pDV = pDK + DS * kQTile;       // diagonal V ring
    static constexpr int kPipe = pDV + DS * kQTile;
    static constexpr int kBars = NP * kPipe;
    // barriers of one pipeline (S, P, PVDone per S buffer: P is written over S)
    static constexpr int bQFull = 0, bQEmpty = 1;
    static constexpr int bKFull = 2, bKEmpty = bKFull + KS;
    static constexpr int bVFull = bKEmpty + KS, bVEmpty = bVFull + VS;
    static constexpr int bSFull = bVEmpty + VS, bSFree = bSFull + 2;
    static constexpr int bPFull = bSFree + 2, bPVDone = bPFull + 2;
    static constexpr int bOInit = bPVDone + 2;
    // distance blocks loaded by the producer with TMA (structured graphs): the
    // ring's barriers and the per-tile block count handed to the softmax warps
    static constexpr int DSX = DS > 0 ? DS : 1;
    static constexpr int bDiagFull = bOInit + 1, bDiagEmpty = bDiagFull + DSX;
    static constexpr int bInfoFull = bDiagEmpty + DSX, bInfoEmpty = bInfoFull + 2;
    static constexpr int nBarsPipe = bInfoEmpty + 2;
    static constexpr int kMisc = kBars + NP * nBarsPipe * 8;  // tmem slot, abort, info[NP][2]
    static constexpr int kTotal = kMisc + 8 + 8 * NP;
    static constexpr int kAlloc = kTotal + 1024;         // alignment slack
    // TMEM columns of pipeline p start at 256 p: S buffers [0, BN) and
    // [BN, 2 BN) (P, bf16, over the first BN/2 columns of its S buffer), O at 2 BN
    static constexpr uint32_t tPipe = 256, tS0 = 0, tO = 2 * BN;
    static constexpr uint32_t kTmemCols = 512;
    static_assert(2 * BN + D <= 256, "TMEM columns of a pipeline");
    static_assert(kQTile % 1024 == 0 && kBlk % 1024 == 0, "swizzle atoms");
};

// Geometry of query tile t (tiles run over B*H slices, 128 queries each).
// 32-bit: the band path requires T < 2^31 and W + 127 < 2^31.
// npre = 1 when the tile starts with the shared-prefix block (keys 0 .. 63,
// kept for row i below min(gp, i - W + 1), i.e. outside its window); the
// band blocks follow.
struct TileGeom {
    int32_t bh, kvbh, q0, kb0, b_first, n_band, npre;
};

// kvbh: the key/value slice that query slice bh reads (query head h of batch
// row b reads key/value head h / (H / Hkv)).
__device__ __forceinline__ TileGeom tile_geom(int64_t t, int64_t ntq, int64_t T, int32_t W,
                                              int64_t H, int64_t Hkv, int32_t gp) {
    TileGeom g;
    const int64_t bh = t / ntq;
    g.bh = (int32_t)bh;
    g.kvbh = (int32_t)((bh / H) * Hkv + (bh % H) / (H / Hkv));
    g.q0 = (int32_t)((t - bh * ntq) * BM);
    g.kb0 = g.q0 - W + 1;                                             // key of u = 0
    const int32_t last_key = (g.q0 + BM - 1 < T - 1) ? g.q0 + BM - 1 : (int32_t)(T - 1);
    const int32_t nblk = (last_key - g.kb0) / BN + 1;                 // blocks up to the last key
    const int32_t need = W - 1 - g.q0;                                // first block with a key >= 0
    g.b_first = need > 0 ? need / BN : 0;
    g.n_band = nblk - g.b_first;
    g.npre = (gp > 0 && last_key >= W) ? 1 : 0;  // (no prefix on structured graphs: W = We)
    return g;
}

// Pipeline p of CTA c takes the tiles c NP + p, c NP + p + NP G, ... (G CTAs):
// the two pipelines of a CTA work on neighbouring tiles.  Every ring keeps its
// phase across tiles, so the loads and MMAs of the next tile proceed while
// the current one finishes.
// LDW selects how the diagonal slots are loaded: false -- the producer loads
// each distance block as TMA boxes (structured graphs: 128 contiguous rows);
// true -- every softmax warp copies its own rows (CSR lists: one random row
// per tile row, rows/sa_rows.cuh).
// DG: the row length of q, k, v and out in global memory; D the width of the
// tiles in shared memory and TMEM.  DG = 32 runs on the D = 64 tiles: the TMA
// boxes read 64 columns, the 32 beyond each row come back as zeros (out of
// bounds of the tensor map) and add nothing to any product.
template <int D, int NP, int KS, int VS, int DS, bool LDW, int DG>
__global__ void __launch_bounds__(128 + 128 * NP, 1)
band_fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tkd,
                const __grid_constant__ CUtensorMap tvd, const FwdArgs a) {
    using L = Layout<D, NP, KS, VS, DS>;
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
    const int64_t ntq = (T + BM - 1) / BM, ntiles = ntq * a.BH;
    const int64_t stride = (int64_t)gridDim.x * NP;

    if (tid == 0) {
        for (int p = 0; p < NP; ++p) {
            tc::mbar_init(bar(p, L::bQFull), 1);
            tc::mbar_init(bar(p, L::bQEmpty), 5);  // last S MMA commit + 4 softmax warps
            for (int s = 0; s < 2; ++s) {
                tc::mbar_init(bar(p, L::bSFull + s), 1);
                tc::mbar_init(bar(p, L::bSFree + s), 1);   // P V of the buffer's block done
                tc::mbar_init(bar(p, L::bPFull + s), 4);
                tc::mbar_init(bar(p, L::bPVDone + s), 1);
            }
            for (int s = 0; s < KS; ++s) {
                tc::mbar_init(bar(p, L::bKFull + s), 1);
                tc::mbar_init(bar(p, L::bKEmpty + s), 1);
            }
            for (int s = 0; s < VS; ++s) {
                tc::mbar_init(bar(p, L::bVFull + s), 1);
                tc::mbar_init(bar(p, L::bVEmpty + s), 1);
            }
            tc::mbar_init(bar(p, L::bOInit), 4);
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
            for (int o = L::pDK + 16 * tid; o < L::kPipe; o += 16 * blockDim.x)
                *(uint4 *)(sm + p * L::kPipe + o) = make_uint4(0, 0, 0, 0);
    }
    if (warp == 1) tc::tmem_alloc(tc::smem_u32(tmem_slot), L::kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 4) {
        // one register budget per warpgroup, set where it dominates the roles
        if (NP == 2) tc::regs_dec<Regs<DS>::producer>();
      if ((warp >> 1) < NP && (warp & 1) == 0) {
        // ---------------- producer of pipeline p (lane 0): per tile Q, the band
        // K/V blocks through their rings and, for a structured graph, the
        // distance blocks (the count first, to the softmax warps) after the
        // band blocks that fit the rings
        const int p = warp >> 1;
        const uint32_t pb = sbase + (uint32_t)(p * L::kPipe);
        volatile int *info = (volatile int *)(sm + L::kMisc + 8) + 2 * p;
        if (lane == 0) {
            tc::tma_prefetch_desc(&tq);
            tc::tma_prefetch_desc(&tk);
            tc::tma_prefetch_desc(&tv);
            uint32_t kc = 0, vc = 0, dc = 0;  // K, V and distance blocks loaded (all tiles)
            bool ok = true;
            int64_t lt = 0;
            for (int64_t t = (int64_t)blockIdx.x * NP + p; ok && t < ntiles; t += stride, ++lt) {
                const TileGeom g = tile_geom(t, ntq, T, a.We, a.H, a.Hkv, a.gp);
                auto load_k = [&](int bl) -> bool {
                    const int st = (int)(kc % KS);
                    const uint32_t use = kc / KS;
                    if (use > 0 && !wait(p, L::bKEmpty + st, (use - 1) & 1)) return false;
                    const int32_t krow = bl < g.npre ? 0 : g.kb0 + (g.b_first + bl - g.npre) * BN;
                    tc::mbar_arrive_expect_tx(bar(p, L::bKFull + st), L::kBlk);
                    for (int x = 0; x < D / 64; ++x)
                        tc::tma_load_3d(pb + L::pK + st * L::kBlk + x * (BN * 128), &tk, x * 64,
                                        krow, g.kvbh, bar(p, L::bKFull + st));
                    ++kc;
                    return true;
                };
                auto load_v = [&](int bl) -> bool {
                    const int st = (int)(vc % VS);
                    const uint32_t use = vc / VS;
                    if (use > 0 && !wait(p, L::bVEmpty + st, (use - 1) & 1)) return false;
                    const int32_t krow = bl < g.npre ? 0 : g.kb0 + (g.b_first + bl - g.npre) * BN;
                    tc::mbar_arrive_expect_tx(bar(p, L::bVFull + st), L::kBlk);
                    for (int x = 0; x < D / 64; ++x)
                        tc::tma_load_3d(pb + L::pV + st * L::kBlk + x * (BN * 128), &tv, x * 64,
                                        krow, g.kvbh, bar(p, L::bVFull + st));
                    ++vc;
                    return true;
                };
                constexpr bool kTmaDiag = DS > 0 && !LDW;
                int nd = 0;
                if constexpr (kTmaDiag) {
                    const int64_t last = (g.q0 + BM - 1 < T - 1) ? g.q0 + BM - 1 : T - 1;
                    for (int x = 0; x < a.n_off; ++x) nd += (a.offs[x] <= last) ? 1 : 0;
                    const int slot = (int)(lt & 1);
                    if (lt >= 2 && !wait(p, L::bInfoEmpty + slot, (uint32_t)(((lt >> 1) - 1) & 1)))
                        break;
                    info[slot] = nd;
                    tc::mbar_arrive(bar(p, L::bInfoFull + slot));
                }
                // Q of this tile once the previous tile's last S MMA and the
                // softmax warps are done with the buffer
                if (lt >= 1 && !wait(p, L::bQEmpty, (uint32_t)((lt - 1) & 1))) break;
                tc::mbar_arrive_expect_tx(bar(p, L::bQFull), L::kQTile);
                for (int x = 0; x < D / 64; ++x)
                    tc::tma_load_3d(pb + L::pQ + x * (BM * 128), &tq, x * 64, (int32_t)g.q0,
                                    (int32_t)g.bh, bar(p, L::bQFull));
                const int nblk = g.npre + g.n_band;
                int bl = 0;
                if constexpr (kTmaDiag) {
                    // the band blocks that fit the rings go before the distance blocks
                    const int n_pre = nblk < (KS < VS ? KS : VS) ? nblk : (KS < VS ? KS : VS);
                    for (; ok && bl < n_pre; ++bl) ok = load_k(bl) && load_v(bl);
                    // distance o: keys q0-o .. q0+127-o, one box per 64 columns;
                    // with K and V beyond L2 the block kPrefetchBlocks ahead is
                    // prefetched into L2 first
                    auto krow_of = [&](int d) { return (int32_t)(g.q0 - a.offs[a.n_off - nd + d]); };
                    auto prefetch_blk = [&](int d) {
                        for (int x = 0; x < D / 64; ++x) {
                            tc::tma_prefetch_3d(&tkd, x * 64, krow_of(d), g.kvbh);
                            tc::tma_prefetch_3d(&tvd, x * 64, krow_of(d), g.kvbh);
                        }
                    };
                    if (a.l2pf)
                        for (int d = 0; d < nd && d < kPrefetchBlocks; ++d) prefetch_blk(d);
                    for (int d = 0; ok && d < nd; ++d) {
                        const int st = (int)(dc % DS);
                        const uint32_t use = dc / DS;
                        if (use > 0 && !wait(p, L::bDiagEmpty + st, (use - 1) & 1)) {
                            ok = false;
                            break;
                        }
                        const uint32_t kdst = pb + L::pDK + st * L::kQTile;
                        const uint32_t vdst = pb + L::pDV + st * L::kQTile;
                        tc::mbar_arrive_expect_tx(bar(p, L::bDiagFull + st), 2 * L::kQTile);
                        for (int x = 0; x < D / 64; ++x) {
                            tc::tma_load_3d(kdst + x * (BM * 128), &tkd, x * 64, krow_of(d), g.kvbh,
                                            bar(p, L::bDiagFull + st));
                            tc::tma_load_3d(vdst + x * (BM * 128), &tvd, x * 64, krow_of(d), g.kvbh,
                                            bar(p, L::bDiagFull + st));
                        }
                        if (a.l2pf && d + kPrefetchBlocks < nd) prefetch_blk(d + kPrefetchBlocks);
                        ++dc;
                    }
                }
                for (; ok && bl < nblk; ++bl) ok = load_k(bl) && load_v(bl);
            }
        }
      } else if ((warp >> 1) < NP) {
        // ---------------- MMA issuer of pipeline p: S of block g, then P V of
        // block g-1
        const int p = warp >> 1;
        const uint32_t pb = sbase + (uint32_t)(p * L::kPipe);
        const uint32_t tp = tmem + p * L::tPipe;
        if (lane == 0) {
            const uint32_t idS = tc::idesc_bf16(BM, BN, false, false);
            const uint32_t idO = tc::idesc_bf16(BM, D, false, true);
            uint32_t kc = 0, gb = 0;  // K stages consumed, band blocks issued (all tiles)
            bool have_pv = false, pv_first = false, ok = true;
            uint32_t pv_gb = 0;
            int64_t pv_lt = 0;
            auto do_pv = [&]() -> bool {
                const int sb = (int)(pv_gb & 1), vst = (int)(pv_gb % VS);
                if (pv_first && !wait(p, L::bOInit, (uint32_t)(pv_lt & 1))) return false;
                if (!wait(p, L::bPFull + sb, (pv_gb >> 1) & 1)) return false;
                if (!wait(p, L::bVFull + vst, (pv_gb / VS) & 1)) return false;
                tc::tc_fence_after();
                // A = P (bf16) in TMEM over the first BN/2 columns of its S buffer
                const uint32_t pt = tp + L::tS0 + sb * BN;
                const uint32_t va = pb + L::pV + vst * L::kBlk;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    tc::mma_bf16_ts(tp + L::tO, pt + kk * 8,
                                    tc::sdesc_sw128(va + kk * 16 * 128, BN * 128, 1024), idO, 1u);
                tc::mma_commit(bar(p, L::bVEmpty + vst));
                tc::mma_commit(bar(p, L::bPVDone + sb));
                tc::mma_commit(bar(p, L::bSFree + sb));
                return true;
            };
            int64_t lt = 0;
            for (int64_t t = (int64_t)blockIdx.x * NP + p; ok && t < ntiles; t += stride, ++lt) {
                const TileGeom g = tile_geom(t, ntq, T, a.We, a.H, a.Hkv, a.gp);
                if (!wait(p, L::bQFull, (uint32_t)(lt & 1))) break;
                const uint32_t qa = pb + L::pQ;
                const int nblk = g.npre + g.n_band;
                for (int bl = 0; bl < nblk; ++bl) {
                    const int st = (int)(kc % KS), sb = (int)(gb & 1);
                    if (!wait(p, L::bKFull + st, (kc / KS) & 1) ||
                        (gb >= 2 && !wait(p, L::bSFree + sb, ((gb >> 1) - 1) & 1))) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t ka = pb + L::pK + st * L::kBlk;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t in = (kk & 3) * 32;
                        tc::mma_bf16_ss(tp + L::tS0 + sb * BN,
                                        tc::sdesc_sw128(qa + (kk >> 2) * (BM * 128) + in, 16, 1024),
                                        tc::sdesc_sw128(ka + (kk >> 2) * (BN * 128) + in, 16, 1024),
                                        idS, kk > 0);
                    }
                    tc::mma_commit(bar(p, L::bSFull + sb));
                    tc::mma_commit(bar(p, L::bKEmpty + st));
                    if (bl == nblk - 1) tc::mma_commit(bar(p, L::bQEmpty));
                    ++kc;
                    // the softmax of this block overlaps P V of the previous one
                    if (have_pv && !do_pv()) {
                        ok = false;
                        break;
                    }
                    have_pv = true;
                    pv_gb = gb;
                    pv_first = (bl == 0);
                    pv_lt = lt;
                    ++gb;
                }
                // the tile's last P V goes now: its epilogue waits for it
                if (ok && have_pv) {
                    ok = do_pv();
                    have_pv = false;
                }
            }
        }
      }
    } else {
        // ---------------- softmax warpgroup of pipeline p: thread r = query
        // row r = TMEM lane r
        if (NP == 2) tc::regs_inc<Regs<DS>::softmax>();
        const int p = (warp - 4) >> 2;
        const int r = tid - 128 - 128 * p;
        uint8_t *pm = sm + p * L::kPipe;
        const uint32_t lane_off = (uint32_t)(((warp - 4) & 3) * 32) << 16;
        const uint32_t tS = tmem + p * L::tPipe + lane_off + L::tS0;
        const uint32_t tO = tmem + p * L::tPipe + lane_off + L::tO;
        const float c2 = a.scale2;
        const int wq = r >> 5;    // warp within the group: rows 32 wq .. 32 wq + 31
        volatile int *info = (volatile int *)(sm + L::kMisc + 8) + 2 * p;
        uint32_t gb = 0, dc = 0;  // band and TMA distance blocks consumed (all tiles)
        bool ok = true;
        int64_t lt = 0;
        for (int64_t t = (int64_t)blockIdx.x * NP + p; ok && t < ntiles; t += stride, ++lt) {
            const TileGeom g = tile_geom(t, ntq, T, a.We, a.H, a.Hkv, a.gp);
            const int32_t q0 = g.q0, bh = g.bh;
            const int32_t i = q0 + r;
            float m_run = -INFINITY, l_run = 0.f;

            // --- diagonal blocks: q row from the Q tile, one key/value row per
            // slot; bf16 x bf16 -> fp32 FMAs (exact products), p rounded to
            // bf16 for the weighted sum as the band path's P is; running max
            // rescaled lazily (only when it grows by more than 2^8)
            {
                float acc[D];
#pragma unroll
                for (int x = 0; x < D; ++x) acc[x] = 0.f;
                if constexpr (DS > 0) {
                    // slots: the tile's distance blocks (count from the
                    // producer), or, for CSR lists, the longest residual list
                    // of this warp's rows
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
                        if (i < T) {
                            // the shared prefix keys outside the window are the
                            // first entries of the sorted list: the prefix block
                            // takes them
                            int32_t gc = i - W + 1 < a.gp ? i - W + 1 : a.gp;
                            gc = gc > 0 ? gc : 0;
                            cst = a.rowptr[i] + gc;
                            resid = (int32_t)(a.rowptr[i + 1] - cst - ((i + 1 < W) ? i + 1 : W));
                        }
                        nd = (int)__reduce_max_sync(0xffffffffu, (unsigned)resid);
                    }
                    const int dfirst = a.n_off - nd;  // distance index of slot 0 (keys ascending)
                    // key of this thread's row in slot d, -1 if the row has none
                    auto key_of = [&](int d) -> int32_t {  // (CSR slots)
                        return d < resid ? __ldg(a.colidx + cst + d) : -1;
                    };
                    const size_t slice = (size_t)g.kvbh * (size_t)T * DG;
                    uint32_t qw[D / 2];
                    // one slot: dot product with the row's key, online-softmax
                    // update, p-weighted value row into acc (Q is read on the
                    // first slot, once its load has landed)
                    auto body = [&](int d, int st) {
                        if (d == 0) {
                            ok = __all_sync(0xffffffffu, wait(p, L::bQFull, (uint32_t)(lt & 1)));
                            if (ok) {
#pragma unroll
                                for (int c = 0; c < DG / 8; ++c) {
                                    const uint4 w4 = *(const uint4 *)(pm + L::pQ +
                                                                      (c >> 3) * (BM * 128) +
                                                                      tc::sw128_off(r, c & 7));
                                    qw[4 * c] = w4.x;
                                    qw[4 * c + 1] = w4.y;
                                    qw[4 * c + 2] = w4.z;
                                    qw[4 * c + 3] = w4.w;
                                }
                            }
                        }
                        const bool valid = LDW ? (d < resid) : (i < T && i >= a.offs[dfirst + d]);
                        if (!ok || !valid) return;
                        const uint8_t *kr = pm + L::pDK + st * L::kQTile;
                        const uint8_t *vr = pm + L::pDV + st * L::kQTile;
                        // eight independent partial sums (short dependency chains)
                        float sp[8];
#pragma unroll
                        for (int x = 0; x < 8; ++x) sp[x] = 0.f;
#pragma unroll
                        for (int c = 0; c < DG / 8; ++c) {
                            const uint4 w4 = *(const uint4 *)(kr + (c >> 3) * (BM * 128) +
                                                              tc::sw128_off(r, c & 7));
                            const uint32_t kw[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                sp[2 * e] = tc::fma_bf_lo(qw[4 * c + e], kw[e], sp[2 * e]);
                                sp[2 * e + 1] = tc::fma_bf_hi(qw[4 * c + e], kw[e], sp[2 * e + 1]);
                            }
                        }
                        const float s = (((sp[0] + sp[1]) + (sp[2] + sp[3])) +
                                         ((sp[4] + sp[5]) + (sp[6] + sp[7]))) *
                                        c2;
                        if (s > m_run + kRescaleThreshold) {
                            const float al = tc::ex2(m_run - s);  // 0 on the first edge
#pragma unroll
                            for (int x = 0; x < D; ++x) acc[x] *= al;
                            l_run *= al;
                            m_run = s;
                        }
                        const float pr = tc::ex2(s - m_run);
                        l_run += pr;
                        const uint32_t p2 = tc::pack_bf16x2(pr, pr);
#pragma unroll
                        for (int c = 0; c < DG / 8; ++c) {
                            const uint4 w4 = *(const uint4 *)(vr + (c >> 3) * (BM * 128) +
                                                              tc::sw128_off(r, c & 7));
                            const uint32_t vw[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                acc[8 * c + 2 * e] = tc::fma_bf_lo(p2, vw[e], acc[8 * c + 2 * e]);
                                acc[8 * c + 2 * e + 1] =
                                    tc::fma_bf_hi(p2, vw[e], acc[8 * c + 2 * e + 1]);
                            }
                        }
                    };
                    if constexpr (LDW) {
                        rows::warp_slots<DG, DS>(
                            nd, sbase + (uint32_t)(p * L::kPipe + L::pDK),
                            sbase + (uint32_t)(p * L::kPipe + L::pDV), (uint32_t)L::kQTile, a.k,
                            a.v, a.l2pf > 0, lane, wq, [&](int) { return slice; }, key_of, body);
                    } else {
                        for (int d = 0; ok && d < nd; ++d) {
                            const int st = (int)(dc % DS);
                            if (!__all_sync(0xffffffffu,
                                            wait(p, L::bDiagFull + st, (dc / DS) & 1))) {
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
                // this warp is done reading Q of the tile
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar(p, L::bQEmpty));
                // initialise O (columns tO .. tO+D) with the diagonal part
#pragma unroll
                for (int c = 0; c < D; c += 32) {
                    uint32_t w[32];
#pragma unroll
                    for (int x = 0; x < 32; ++x) w[x] = __float_as_uint(acc[c + x]);
                    tc::tmem_st32(tO + c, w);
                }
                tc::tmem_st_wait();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar(p, L::bOInit));
            }

            // --- band blocks
            uint32_t gb_last = gb;
            const int nblk = g.npre + g.n_band;
            for (int bl = 0; ok && bl < nblk; ++bl, ++gb) {
                const int sb = (int)(gb & 1);
                const int32_t b = g.b_first + bl - g.npre;
                gb_last = gb;
                if (!wait(p, L::bSFull + sb, (gb >> 1) & 1)) {
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                // mask: r <= u <= r+W-1 and key >= 0, with u = BN b + c, i.e.
                // the column range [c_lo, c_hi] of this block.  Scores stay raw
                // (the scale is folded into the exponent's FFMA); a masked raw
                // score is set to the extreme that the max/min below ignores.
                // block coordinates u = BN b + c from key q0 - We + 1: row r
                // keeps its window u in [r + We - W, r + We - 1], the folded
                // links u = r + We - 1 - o, and keys >= 0 (u >= We - 1 - q0)
                const int32_t We = a.We;
                const int32_t u0 = b * BN;
                const bool pre = bl < g.npre;
                const bool need_mask = pre || a.nf > 0 || (u0 < BM - 1) ||
                                       (u0 + BN - 1 > We - 1) || (u0 + q0 < We - 1);
                uint64_t keep = ~0ull;  // bit c: this row keeps column c of the block
                if (pre) {
                    // shared prefix: keys 0 .. min(gp, i - W + 1) - 1
                    const int32_t n = i - W + 1 < a.gp ? i - W + 1 : a.gp;
                    keep = tc::bits_range(0, n - 1);
                } else if (need_mask) {
                    const int32_t kmin = We - 1 - q0;  // u of key 0
                    const int32_t lo = (r + We - W > kmin) ? r + We - W : kmin;
                    const int32_t hi = r + We - 1;
                    const int c_lo = lo - u0 < 0 ? 0 : (lo - u0 > BN ? BN : lo - u0);
                    const int c_hi = hi - u0 > BN - 1 ? BN - 1 : (hi - u0 < -1 ? -1 : hi - u0);
                    keep = tc::bits_range(c_lo, c_hi);
                    if (a.nf > 0) {
#pragma unroll
                        for (int x = 0; x < kMaxFold; ++x) {
                            const int32_t u = r + We - 1 - a.fold[x];
                            if (x < a.nf && u >= kmin && u >= u0 && u < u0 + BN)
                                keep |= 1ull << (u - u0);
                        }
                    }
                }
                if (need_mask && __all_sync(0xffffffffu, keep == 0ull)) {
                    // no row of this warp keeps a key of the block: P = 0
                    uint32_t z[BN / 2];
#pragma unroll
                    for (int x = 0; x < BN / 2; ++x) z[x] = 0u;
                    tc::tmem_st_n<BN / 2>(tS + sb * BN, z);
                    tc::tmem_st_wait();
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar(p, L::bPFull + sb));
                    continue;
                }
                float s[BN];
#pragma unroll
                for (int c = 0; c < BN; c += 32)
                    tc::tmem_ld32(tS + sb * BN + c, (uint32_t *)(s + c));
                tc::tmem_ld_wait();
                const bool pos = c2 >= 0.f;
                const float ext = pos ? -INFINITY : INFINITY;
                // 16-column chunks holding a kept key of some row of this warp;
                // the others get no masking, max or exponentials (P = 0 there)
                uint32_t live = (1u << (BN / 16)) - 1u;
                if (need_mask) {
                    live = 0u;
#pragma unroll
                    for (int c16 = 0; c16 < BN / 16; ++c16)
                        if (__any_sync(0xffffffffu, ((keep >> (16 * c16)) & 0xffffull) != 0ull))
                            live |= 1u << c16;
#pragma unroll
                    for (int c16 = 0; c16 < BN / 16; ++c16) {
                        if ((live >> c16) & 1u) {
#pragma unroll
                            for (int c = 16 * c16; c < 16 * c16 + 16; ++c)
                                s[c] = ((keep >> c) & 1ull) ? s[c] : ext;
                        }
                    }
                }
                float mr[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) mr[x] = ext;
#pragma unroll
                for (int c16 = 0; c16 < BN / 16; ++c16) {
                    if ((live >> c16) & 1u) {
                        if (pos) {
#pragma unroll
                            for (int c = 16 * c16; c < 16 * c16 + 16; ++c)
                                mr[c & 7] = fmaxf(mr[c & 7], s[c]);
                        } else {
#pragma unroll
                            for (int c = 16 * c16; c < 16 * c16 + 16; ++c)
                                mr[c & 7] = fminf(mr[c & 7], s[c]);
                        }
                    }
                }
                if (pos) {
#pragma unroll
                    for (int x = 4; x > 0; x >>= 1)
                        for (int y = 0; y < x; ++y) mr[y] = fmaxf(mr[y], mr[y + x]);
                } else {
#pragma unroll
                    for (int x = 4; x > 0; x >>= 1)
                        for (int y = 0; y < x; ++y) mr[y] = fminf(mr[y], mr[y + x]);
                }
                const float mblk = (mr[0] == ext) ? -INFINITY : mr[0] * c2;
                // conditional rescale of O (and l) when the max grows by more than 2^8
                const bool grow = mblk > m_run + kRescaleThreshold;
                if (__any_sync(0xffffffffu, grow)) {
                    const float m_new = grow ? mblk : m_run;
                    const float alpha = grow ? tc::ex2(m_run - m_new) : 1.f;
                    if (bl > 0) {  // O must hold P V of the previous block of this tile
                        const uint32_t pg = gb - 1;
                        if (!wait(p, L::bPVDone + (int)(pg & 1), (pg >> 1) & 1)) {
                            ok = false;
                            break;
                        }
                        tc::tc_fence_after();
                    }
#pragma unroll
                    for (int c = 0; c < D; c += 32) {
                        uint32_t w[32];
                        tc::tmem_ld32(tO + c, w);
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int x = 0; x < 32; ++x)
                            w[x] = __float_as_uint(__uint_as_float(w[x]) * alpha);
                        tc::tmem_st32(tO + c, w);
                    }
                    l_run *= alpha;
                    m_run = m_new;
                }
                // p = 2^(s - m), row sum, bf16 P over the first BN/2 columns of
                // this S buffer (its scores are already in registers)
                const float m_use = (m_run == -INFINITY) ? 0.f : m_run;  // all-masked row: p = 0
                float ls[4] = {0.f, 0.f, 0.f, 0.f};
                uint32_t pw[BN / 2];
                if (need_mask) {
                    // a masked score is the extreme whose scaled value is -inf
                    // (the scale is nonzero on this path), so its p is 0
#pragma unroll
                    for (int c16 = 0; c16 < BN / 16; ++c16) {
                        if ((live >> c16) & 1u) {
#pragma unroll
                            for (int c = 8 * c16; c < 8 * c16 + 8; ++c) {
                                const float p0 = tc::ex2(fmaf(s[2 * c], c2, -m_use));
                                const float p1 = tc::ex2(fmaf(s[2 * c + 1], c2, -m_use));
                                ls[c & 3] += p0 + p1;
                                pw[c] = tc::pack_bf16x2(p0, p1);
                            }
                        } else {
#pragma unroll
                            for (int c = 8 * c16; c < 8 * c16 + 8; ++c) pw[c] = 0u;
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < BN / 2; ++c) {
                        const float p0 = tc::ex2(fmaf(s[2 * c], c2, -m_use));
                        const float p1 = tc::ex2(fmaf(s[2 * c + 1], c2, -m_use));
                        ls[c & 3] += p0 + p1;
                        pw[c] = tc::pack_bf16x2(p0, p1);
                    }
                }
                l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
#pragma unroll
                for (int c = 0; c < BN / 2; c += 32) tc::tmem_st32(tS + sb * BN + c, pw + c);
                tc::tmem_st_wait();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar(p, L::bPFull + sb));
            }
            if (!ok) break;

            // --- epilogue: O / l and lse once the tile's last P V is done
            if (!wait(p, L::bPVDone + (int)(gb_last & 1), (gb_last >> 1) & 1)) break;
            tc::tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            if constexpr (DG % 64 == 0) {
                // the warp's 32 rows in whole sectors, staged in O's first
                // columns (O is read out first)
                uint32_t pk[DG / 2];
#pragma unroll
                for (int c = 0; c < DG; c += 32) {
                    uint32_t w[32];
                    tc::tmem_ld32(tO + c, w);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int x = 0; x < 32; x += 2)
                        pk[(c + x) / 2] = tc::pack_bf16x2(__uint_as_float(w[x]) * inv,
                                                          __uint_as_float(w[x + 1]) * inv);
                }
                const int64_t row0 = (int64_t)q0 + 32 * wq;
                const int64_t nr = T - row0;
                tc::tmem_rows_store<DG / 2>(tO, pk, a.out + ((size_t)bh * (size_t)T + row0) * DG, DG,
                                            nr < 0 ? 0 : (nr > 32 ? 32 : (int)nr), lane);
            } else {
                __nv_bfloat16 *orow = a.out + ((size_t)bh * (size_t)T + (size_t)i) * DG;
    #pragma unroll
                for (int c = 0; c < DG; c += 32) {
                    uint32_t w[32];
                    tc::tmem_ld32(tO + c, w);
                    tc::tmem_ld_wait();
                    if (i < T) {
    #pragma unroll
                        for (int x = 0; x < 32; x += 8) {
                            uint4 o4;
                            o4.x = tc::pack_bf16x2(__uint_as_float(w[x]) * inv,
                                                   __uint_as_float(w[x + 1]) * inv);
                            o4.y = tc::pack_bf16x2(__uint_as_float(w[x + 2]) * inv,
                                                   __uint_as_float(w[x + 3]) * inv);
                            o4.z = tc::pack_bf16x2(__uint_as_float(w[x + 4]) * inv,
                                                   __uint_as_float(w[x + 5]) * inv);
                            o4.w = tc::pack_bf16x2(__uint_as_float(w[x + 6]) * inv,
                                                   __uint_as_float(w[x + 7]) * inv);
                            *(uint4 *)(orow + c + x) = o4;
                        }
                    }
                }
            }
            if (i < T)
                a.lse[(size_t)bh * (size_t)T + (size_t)i] =
                    l_run > 0.f ? (m_run + tc::lg2(l_run)) * kLn2 : -INFINITY;
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, L::kTmemCols);
    }
}

template <int D, int NP, int KS, int VS, int DS, bool LDW, int DG>
sa_status launch_band_fwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                          const sa_graph_s *g, float scale, sa_tensor *out, float *lse,
                          cudaStream_t s) {
    using L = Layout<D, NP, KS, VS, DS>;
    static_assert(L::kAlloc <= 232448, "shared memory budget");
    constexpr int kThreads = 128 + 128 * NP;
    static_assert(DG == D || (D == 64 && DG == 32), "row length");
    auto kern = band_fwd_kernel<D, NP, KS, VS, DS, LDW, DG>;
    if (NP == 2) {
        // setmaxnreg.inc waits until the CTA's pool holds the registers it
        // asks for: the launch must provide the whole split
        static int regs_ok = -1;
        if (regs_ok < 0) {
            cudaFuncAttributes fa;
            SA_CUDA_TRY(cudaFuncGetAttributes(&fa, (const void *)kern));
            regs_ok = fa.numRegs * kThreads >= 128 * Regs<DS>::producer + 128 * NP * Regs<DS>::softmax;
        }
        if (!regs_ok) {
            sa_record_cuda_error(cudaErrorInvalidConfiguration,
                                 "band_fwd: launch registers below the warpgroup split");
            return SA_ERR_CUDA;
        }
    }
    const int64_t BH = q->B * q->H, BHkv = k->B * k->H, T = q->T;
    CUtensorMap mq, mk, mv, mkd, mvd;  // 64-row band boxes, 128-row distance blocks
    if (!sa_tmap_bf16_3d(&mq, q->ptr, DG, T, BH, BM) ||
        !sa_tmap_bf16_3d(&mk, k->ptr, DG, T, BHkv, BN) ||
        !sa_tmap_bf16_3d(&mv, v->ptr, DG, T, BHkv, BN) ||
        !sa_tmap_bf16_3d(&mkd, k->ptr, DG, T, BHkv, BM) ||
        !sa_tmap_bf16_3d(&mvd, v->ptr, DG, T, BHkv, BM)) {
        sa_record_cuda_error(cudaErrorInvalidValue, "band_fwd: tensor map encoding");
        return SA_ERR_CUDA;
    }
    FwdArgs a{};
    a.T = T;
    a.BH = BH;
    a.H = q->H;
    a.Hkv = k->H;
    a.W = g->W;
    a.kind = g->kind;
    a.gp = g->kind == 1 ? g->gprefix : 0;
    a.We = sa_fold_links(g, BN, kMaxFold, a.fold, &a.nf, a.offs, &a.n_off);
    a.l2pf = (double)BHkv * (double)T * DG * 2 * 2 > kL2ResidentBytes ? 1 : 0;
    a.rowptr = g->rowptr;
    a.colidx = g->colidx;
    a.k = (const __nv_bfloat16 *)k->ptr;
    a.v = (const __nv_bfloat16 *)v->ptr;
    a.out = (__nv_bfloat16 *)out->ptr;
    a.lse = lse;
    a.scale2 = scale * kLog2e;
    a.err = sa_device_error_word();
    if (!a.err) return SA_ERR_CUDA;
    SA_CUDA_TRY(sa_smem_optin((const void *)kern, L::kAlloc));
    // persistent: one CTA per SM, NP tiles in flight in each
    const int64_t ntiles = ((T + BM - 1) / BM) * BH;
    const int64_t nctas = (ntiles + NP - 1) / NP;
    int sms = 0;
    SA_CUDA_TRY(sa_sm_count(&sms));
    const unsigned grid = (unsigned)(nctas < sms ? nctas : sms);
    SA_LAUNCH("band_fwd", s,
              kern<<<grid, kThreads, L::kAlloc, s>>>(mq, mk, mv, mkd, mvd, a));
    SA_CUDA_TRY(cudaGetLastError());
    return SA_OK;
}

}  // namespace

bool sa_band_fwd_supported(const sa_tensor *q, const sa_graph_s *g) {
    if (q->dtype != SA_BF16 || (q->D != 32 && q->D != 64 && q->D != 128)) return false;
    if (g->W < 1) return false;                       // no band: gather path
    // 32-bit tile coordinates (TMA takes int32 row and slice indices)
    if (q->B * q->H >= ((int64_t)1 << 31) || q->T >= ((int64_t)1 << 31)) return false;
    if (g->kind == 1 && !g->rowptr) return false;
    return true;
}

namespace {

// Links of at least kLongSpan rows, all multiples of kLongSpan, can go to a
// second pass (attn_links.cu): in sequence order their rows are old in L2 by
// the time a link reads them (the sweep reads ~6 KB of K/V per row of
// progress, so rows 2^13 back are ~50 MB old, 2^15 back ~200 MB), while the
// second pass runs the tiles in an order that keeps them there.  The second
// pass re-reads q, out and lse, so it pays only on long sequences.  Measured
// on B200 with window 32 and links 2^k: at T = 2^27 the split at 2^13 took
// 84.7-86.2 ms, at 2^10 89.0, 2^11 85.8, 2^12 85.5, 2^14 88.1, 2^15 89.4-90.1,
// 2^16 95.6; with the split at 2^13 two passes beat one from T = 2^23 (K and
// V 2 GiB: 4.36 vs 4.60 ms; 2^24 8.99 vs 10.22; 2^25 18.3 vs 22.7; 2^26 39.7
// vs 50.4) and lose at 2^22 (2.16 vs 2.06) and below.  What counts is the
// length of one slice's sweep, not the job's size: with 4 slices of 2^22 two
// passes won (8.56 vs 8.98 ms), with 16 slices of 2^20 (7.77 vs 8.23 ms one
// pass) and 64 of 2^17 (3.18 vs 3.72) one pass did.
constexpr int64_t kLongSpan = (int64_t)1 << 13;
constexpr int kMinLong = 3;
constexpr double kTwoPassSlice = 1.0 * 1024 * 1024 * 1024;  // K and V of one slice
constexpr double kTwoPassBytes = 2.0 * 1024 * 1024 * 1024;  // K and V together

int long_links(const sa_tensor *k, const sa_graph_s *g) {
    const int mode = sa_link_pass_mode();
    if (g->kind != 0 || mode == SA_LINKS_ONE_PASS) return 0;
    int n = 0;
    while (n < g->n_off && g->offs[n] >= kLongSpan) {  // descending
        if (g->offs[n] % kLongSpan != 0) return 0;
        ++n;
    }
    if (mode == SA_LINKS_SPLIT) return n;
    const double slice = (double)k->T * k->D * 2 * 2;  // bf16 K and V rows of one slice
    const double kv = slice * (double)k->B * (double)k->H;
    return (slice >= kTwoPassSlice && kv >= kTwoPassBytes && n >= kMinLong) ? n : 0;
}

sa_status band_fwd_dispatch(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                            const sa_graph_s *g, float scale, sa_tensor *out, float *lse,
                            cudaStream_t s);

}  // namespace

sa_status sa_band_fwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                      const sa_graph_s *g_in, const GraphView &, float scale, sa_tensor *out,
                      float *lse, cudaStream_t s) {
    // the first pass takes the window and the links shorter than kLongSpan
    const int n_long = long_links(k, g_in);
    sa_graph_s g_short;
    const sa_graph_s *g = g_in;
    if (n_long > 0) {
        g_short = *g_in;
        g_short.n_off = g_in->n_off - n_long;
        for (int x = 0; x < SA_MAX_OFFSETS; ++x)
            g_short.offs[x] = x < g_short.n_off ? g_in->offs[x + n_long] : 0;
        g = &g_short;
    }
    const sa_status st = band_fwd_dispatch(q, k, v, g, scale, out, lse, s);
    if (st != SA_OK || n_long == 0) return st;
    return sa_link_pass(q, k, v, g_in->offs, n_long, kLongSpan, scale, out, lse, s);
}

namespace {

sa_status band_fwd_dispatch(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                            const sa_graph_s *g, float scale, sa_tensor *out, float *lse,
                            cudaStream_t s) {
    const bool diag = (g->kind == 0) ? g->n_off > 0 : g->max_resid > 0;
    const bool csr = g->kind == 1;
    // <D, pipelines, K stages, V stages, diagonal stages, per-warp slots>,
    // sized to the 227 KB of shared memory
    // (D = 32 runs on the D = 64 tiles, its rows zero-extended)
    if (q->D == 32) {
        if (!diag) return launch_band_fwd<64, 2, 4, 4, 0, false, 32>(q, k, v, g, scale, out, lse, s);
        return csr ? launch_band_fwd<64, 2, 2, 2, 2, true, 32>(q, k, v, g, scale, out, lse, s)
                   : launch_band_fwd<64, 2, 2, 2, 2, false, 32>(q, k, v, g, scale, out, lse, s);
    }
    if (q->D == 64) {
        if (!diag) return launch_band_fwd<64, 2, 4, 4, 0, false, 64>(q, k, v, g, scale, out, lse, s);
        return csr ? launch_band_fwd<64, 2, 2, 2, 2, true, 64>(q, k, v, g, scale, out, lse, s)
                   : launch_band_fwd<64, 2, 2, 2, 2, false, 64>(q, k, v, g, scale, out, lse, s);
    }
    if (!diag) return launch_band_fwd<128, 2, 3, 2, 0, false, 128>(q, k, v, g, scale, out, lse, s);
    return csr ? launch_band_fwd<128, 1, 2, 2, 2, true, 128>(q, k, v, g, scale, out, lse, s)
               : launch_band_fwd<128, 1, 2, 2, 2, false, 128>(q, k, v, g, scale, out, lse, s);
}

}  // namespace
