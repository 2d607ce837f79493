// attn_band.cu -- forward on tcgen05 band tiles fused with the gathered edges.
//
// One CTA owns 128 consecutive queries [q0, q0+128) of one (b, h) slice.
//  * Window edges (the band of "MiniGPT (Part 6)", section "A mask is not
//    enough": keys j <= i with i - j < W) run as dense 128 x 128 tiles on the
//    tensor cores: keys [q0-W+1, q0+127] are cut into blocks of 128 starting
//    at q0-W+1, so in block coordinates u = 128 b + c a query row r keeps
//    exactly r <= u <= r+W-1 (and j >= 0).  S = Q K^T lands in TMEM, the
//    softmax warpgroup turns it into P (bf16, shared memory), and O += P V
//    accumulates in TMEM.
//  * Every other edge -- the 2^k distance links of "SpatialLM-Mini ...",
//    section "How tokens choose whom to listen to", or the non-window part of
//    a CSR list ("Longer Attention Span ...", Abstract) -- is a "diagonal"
//    block: 128 key rows, row r belonging to query r.  For a distance o the
//    rows are the contiguous keys q0-o .. q0+127-o (one TMA box); for CSR
//    lists slot s of every row is gathered with 16-byte cp.async into the
//    same swizzled layout.  Thread r takes the dot product of its own row.
//  * One online softmax (running max m and sum l per row, base 2) covers both
//    classes: the diagonal blocks go first, their weighted sum initialises O
//    in TMEM, then the band blocks rescale O only when a row's max grows by
//    more than 2^8 (the stale max keeps every p <= 256, exact in fp32).
//  * Epilogue: out = O / l (bf16, round to nearest even), lse = (m + log2 l) ln 2.
//
// Warp roles (256 threads): 0 TMA producer for Q and the band K/V ring,
// 1 TMEM allocator + MMA issuer, 2-3 producers of the diagonal blocks,
// 4-7 softmax warpgroup (thread = query row = TMEM lane).
// Every mbarrier wait is bounded (2 s); on expiry the CTA records
// SA_DEVERR_TIMEOUT in the device error word, all roles leave their loops,
// TMEM is freed and the kernel returns.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sa_band.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace {

constexpr int BM = 128;             // queries per CTA
constexpr int BN = 128;             // keys per band block
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct FwdArgs {
    int64_t T;
    int32_t W;          // band width (structured window or verified CSR band)
    int32_t kind;       // 0 structured, 1 CSR
    int32_t n_off;
    int64_t offs[SA_MAX_OFFSETS];  // distances (structured), descending
    const int64_t *rowptr;         // CSR
    const int32_t *colidx;
    const __nv_bfloat16 *k;        // CSR gathers read K/V directly
    const __nv_bfloat16 *v;
    __nv_bfloat16 *out;
    float *lse;
    float scale2;                  // scale * log2(e)
    int *err;
};

template <int D, int KS, int VS, int DS, int PB>
struct Layout {
    static constexpr int kTile = BM * D * 2;            // 128 rows x D bf16
    static constexpr int kQ = 0;
    static constexpr int kBandK = kQ + kTile;
    static constexpr int kBandV = kBandK + KS * kTile;
    static constexpr int kP = kBandV + VS * kTile;
    static constexpr int kPTile = BM * BN * 2;
    static constexpr int kDiagK = kP + PB * kPTile;
    static constexpr int kDiagV = kDiagK + DS * kTile;
    static constexpr int kBars = kDiagV + DS * kTile;
    // barriers
    static constexpr int bQFull = 0;
    static constexpr int bKFull = 1;
    static constexpr int bKEmpty = bKFull + KS;
    static constexpr int bVFull = bKEmpty + KS;
    static constexpr int bVEmpty = bVFull + VS;
    static constexpr int bSFull = bVEmpty + VS;
    static constexpr int bSFree = bSFull + 2;
    static constexpr int bPFull = bSFree + 2;
    static constexpr int bPVDone = bPFull + PB;
    static constexpr int bOInit = bPVDone + PB;
    static constexpr int bDiagFull = bOInit + 1;
    static constexpr int bDiagEmpty = bDiagFull + (DS > 0 ? DS : 1);
    static constexpr int nBars = bDiagEmpty + (DS > 0 ? DS : 1);
    static constexpr int kMisc = kBars + nBars * 8;      // tmem slot, abort, n_diag
    static constexpr int kTotal = kMisc + 16;
    static constexpr int kAlloc = kTotal + 1024;         // alignment slack
    // TMEM columns: S buffers [0,128) and [128,256), O at 256
    static constexpr uint32_t tS0 = 0, tO = 256;
    static constexpr uint32_t kTmemCols = 512;
};

__device__ __forceinline__ int64_t band_first_block(int64_t q0, int32_t W) {
    // first block holding a key >= 0: u >= W-1-q0
    int64_t need = (int64_t)W - 1 - q0;
    return need > 0 ? need / BN : 0;
}

template <int D, int KS, int VS, int DS, int PB>
__global__ void __launch_bounds__(256, 1)
band_fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tkr,
                const __grid_constant__ CUtensorMap tvr, const FwdArgs a) {
    using L = Layout<D, KS, VS, DS, PB>;
    constexpr int DSX = DS > 0 ? DS : 1;  // ring modulus (no diagonal ring when DS == 0)
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = tc::smem_u32(sm);
    uint64_t *bars = (uint64_t *)(sm + L::kBars);
    uint32_t *tmem_slot = (uint32_t *)(sm + L::kMisc);
    volatile int *abort = (volatile int *)(sm + L::kMisc + 4);
    int *n_diag_s = (int *)(sm + L::kMisc + 8);
    auto bar = [&](int b) { return sbase + L::kBars + 8u * (uint32_t)b; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t tile = blockIdx.x, bh = blockIdx.y;
    const int64_t q0 = tile * BM;
    const int64_t T = a.T;
    const int32_t W = a.W;
    const int64_t kb0 = q0 - W + 1;                              // key of u = 0
    const int64_t last_key = (q0 + BM - 1 < T - 1) ? q0 + BM - 1 : T - 1;
    const int64_t nblk = (last_key - kb0) / BN + 1;              // blocks up to the last key
    const int64_t b_first = band_first_block(q0, W);
    const int n_band = (int)(nblk - b_first);

    if (tid == 0) {
        tc::mbar_init(bar(L::bQFull), 1);
        for (int s = 0; s < KS; ++s) {
            tc::mbar_init(bar(L::bKFull + s), 1);
            tc::mbar_init(bar(L::bKEmpty + s), 1);
        }
        for (int s = 0; s < VS; ++s) {
            tc::mbar_init(bar(L::bVFull + s), 1);
            tc::mbar_init(bar(L::bVEmpty + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(bar(L::bSFull + s), 1);
            tc::mbar_init(bar(L::bSFree + s), 4);
        }
        for (int s = 0; s < PB; ++s) {
            tc::mbar_init(bar(L::bPFull + s), 4);
            tc::mbar_init(bar(L::bPVDone + s), 1);
        }
        tc::mbar_init(bar(L::bOInit), 4);
        for (int s = 0; s < DS; ++s) {
            tc::mbar_init(bar(L::bDiagFull + s), 1);
            tc::mbar_init(bar(L::bDiagEmpty + s), 4);
        }
        *abort = 0;
        *n_diag_s = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) tc::tmem_alloc(tc::smem_u32(tmem_slot), L::kTmemCols);
    __syncthreads();

    // number of diagonal blocks of this tile
    if (warp >= 4) {
        int nd = 0;
        const int64_t i = q0 + (tid - 128);
        if (a.kind == 0) {
            const int64_t last = (q0 + BM - 1 < T - 1) ? q0 + BM - 1 : T - 1;
            for (int x = 0; x < a.n_off; ++x) nd += (a.offs[x] <= last) ? 1 : 0;
        } else if (i < T) {
            const int64_t deg = a.rowptr[i + 1] - a.rowptr[i];
            const int64_t inband = (i + 1 < W) ? i + 1 : W;
            nd = (int)(deg - inband);
        }
        atomicMax(n_diag_s, nd);
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_diag = (DS > 0) ? *n_diag_s : 0;

    if (warp == 0) {
        // ---------------- TMA producer: Q, then the band K/V ring
        if (lane == 0) {
            tc::tma_prefetch_desc(&tq);
            tc::tma_prefetch_desc(&tk);
            tc::tma_prefetch_desc(&tv);
            tc::mbar_arrive_expect_tx(bar(L::bQFull), L::kTile);
            for (int x = 0; x < D / 64; ++x)
                tc::tma_load_3d(sbase + L::kQ + x * (BM * 128), &tq, x * 64, (int32_t)q0,
                                (int32_t)bh, bar(L::bQFull));
            // K runs one block ahead of V: K(b) is released as soon as S(b) is
            // done, V(b) only after P(b) V(b)
            auto load_k = [&](int bl) -> bool {
                const int st = bl % KS, use = bl / KS;
                if (use > 0 && !tc::mbar_wait(bar(L::bKEmpty + st), (use - 1) & 1, abort, a.err,
                                              SA_DEVERR_TIMEOUT))
                    return false;
                const int32_t krow = (int32_t)(kb0 + (b_first + bl) * BN);
                tc::mbar_arrive_expect_tx(bar(L::bKFull + st), L::kTile);
                for (int x = 0; x < D / 64; ++x)
                    tc::tma_load_3d(sbase + L::kBandK + st * L::kTile + x * (BN * 128), &tk,
                                    x * 64, krow, (int32_t)bh, bar(L::bKFull + st));
                return true;
            };
            auto load_v = [&](int bl) -> bool {
                const int st = bl % VS, use = bl / VS;
                if (use > 0 && !tc::mbar_wait(bar(L::bVEmpty + st), (use - 1) & 1, abort, a.err,
                                              SA_DEVERR_TIMEOUT))
                    return false;
                const int32_t krow = (int32_t)(kb0 + (b_first + bl) * BN);
                tc::mbar_arrive_expect_tx(bar(L::bVFull + st), L::kTile);
                for (int x = 0; x < D / 64; ++x)
                    tc::tma_load_3d(sbase + L::kBandV + st * L::kTile + x * (BN * 128), &tv,
                                    x * 64, krow, (int32_t)bh, bar(L::bVFull + st));
                return true;
            };
            bool ok = n_band > 0 ? load_k(0) : true;
            for (int bl = 0; ok && bl < n_band; ++bl) {
                if (bl + 1 < n_band && !load_k(bl + 1)) break;
                if (!load_v(bl)) break;
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            const uint32_t idS = tc::idesc_bf16(BM, BN, false, false);
            const uint32_t idO = tc::idesc_bf16(BM, D, false, true);
            bool ok = tc::mbar_wait(bar(L::bQFull), 0, abort, a.err, SA_DEVERR_TIMEOUT);
            auto issue_S = [&](int bl) -> bool {
                const int st = bl % KS, sb = bl & 1;
                if (!tc::mbar_wait(bar(L::bKFull + st), (bl / KS) & 1, abort, a.err,
                                   SA_DEVERR_TIMEOUT))
                    return false;
                if (bl >= 2 && !tc::mbar_wait(bar(L::bSFree + sb), ((bl >> 1) - 1) & 1, abort,
                                              a.err, SA_DEVERR_TIMEOUT))
                    return false;
                tc::tc_fence_after();
                const uint32_t qa = sbase + L::kQ, ka = sbase + L::kBandK + st * L::kTile;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                    tc::mma_bf16_ss(tmem + L::tS0 + sb * BN, tc::sdesc_sw128(qa + off, 16, 1024),
                                    tc::sdesc_sw128(ka + off, 16, 1024), idS, kk > 0);
                }
                tc::mma_commit(bar(L::bSFull + sb));
                tc::mma_commit(bar(L::bKEmpty + st));
                return true;
            };
            if (ok && n_band > 0) ok = issue_S(0);
            for (int bl = 0; ok && bl < n_band; ++bl) {
                // S of the next block overlaps the softmax of this one (with a
                // single K stage its K arrives once S of this block is done)
                if (bl + 1 < n_band && !issue_S(bl + 1)) break;
                const int pb = bl % PB, vst = bl % VS;
                if (bl == 0 &&
                    !tc::mbar_wait(bar(L::bOInit), 0, abort, a.err, SA_DEVERR_TIMEOUT))
                    break;
                if (!tc::mbar_wait(bar(L::bPFull + pb), (bl / PB) & 1, abort, a.err,
                                   SA_DEVERR_TIMEOUT))
                    break;
                if (!tc::mbar_wait(bar(L::bVFull + vst), (bl / VS) & 1, abort, a.err,
                                   SA_DEVERR_TIMEOUT))
                    break;
                tc::tc_fence_after();
                const uint32_t pa = sbase + L::kP + pb * L::kPTile;
                const uint32_t va = sbase + L::kBandV + vst * L::kTile;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint32_t offp = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                    const uint32_t offv = kk * 16 * 128;
                    tc::mma_bf16_ss(tmem + L::tO, tc::sdesc_sw128(pa + offp, 16, 1024),
                                    tc::sdesc_sw128(va + offv, BN * 128, 1024), idO, 1u);
                }
                tc::mma_commit(bar(L::bVEmpty + vst));
                tc::mma_commit(bar(L::bPVDone + pb));
            }
        }
    } else if (warp == 2 || warp == 3) {
        // warp 2 stages the diagonal blocks; warp 3 has no role
        // ---------------- diagonal-block producer
        if (warp == 2 && DS > 0) {
            // CSR: lane l owns rows 4l .. 4l+3: list start, residual count and
            // the key of the next slot (fetched one slot ahead)
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
                const uint32_t kdst = sbase + L::kDiagK + st * L::kTile;
                const uint32_t vdst = sbase + L::kDiagV + st * L::kTile;
                if (use > 0 && !tc::mbar_wait(bar(L::bDiagEmpty + st), (use - 1) & 1, abort,
                                              a.err, SA_DEVERR_TIMEOUT))
                    break;
                if (lane == 0) tc::mbar_arrive_expect_tx(bar(L::bDiagFull + st), 2 * L::kTile);
                if (a.kind == 0) {
                    if (lane == 0) {
                        // distance links: keys q0-o .. q0+127-o, one box each for K and V
                        const int32_t krow = (int32_t)(q0 - a.offs[a.n_off - n_diag + d]);
                        for (int x = 0; x < D / 64; ++x) {
                            tc::tma_load_3d(kdst + x * (BM * 128), &tk, x * 64, krow, (int32_t)bh,
                                            bar(L::bDiagFull + st));
                            tc::tma_load_3d(vdst + x * (BM * 128), &tv, x * 64, krow, (int32_t)bh,
                                            bar(L::bDiagFull + st));
                        }
                    }
                } else {
                    // CSR slot d: 4-row TMA gathers of K and V rows (unswizzled);
                    // a row without slot d loads its own key (masked later)
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
        // ---------------- softmax warpgroup: thread r = query row r = TMEM lane r
        const int r = tid - 128;
        const int64_t i = q0 + r;
        const uint32_t lane_off = (uint32_t)((warp - 4) * 32) << 16;
        const uint32_t tS = tmem + lane_off + L::tS0, tO = tmem + lane_off + L::tO;
        const float c2 = a.scale2;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;

        // --- diagonal blocks: q row from the Q tile, one key/value row per block
        {
            float acc[D];
#pragma unroll
            for (int x = 0; x < D; ++x) acc[x] = 0.f;
            if (n_diag > 0) {
                ok = tc::mbar_wait(bar(L::bQFull), 0, abort, a.err, SA_DEVERR_TIMEOUT);
                uint32_t qr[D / 2];
                if (ok) {
                    // Structured blocks are swizzled like Q: q in logical order.
                    // CSR gathers are unswizzled: reading them at the swizzled
                    // address gives chunk c ^ (r & 7), which pairs with the
                    // physical (unpermuted-address) chunks of the Q row; the
                    // accumulator is then in that permuted order (undone below).
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) {
                        const uint32_t qoff = (c >> 3) * (BM * 128) +
                                              (a.kind == 0 ? tc::sw128_off(r, c & 7)
                                                           : (uint32_t)r * 128u + ((c & 7) << 4));
                        const uint4 w4 = *(const uint4 *)(sm + L::kQ + qoff);
                        qr[4 * c] = w4.x;
                        qr[4 * c + 1] = w4.y;
                        qr[4 * c + 2] = w4.z;
                        qr[4 * c + 3] = w4.w;
                    }
                }
                int64_t resid = 0;
                if (a.kind == 1 && i < T) {
                    const int64_t deg = a.rowptr[i + 1] - a.rowptr[i];
                    resid = deg - ((i + 1 < W) ? i + 1 : W);
                }
                for (int d = 0; ok && d < n_diag; ++d) {
                    const int st = d % DSX;
                    if (!tc::mbar_wait(bar(L::bDiagFull + st), (d / DSX) & 1, abort, a.err,
                                       SA_DEVERR_TIMEOUT)) {
                        ok = false;
                        break;
                    }
                    bool valid;
                    if (a.kind == 0)
                        valid = i < T && i >= a.offs[a.n_off - n_diag + d];
                    else
                        valid = d < resid;
                    if (valid) {
                        const uint8_t *kr = sm + L::kDiagK + st * L::kTile;
                        const uint8_t *vr = sm + L::kDiagV + st * L::kTile;
                        float s = 0.f;
#pragma unroll
                        for (int c = 0; c < D / 8; ++c) {
                            const uint4 w4 = *(const uint4 *)(kr + (c >> 3) * (BM * 128) +
                                                              tc::sw128_off(r, c & 7));
                            const uint32_t kw[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                s = fmaf(tc::bf16lo(qr[4 * c + e]), tc::bf16lo(kw[e]), s);
                                s = fmaf(tc::bf16hi(qr[4 * c + e]), tc::bf16hi(kw[e]), s);
                            }
                        }
                        s *= c2;
                        const float mn = fmaxf(m_run, s);
                        const float al = tc::ex2(m_run - mn), p = tc::ex2(s - mn);
                        l_run = l_run * al + p;
#pragma unroll
                        for (int c = 0; c < D / 8; ++c) {
                            const uint4 w4 = *(const uint4 *)(vr + (c >> 3) * (BM * 128) +
                                                              tc::sw128_off(r, c & 7));
                            const uint32_t vw[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                acc[8 * c + 2 * e] =
                                    fmaf(p, tc::bf16lo(vw[e]), acc[8 * c + 2 * e] * al);
                                acc[8 * c + 2 * e + 1] =
                                    fmaf(p, tc::bf16hi(vw[e]), acc[8 * c + 2 * e + 1] * al);
                            }
                        }
                        m_run = mn;
                    }
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar(L::bDiagEmpty + st));
                }
                if (a.kind == 1) {
                    // undo the chunk permutation through the (now idle) first
                    // diagonal stage: row r of D fp32 at r * 4D bytes
                    tc::named_barrier(1, 128);
                    float *scr = (float *)(sm + L::kDiagK) + (size_t)r * D;
#pragma unroll
                    for (int t = 0; t < D / 8; ++t) {
                        const int lc = (t & ~7) | ((t & 7) ^ (r & 7));
                        *(float4 *)(scr + 8 * lc) =
                            make_float4(acc[8 * t], acc[8 * t + 1], acc[8 * t + 2], acc[8 * t + 3]);
                        *(float4 *)(scr + 8 * lc + 4) = make_float4(
                            acc[8 * t + 4], acc[8 * t + 5], acc[8 * t + 6], acc[8 * t + 7]);
                    }
                    __syncwarp();
#pragma unroll
                    for (int t = 0; t < D / 4; ++t) {
                        const float4 f = *(const float4 *)(scr + 4 * t);
                        acc[4 * t] = f.x;
                        acc[4 * t + 1] = f.y;
                        acc[4 * t + 2] = f.z;
                        acc[4 * t + 3] = f.w;
                    }
                }
            }
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
            if (lane == 0) tc::mbar_arrive(bar(L::bOInit));
        }

        // --- band blocks
        for (int bl = 0; ok && bl < n_band; ++bl) {
            const int sb = bl & 1, pb = bl % PB;
            const int64_t b = b_first + bl;
            if (!tc::mbar_wait(bar(L::bSFull + sb), (bl >> 1) & 1, abort, a.err,
                               SA_DEVERR_TIMEOUT)) {
                ok = false;
                break;
            }
            tc::tc_fence_after();
            float s[BN];
#pragma unroll
            for (int c = 0; c < BN; c += 32) tc::tmem_ld32(tS + sb * BN + c, (uint32_t *)(s + c));
            tc::tmem_ld_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(L::bSFree + sb));

            // mask: r <= u <= r+W-1 and key >= 0, with u = 128 b + c, i.e. the
            // column range [c_lo, c_hi] of this block.  Scores stay raw (the
            // scale is folded into the exponent's FFMA); a masked raw score is
            // set to the extreme that the max/min below ignores.
            const int64_t u0 = b * BN;
            const bool need_mask = (u0 < BM - 1) || (u0 + BN - 1 > (int64_t)W - 1) ||
                                   (u0 + q0 < (int64_t)W - 1);
            const bool pos = c2 >= 0.f;
            const float ext = pos ? -INFINITY : INFINITY;
            if (need_mask) {
                const int64_t lo = ((int64_t)r > (int64_t)W - 1 - q0) ? r : (int64_t)W - 1 - q0;
                const int64_t hi = (int64_t)r + W - 1;
                const int c_lo = (int)(lo - u0 < 0 ? 0 : (lo - u0 > BN ? BN : lo - u0));
                const int c_hi = (int)(hi - u0 > BN - 1 ? BN - 1 : (hi - u0 < -1 ? -1 : hi - u0));
#pragma unroll
                for (int c = 0; c < BN; ++c) s[c] = (c >= c_lo && c <= c_hi) ? s[c] : ext;
            }
            float mr[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) mr[x] = ext;
            if (pos) {
#pragma unroll
                for (int c = 0; c < BN; ++c) mr[c & 7] = fmaxf(mr[c & 7], s[c]);
#pragma unroll
                for (int x = 4; x > 0; x >>= 1)
                    for (int y = 0; y < x; ++y) mr[y] = fmaxf(mr[y], mr[y + x]);
            } else {
#pragma unroll
                for (int c = 0; c < BN; ++c) mr[c & 7] = fminf(mr[c & 7], s[c]);
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
                if (bl > 0) {
                    const int pp = (bl - 1) % PB;
                    if (!tc::mbar_wait(bar(L::bPVDone + pp), ((bl - 1) / PB) & 1, abort, a.err,
                                       SA_DEVERR_TIMEOUT)) {
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
            // p = 2^(s - m), row sum, bf16 P into the swizzled K-major tile
            if (bl >= PB) {
                if (!tc::mbar_wait(bar(L::bPVDone + pb), ((bl - PB) / PB) & 1, abort, a.err,
                                   SA_DEVERR_TIMEOUT)) {
                    ok = false;
                    break;
                }
            }
            uint8_t *prow = sm + L::kP + pb * L::kPTile;
            const float m_use = (m_run == -INFINITY) ? 0.f : m_run;  // all-masked row: p = 0
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
            if (need_mask) {
#pragma unroll
                for (int c8 = 0; c8 < BN / 8; ++c8) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float x0 = s[8 * c8 + 2 * e], x1 = s[8 * c8 + 2 * e + 1];
                        const float p0 = (x0 != ext) ? tc::ex2(fmaf(x0, c2, -m_use)) : 0.f;
                        const float p1 = (x1 != ext) ? tc::ex2(fmaf(x1, c2, -m_use)) : 0.f;
                        ls[e] += p0 + p1;
                        w[e] = tc::pack_bf16x2(p0, p1);
                    }
                    *(uint4 *)(prow + (c8 >> 3) * (BM * 128) + tc::sw128_off(r, c8 & 7)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                }
            } else {
#pragma unroll
                for (int c8 = 0; c8 < BN / 8; ++c8) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float p0 = tc::ex2(fmaf(s[8 * c8 + 2 * e], c2, -m_use));
                        const float p1 = tc::ex2(fmaf(s[8 * c8 + 2 * e + 1], c2, -m_use));
                        ls[e] += p0 + p1;
                        w[e] = tc::pack_bf16x2(p0, p1);
                    }
                    *(uint4 *)(prow + (c8 >> 3) * (BM * 128) + tc::sw128_off(r, c8 & 7)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            const float lsum = (ls[0] + ls[1]) + (ls[2] + ls[3]);
            l_run += lsum;
            tc::fence_proxy_async_smem();
            tc::tmem_st_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar(L::bPFull + pb));
        }

        // --- epilogue
        if (ok && n_band > 0) {
            const int lb = n_band - 1;
            ok = tc::mbar_wait(bar(L::bPVDone + lb % PB), (lb / PB) & 1, abort, a.err,
                               SA_DEVERR_TIMEOUT);
        }
        if (ok) {
            tc::tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            __nv_bfloat16 *orow = a.out + ((size_t)bh * (size_t)T + (size_t)i) * D;
#pragma unroll
            for (int c = 0; c < D; c += 32) {
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

template <int D, int KS, int VS, int DS, int PB>
sa_status launch_band_fwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                          const sa_graph_s *g, float scale, sa_tensor *out, float *lse,
                          cudaStream_t s) {
    using L = Layout<D, KS, VS, DS, PB>;
    static_assert(L::kAlloc <= 232448, "shared memory budget");
    const int64_t BH = q->B * q->H, T = q->T;
    CUtensorMap mq, mk, mv, mkr, mvr;
    if (!sa_tmap_bf16_3d(&mq, q->ptr, D, T, BH, BM) || !sa_tmap_bf16_3d(&mk, k->ptr, D, T, BH, BN) ||
        !sa_tmap_bf16_3d(&mv, v->ptr, D, T, BH, BN) ||
        !sa_tmap_bf16_rows(&mkr, k->ptr, D, (uint64_t)(BH * T)) ||
        !sa_tmap_bf16_rows(&mvr, v->ptr, D, (uint64_t)(BH * T)))
    {
        sa_record_cuda_error(cudaErrorInvalidValue, "band_fwd: tensor map encoding");
        return SA_ERR_CUDA;
    }
    FwdArgs a{};
    a.T = T;
    a.W = g->W;
    a.kind = g->kind;
    a.n_off = g->kind == 0 ? g->n_off : 0;
    for (int x = 0; x < SA_MAX_OFFSETS; ++x) a.offs[x] = x < a.n_off ? g->offs[x] : 0;
    a.rowptr = g->rowptr;
    a.colidx = g->colidx;
    a.k = (const __nv_bfloat16 *)k->ptr;
    a.v = (const __nv_bfloat16 *)v->ptr;
    a.out = (__nv_bfloat16 *)out->ptr;
    a.lse = lse;
    a.scale2 = scale * kLog2e;
    a.err = sa_device_error_word();
    if (!a.err) return SA_ERR_CUDA;
    auto kern = band_fwd_kernel<D, KS, VS, DS, PB>;
    SA_CUDA_TRY(sa_smem_optin((const void *)kern, L::kAlloc));
    dim3 grid((unsigned)((T + BM - 1) / BM), (unsigned)BH);
    SA_LAUNCH("band_fwd", s, kern<<<grid, 256, L::kAlloc, s>>>(mq, mk, mv, mkr, mvr, a));
    SA_CUDA_TRY(cudaGetLastError());
    return SA_OK;
}

}  // namespace

bool sa_band_fwd_supported(const sa_tensor *q, const sa_graph_s *g) {
    if (q->dtype != SA_BF16 || (q->D != 64 && q->D != 128)) return false;
    if (g->W < 1) return false;                       // no band: gather path
    if (q->B * q->H > 65535 || q->T >= ((int64_t)1 << 31)) return false;
    if (g->kind == 1 && !g->rowptr) return false;
    return true;
}

sa_status sa_band_fwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                      const sa_graph_s *g, const GraphView &, float scale, sa_tensor *out,
                      float *lse, cudaStream_t s) {
    const bool diag = (g->kind == 0) ? g->n_off > 0 : g->max_resid > 0;
    // <D, K stages, V stages, diagonal stages, P buffers>, sized to the
    // 227 KB of shared memory
    if (q->D == 64) {
        return diag ? launch_band_fwd<64, 2, 3, 2, 2>(q, k, v, g, scale, out, lse, s)
                    : launch_band_fwd<64, 2, 3, 0, 2>(q, k, v, g, scale, out, lse, s);
    }
    return diag ? launch_band_fwd<128, 1, 1, 1, 1>(q, k, v, g, scale, out, lse, s)
                : launch_band_fwd<128, 2, 3, 0, 1>(q, k, v, g, scale, out, lse, s);
}
