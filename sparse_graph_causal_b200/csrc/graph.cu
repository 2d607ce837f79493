// graph.cu -- building the neighbour graph on the device.
//
// Structured graph (page "SpatialLM-Mini ...", section "How tokens choose
// whom to listen to"; window rule of "MiniGPT (Part 6)", section "A mask is
// not enough"): every row and every transpose row has a closed-form start
// and contents, so one thread writes one row; no scan, no sort.
//
// CSR graph (page "Longer Attention Span ...", Abstract: the mask is an edge
// set): validate -> stable LSD radix sort of (key, row) pairs by key, then by
// row -> drop repeats -> compact.  The transpose is one more stable sort of
// the normalised (row, key) pairs by key, so each transpose list comes out
// with its queries ascending.  Every step is deterministic.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "sa_internal.cuh"

namespace {

constexpr int kThreads = 256;
// Longest shared key prefix looked for: one 64-key block of the forward.
const int kPrefixCap = 64;

// ------------------------------------------------------------------ scan

constexpr int kScanItems = 8;
constexpr int kScanTile = kThreads * kScanItems;  // 2048

template <typename Tin>
__global__ void scan_tile_sums(const Tin *in, int64_t n, int64_t *tile_sums) {
    __shared__ int64_t warp_sums[kThreads / 32];
    int64_t base = (int64_t)blockIdx.x * kScanTile;
    int64_t s = 0;
    for (int r = 0; r < kScanItems; ++r) {
        int64_t idx = base + (int64_t)r * kThreads + threadIdx.x;
        if (idx < n) s += (int64_t)in[idx];
    }
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        int64_t t = 0;
        for (int w = 0; w < kThreads / 32; ++w) t += warp_sums[w];
        tile_sums[blockIdx.x] = t;
    }
}

// Exclusive scan of tile sums in one block (sequential over chunks).
__global__ void scan_tile_offsets(int64_t *tile_sums, int64_t ntiles, int64_t *total) {
    __shared__ int64_t buf[kThreads];
    __shared__ int64_t carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int64_t c0 = 0; c0 < ntiles; c0 += kThreads) {
        int64_t idx = c0 + threadIdx.x;
        int64_t v = idx < ntiles ? tile_sums[idx] : 0;
        buf[threadIdx.x] = v;
        __syncthreads();
        for (int o = 1; o < kThreads; o <<= 1) {
            int64_t add = threadIdx.x >= o ? buf[threadIdx.x - o] : 0;
            __syncthreads();
            buf[threadIdx.x] += add;
            __syncthreads();
        }
        int64_t incl = buf[threadIdx.x];
        if (idx < ntiles) tile_sums[idx] = carry + incl - v;
        __syncthreads();
        if (threadIdx.x == kThreads - 1) carry += incl;
        __syncthreads();
    }
    if (threadIdx.x == 0 && total) *total = carry;
}

template <typename Tin, typename Tout>
__global__ void scan_tiles_apply(const Tin *in, int64_t n, const int64_t *tile_offsets, Tout *out) {
    __shared__ int64_t warp_tot[kThreads / 32];
    int64_t base = (int64_t)blockIdx.x * kScanTile;
    // each thread owns kScanItems consecutive elements
    int64_t first = base + (int64_t)threadIdx.x * kScanItems;
    int64_t vals[kScanItems];
    int64_t s = 0;
    for (int r = 0; r < kScanItems; ++r) {
        int64_t idx = first + r;
        vals[r] = idx < n ? (int64_t)in[idx] : 0;
        s += vals[r];
    }
    int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t incl = s;
    for (int o = 1; o < 32; o <<= 1) {
        int64_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int64_t wbase = 0;
    for (int w = 0; w < warp; ++w) wbase += warp_tot[w];
    int64_t run = tile_offsets[blockIdx.x] + wbase + incl - s;
    for (int r = 0; r < kScanItems; ++r) {
        int64_t idx = first + r;
        if (idx < n) out[idx] = (Tout)run;
        run += vals[r];
    }
}

// out[i] = sum_{i' < i} in[i'] for i in [0, n); *total (device) = sum of all.
template <typename Tin, typename Tout>
sa_status exclusive_scan(const Tin *in, int64_t n, Tout *out, int64_t *total_dev, int64_t *tmp,
                         cudaStream_t s) {
    int64_t ntiles = (n + kScanTile - 1) / kScanTile;
    if (ntiles == 0) ntiles = 1;
    SA_LAUNCH("graph_scan_sums", s, scan_tile_sums<Tin><<<(unsigned)ntiles, kThreads, 0, s>>>(in, n, tmp));
    SA_LAUNCH("graph_scan_offsets", s, scan_tile_offsets<<<1, kThreads, 0, s>>>(tmp, ntiles, total_dev));
    SA_LAUNCH("graph_scan_apply", s,
              scan_tiles_apply<Tin, Tout><<<(unsigned)ntiles, kThreads, 0, s>>>(in, n, tmp, out));
    SA_CUDA_TRY(cudaGetLastError());
    return SA_OK;
}

int64_t scan_tmp_elems(int64_t n) { return (n + kScanTile - 1) / kScanTile + 1; }

// ------------------------------------------------------------ radix sort

constexpr int kRsItems = 16;
constexpr int kRsTile = kThreads * kRsItems;  // 4096 keys per tile

__global__ void rs_hist(const uint32_t *keys, int64_t n, int shift, uint32_t *counts,
                        int64_t ntiles) {
    __shared__ uint32_t h[256];
    h[threadIdx.x] = 0;
    __syncthreads();
    int64_t base = (int64_t)blockIdx.x * kRsTile;
    for (int r = 0; r < kRsItems; ++r) {
        int64_t idx = base + (int64_t)r * kThreads + threadIdx.x;
        if (idx < n) atomicAdd(&h[(keys[idx] >> shift) & 255u], 1u);
    }
    __syncthreads();
    counts[(int64_t)threadIdx.x * ntiles + blockIdx.x] = h[threadIdx.x];
}

// Stable scatter: keys are taken in index order, 256 at a time; within a
// round the rank of a key among equal digits is (earlier warps) + (earlier
// lanes of its own warp).
__global__ void rs_scatter(const uint32_t *keys_in, const uint32_t *vals_in, uint32_t *keys_out,
                           uint32_t *vals_out, int64_t n, int shift, const uint32_t *offsets,
                           int64_t ntiles) {
    __shared__ uint32_t base[256];
    __shared__ uint32_t whist[kThreads / 32][256];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    base[tid] = offsets[(int64_t)tid * ntiles + blockIdx.x];
    int64_t tile0 = (int64_t)blockIdx.x * kRsTile;
    for (int r = 0; r < kRsItems; ++r) {
        for (int w = 0; w < kThreads / 32; ++w) whist[w][tid] = 0;
        __syncthreads();
        int64_t idx = tile0 + (int64_t)r * kThreads + tid;
        bool valid = idx < n;
        uint32_t key = valid ? keys_in[idx] : 0u;
        uint32_t val = valid ? vals_in[idx] : 0u;
        uint32_t d = (key >> shift) & 255u;
        uint32_t peers = __match_any_sync(0xffffffffu, valid ? d : 0x1000u);
        int rank = __popc(peers & ((1u << lane) - 1u));
        if (valid && rank == 0) whist[warp][d] = __popc(peers);
        __syncthreads();
        uint32_t run = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            uint32_t c = whist[w][tid];
            whist[w][tid] = run;
            run += c;
        }
        __syncthreads();
        if (valid) {
            uint32_t pos = base[d] + whist[warp][d] + (uint32_t)rank;
            keys_out[pos] = key;
            vals_out[pos] = val;
        }
        __syncthreads();
        base[tid] += run;
        __syncthreads();
    }
}

struct SortBuffers {
    uint32_t *k2 = nullptr, *v2 = nullptr, *counts = nullptr, *offs = nullptr;
    int64_t *tmp = nullptr, *total = nullptr;
};

unsigned blocks_for(int64_t n, int per = kThreads) {
    int64_t b = (n + per - 1) / per;
    return (unsigned)(b < 1 ? 1 : b);
}

// Stable sort of (keys, vals) by the low `bits` bits of keys, in place
// (ping-pong through the scratch buffers; an odd pass count copies back).
sa_status radix_sort_pairs(uint32_t *keys, uint32_t *vals, int64_t n, int bits, SortBuffers &b,
                           cudaStream_t s) {
    if (n <= 1) return SA_OK;
    int64_t ntiles = (n + kRsTile - 1) / kRsTile;
    int64_t nc = 256 * ntiles;
    uint32_t *ki = keys, *vi = vals, *ko = b.k2, *vo = b.v2;
    int passes = 0;
    for (int shift = 0; shift < bits; shift += 8, ++passes) {
        SA_LAUNCH("graph_radix_hist", s,
                  rs_hist<<<(unsigned)ntiles, kThreads, 0, s>>>(ki, n, shift, b.counts, ntiles));
        sa_status st = exclusive_scan<uint32_t, uint32_t>(b.counts, nc, b.offs, b.total, b.tmp, s);
        if (st != SA_OK) return st;
        SA_LAUNCH("graph_radix_scatter", s,
                  rs_scatter<<<(unsigned)ntiles, kThreads, 0, s>>>(ki, vi, ko, vo, n, shift, b.offs,
                                                                   ntiles));
        std::swap(ki, ko);
        std::swap(vi, vo);
    }
    if (ki != keys) {
        SA_CUDA_TRY(cudaMemcpyAsync(keys, ki, n * 4, cudaMemcpyDeviceToDevice, s));
        SA_CUDA_TRY(cudaMemcpyAsync(vals, vi, n * 4, cudaMemcpyDeviceToDevice, s));
    }
    SA_CUDA_TRY(cudaGetLastError());
    return SA_OK;
}

int bits_for(int64_t maxval) {
    int b = 0;
    while (b < 32 && (((int64_t)1 << b) <= maxval)) ++b;
    return b < 1 ? 1 : b;
}

// ------------------------------------------------------- structured rows

struct OffsetsArg {
    int64_t o[SA_MAX_OFFSETS];
};

// Row i: the distance links (largest distance first, so keys ascend), then
// the window max(0, i-W+1) .. i.
__global__ void structured_rows(int64_t T, int32_t W, int n_off, OffsetsArg offs, int64_t *rowptr,
                                int32_t *colidx) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i > T) return;
    int64_t start = sg_rowptr(i, W, n_off, offs.o);
    rowptr[i] = start;
    if (i == T) return;
    int64_t p = start;
    for (int a = 0; a < n_off; ++a)
        if (offs.o[a] <= i) colidx[p++] = (int32_t)(i - offs.o[a]);
    int64_t lo = i - W + 1;
    if (lo < 0) lo = 0;
    for (int64_t j = lo; j <= i; ++j) colidx[p++] = (int32_t)j;
}

// Transpose row j: queries j .. min(T-1, j+W-1), then j + o for ascending
// distances o with j + o < T.
__global__ void structured_rev_rows(int64_t T, int32_t W, int n_off, OffsetsArg offs,
                                    int64_t *rev_rowptr, int32_t *rev_colidx) {
    int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j > T) return;
    int64_t start = sg_rev_rowptr(j, T, W, n_off, offs.o);
    rev_rowptr[j] = start;
    if (j == T) return;
    int64_t p = start;
    int64_t hi = j + W - 1;
    if (hi > T - 1) hi = T - 1;
    for (int64_t i = j; i <= hi; ++i) rev_colidx[p++] = (int32_t)i;
    for (int a = n_off - 1; a >= 0; --a)
        if (j + offs.o[a] < T) rev_colidx[p++] = (int32_t)(j + offs.o[a]);
}

// -------------------------------------------------------------- CSR build

#define CSR_ERR_ROWPTR 1
#define CSR_ERR_LOOKAHEAD 2
#define CSR_ERR_NEGATIVE 4
#define CSR_ERR_BAND 8

// One warp per row: rowptr shape, key range, and the row id of every edge.
__global__ void csr_validate_expand(int64_t T, const int64_t *rowptr, const int32_t *colidx,
                                    int64_t nnz, uint32_t *row_of_edge, uint32_t *key_of_edge,
                                    int *err) {
    int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int lane = threadIdx.x & 31;
    if (i >= T) return;
    int64_t b = rowptr[i], e = rowptr[i + 1];
    if (lane == 0) {
        if ((i == 0 && b != 0) || e < b || (i == T - 1 && e != nnz) || e > nnz || b < 0)
            atomicOr(err, CSR_ERR_ROWPTR);
    }
    if (e < b || b < 0 || e > nnz) return;
    int bad = 0;
    for (int64_t p = b + lane; p < e; p += 32) {
        int32_t j = colidx[p];
        if (j < 0) bad |= CSR_ERR_NEGATIVE;
        else if ((int64_t)j > i) bad |= CSR_ERR_LOOKAHEAD;
        row_of_edge[p] = (uint32_t)i;
        key_of_edge[p] = (uint32_t)(j < 0 ? 0 : j);
    }
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (lane == 0 && bad) atomicOr(err, bad);
}

// keep[e] = 1 when edge e (sorted by row, then key) differs from e-1.
__global__ void csr_mark_unique(const uint32_t *rows, const uint32_t *keys, int64_t n,
                                int32_t *keep) {
    int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n) return;
    keep[e] = (e == 0 || rows[e] != rows[e - 1] || keys[e] != keys[e - 1]) ? 1 : 0;
}

__global__ void csr_compact(const uint32_t *keys, const int32_t *keep, const int64_t *pos,
                            int64_t n, int32_t *colidx) {
    int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n) return;
    if (keep[e]) colidx[pos[e]] = (int32_t)keys[e];
}

// The sorted edge array keeps the caller's row segments, so the new row
// start is the count of kept edges before the old row start.
__global__ void csr_new_rowptr(int64_t T, const int64_t *rowptr_in, const int64_t *pos,
                               const int64_t *total, int64_t *rowptr_out) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i > T) return;
    int64_t b = rowptr_in[i];
    rowptr_out[i] = (i == T) ? *total : pos[b];
}

// Band check: the last min(i+1, Wb) keys of sorted, repeat-free row i must be
// exactly the window; also the largest count of edges outside the band.
__global__ void csr_band_check(int64_t T, const int64_t *rowptr, const int32_t *colidx, int32_t Wb,
                               int *err, int *max_resid) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= T) return;
    int64_t deg = rowptr[i + 1] - rowptr[i];
    int64_t c = (i + 1 < Wb) ? i + 1 : Wb;
    if (c > 0) {
        if (deg < c || colidx[rowptr[i + 1] - c] != (int32_t)(i - c + 1)) {
            atomicOr(err, CSR_ERR_BAND);
            return;
        }
    }
    int64_t r = deg - c;
    atomicMax(max_resid, (int)(r > 0x7fffffff ? 0x7fffffff : r));
}

// Shared key prefix: the largest G <= cap such that every row i holds the
// keys 0 .. min(G, i + 1) - 1 (global tokens every query sees).  Row i holds
// them when its sorted list starts 0, 1, ..., so each row that does not hold
// all of 0 .. i bounds G by the length of its run of leading keys 0, 1, ...
// (*g_min starts at cap).
__global__ void csr_key_prefix(int64_t T, const int64_t *rowptr, const int32_t *colidx, int cap,
                               int *g_min) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= T) return;
    const int64_t s = rowptr[i], deg = rowptr[i + 1] - s;
    int run = 0;
    while (run < cap && run < deg && colidx[s + run] == run) ++run;
    if (run < cap && (int64_t)run < i + 1) atomicMin(g_min, run);
}

__global__ void csr_rev_counts(const int32_t *colidx, int64_t nnz, int32_t *indeg) {
    int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e < nnz) atomicAdd(&indeg[colidx[e]], 1);
}

__global__ void csr_expand_rows(int64_t T, const int64_t *rowptr, uint32_t *row_of_edge,
                                uint32_t *key_of_edge, const int32_t *colidx) {
    int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int lane = threadIdx.x & 31;
    if (i >= T) return;
    for (int64_t p = rowptr[i] + lane; p < rowptr[i + 1]; p += 32) {
        row_of_edge[p] = (uint32_t)i;
        key_of_edge[p] = (uint32_t)colidx[p];
    }
}

__global__ void u32_to_i32(const uint32_t *in, int32_t *out, int64_t n) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = (int32_t)in[i];
}

// Largest transpose count outside the band: keys j see band queries
// j .. j+Wb-1 (clipped at T-1) first in their ascending list.
__global__ void csr_rev_resid(int64_t T, const int64_t *rev_rowptr, int32_t Wb, int *max_resid) {
    int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= T) return;
    int64_t deg = rev_rowptr[j + 1] - rev_rowptr[j];
    int64_t c = (T - j < Wb) ? T - j : Wb;
    int64_t r = deg - c;
    if (r < 0) r = 0;
    atomicMax(max_resid, (int)(r > 0x7fffffff ? 0x7fffffff : r));
}

// The graph builds' device memory (the CSR build's temporaries, 28 bytes per
// input entry: 2.8 GB for 10^8 entries, and the graph's own lists) comes
// from one memory pool per device that keeps up to kTmpKeep bytes between
// builds; from the default pool it went back to the driver at every
// synchronisation (or graph release), and mapping it again cost more than
// the sorts.  Null when no pool could be made (then the default pool serves).
constexpr uint64_t kTmpKeep = (uint64_t)4 << 30;
cudaMemPool_t tmp_pool() {
    static std::mutex mu;
    static cudaMemPool_t pools[64] = {};
    static bool tried[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(mu);
    if (!tried[dev]) {
        tried[dev] = true;
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t p = nullptr;
        if (cudaMemPoolCreate(&p, &props) == cudaSuccess) {
            uint64_t keep = kTmpKeep;
            cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
            pools[dev] = p;
        } else {
            cudaGetLastError();
        }
    }
    return pools[dev];
}

template <typename T>
sa_status dtmp(T **p, int64_t n, cudaStream_t s) {
    if (n < 1) n = 1;
    cudaMemPool_t pool = tmp_pool();
    cudaError_t e = pool ? cudaMallocFromPoolAsync((void **)p, sizeof(T) * (size_t)n, pool, s)
                         : cudaMallocAsync((void **)p, sizeof(T) * (size_t)n, s);
    if (e != cudaSuccess) {
        *p = nullptr;
        cudaGetLastError();
        return SA_ERR_OOM;
    }
    return SA_OK;
}

// The graph's own lists (released by sparse_attn_graph_destroy, whose
// cudaFree returns them to the pool).
template <typename T>
sa_status dalloc(T **p, int64_t n, cudaStream_t s) {
    return dtmp(p, n, s);
}

}  // namespace

sa_status sa_graph_materialize_structured(sa_graph_s *g, cudaStream_t s) {
    OffsetsArg oa;
    for (int a = 0; a < SA_MAX_OFFSETS; ++a) oa.o[a] = a < g->n_off ? g->offs[a] : 0;
    sa_status st;
    if ((st = dalloc(&g->rowptr, g->T + 1, s)) != SA_OK) return st;
    if ((st = dalloc(&g->colidx, g->nnz, s)) != SA_OK) return st;
    if ((st = dalloc(&g->rev_rowptr, g->T + 1, s)) != SA_OK) return st;
    if ((st = dalloc(&g->rev_colidx, g->nnz, s)) != SA_OK) return st;
    unsigned nb = blocks_for(g->T + 1);
    SA_LAUNCH("graph_structured_rows", s,
              structured_rows<<<nb, kThreads, 0, s>>>(g->T, g->W, g->n_off, oa, g->rowptr,
                                                      g->colidx));
    SA_LAUNCH("graph_structured_rev_rows", s,
              structured_rev_rows<<<nb, kThreads, 0, s>>>(g->T, g->W, g->n_off, oa, g->rev_rowptr,
                                                          g->rev_colidx));
    SA_CUDA_TRY(cudaGetLastError());
    g->materialized = 1;
    return SA_OK;
}

sa_status sa_graph_from_csr(sa_graph_s *g, const int64_t *rowptr, const int32_t *colidx,
                            int64_t nnz, int32_t band, cudaStream_t s) {
    const int64_t T = g->T;
    sa_status st = SA_OK;
    uint32_t *rows = nullptr, *keys = nullptr;
    int32_t *keep = nullptr, *indeg = nullptr;
    int64_t *pos = nullptr;
    int *flags = nullptr;  // [0] errors, [1] max resid, [2] max resid rev, [3] key prefix
    SortBuffers sb;
    int64_t n = nnz;
    int64_t ntiles = (n + kRsTile - 1) / kRsTile;
    int64_t nc = 256 * (ntiles < 1 ? 1 : ntiles);
    int64_t scan_n = std::max<int64_t>(std::max<int64_t>(n + 1, T + 1), nc);
    int host_flags[4] = {0, 0, 0, 0};
    int kbits = bits_for(T > 0 ? T - 1 : 0);

#define TRY(...)                        \
    do {                                \
        st = (__VA_ARGS__);             \
        if (st != SA_OK) goto cleanup;  \
    } while (0)
#define CTRY(x)                                   \
    do {                                          \
        if ((x) != cudaSuccess) {                 \
            st = SA_ERR_CUDA;                     \
            goto cleanup;                         \
        }                                         \
    } while (0)

    TRY(dtmp(&rows, n, s));
    TRY(dtmp(&keys, n, s));
    TRY(dtmp(&keep, n + 1, s));
    TRY(dtmp(&pos, n + 1, s));
    TRY(dtmp(&flags, 4, s));
    TRY(dtmp(&sb.k2, n, s));
    TRY(dtmp(&sb.v2, n, s));
    TRY(dtmp(&sb.counts, nc, s));
    TRY(dtmp(&sb.offs, nc, s));
    TRY(dtmp(&sb.tmp, scan_tmp_elems(scan_n), s));
    TRY(dtmp(&sb.total, 1, s));
    CTRY(cudaMemsetAsync(flags, 0, 4 * sizeof(int), s));

    // 1. validate, expand (row, key) pairs
    SA_LAUNCH("graph_csr_validate", s,
              csr_validate_expand<<<blocks_for(T * 32), kThreads, 0, s>>>(T, rowptr, colidx, nnz,
                                                                           rows, keys, flags));
    CTRY(cudaMemcpyAsync(host_flags, flags, sizeof(int), cudaMemcpyDeviceToHost, s));
    CTRY(cudaStreamSynchronize(s));
    if (host_flags[0]) {
        st = SA_ERR_INVALID_GRAPH;
        goto cleanup;
    }
    // 2. sort by key, then (stably) by row: rows grouped, keys ascending
    TRY(radix_sort_pairs(keys, rows, n, kbits, sb, s));
    TRY(radix_sort_pairs(rows, keys, n, kbits, sb, s));
    // 3. drop repeats and compact
    if (n > 0) {
        SA_LAUNCH("graph_csr_unique", s,
                  csr_mark_unique<<<blocks_for(n), kThreads, 0, s>>>(rows, keys, n, keep));
    }
    TRY(exclusive_scan<int32_t, int64_t>(keep, n, pos, sb.total, sb.tmp, s));
    CTRY(cudaMemcpyAsync(pos + n, sb.total, sizeof(int64_t), cudaMemcpyDeviceToDevice, s));
    int64_t new_nnz;
    CTRY(cudaMemcpyAsync(&new_nnz, sb.total, sizeof(int64_t), cudaMemcpyDeviceToHost, s));
    CTRY(cudaStreamSynchronize(s));
    g->nnz = new_nnz;
    TRY(dalloc(&g->rowptr, T + 1, s));
    TRY(dalloc(&g->colidx, new_nnz, s));
    TRY(dalloc(&g->rev_rowptr, T + 1, s));
    TRY(dalloc(&g->rev_colidx, new_nnz, s));
    TRY(dtmp(&indeg, T + 1, s));
    if (n > 0) {
        SA_LAUNCH("graph_csr_compact", s,
                  csr_compact<<<blocks_for(n), kThreads, 0, s>>>(keys, keep, pos, n, g->colidx));
    }
    SA_LAUNCH("graph_csr_rowptr", s,
              csr_new_rowptr<<<blocks_for(T + 1), kThreads, 0, s>>>(T, rowptr, pos, sb.total,
                                                                     g->rowptr));
    // 4. band check
    // (band 0: every edge lies outside the empty band)
    SA_LAUNCH("graph_csr_band", s,
              csr_band_check<<<blocks_for(T), kThreads, 0, s>>>(T, g->rowptr, g->colidx, band,
                                                                 flags, flags + 1));
    // shared key prefix (at most one 64-key block), for the forward's dense
    // prefix block
    CTRY(cudaMemcpyAsync(flags + 3, &kPrefixCap, sizeof(int), cudaMemcpyHostToDevice, s));
    SA_LAUNCH("graph_csr_prefix", s,
              csr_key_prefix<<<blocks_for(T), kThreads, 0, s>>>(T, g->rowptr, g->colidx,
                                                                 kPrefixCap, flags + 3));
    // 5. transpose: stable sort of (key, row) pairs of the normalised lists by key
    CTRY(cudaMemsetAsync(indeg, 0, sizeof(int32_t) * (size_t)(T + 1), s));
    if (new_nnz > 0) {
        SA_LAUNCH("graph_csr_indegree", s,
                  csr_rev_counts<<<blocks_for(new_nnz), kThreads, 0, s>>>(g->colidx, new_nnz,
                                                                          indeg));
        SA_LAUNCH("graph_csr_expand", s,
                  csr_expand_rows<<<blocks_for(T * 32), kThreads, 0, s>>>(T, g->rowptr, rows, keys,
                                                                           g->colidx));
    }
    TRY(exclusive_scan<int32_t, int64_t>(indeg, T + 1, g->rev_rowptr, sb.total, sb.tmp, s));
    TRY(radix_sort_pairs(keys, rows, new_nnz, kbits, sb, s));
    if (new_nnz > 0) {
        SA_LAUNCH("graph_csr_rev_copy", s,
                  u32_to_i32<<<blocks_for(new_nnz), kThreads, 0, s>>>(rows, g->rev_colidx,
                                                                      new_nnz));
    }
    SA_LAUNCH("graph_csr_rev_resid", s,
              csr_rev_resid<<<blocks_for(T), kThreads, 0, s>>>(T, g->rev_rowptr, band, flags + 2));
    CTRY(cudaGetLastError());
    CTRY(cudaMemcpyAsync(host_flags, flags, 4 * sizeof(int), cudaMemcpyDeviceToHost, s));
    CTRY(cudaStreamSynchronize(s));
    if (host_flags[0]) {
        st = SA_ERR_INVALID_GRAPH;
        goto cleanup;
    }
    g->W = band;
    g->max_resid = host_flags[1];
    g->max_resid_rev = host_flags[2];
    g->gprefix = host_flags[3];
    g->materialized = 1;

cleanup:
    cudaFreeAsync(rows, s);
    cudaFreeAsync(keys, s);
    cudaFreeAsync(keep, s);
    cudaFreeAsync(pos, s);
    cudaFreeAsync(flags, s);
    cudaFreeAsync(indeg, s);
    cudaFreeAsync(sb.k2, s);
    cudaFreeAsync(sb.v2, s);
    cudaFreeAsync(sb.counts, s);
    cudaFreeAsync(sb.offs, s);
    cudaFreeAsync(sb.tmp, s);
    cudaFreeAsync(sb.total, s);
#undef TRY
#undef CTRY
    return st;
}
