// sa_internal.cuh -- shared internals of libsparse_attn (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sparse_attn.h"

#define SA_MAX_OFFSETS 63

// Library-side graph.  A structured graph is implicit (W + distances); its
// CSR arrays exist only when materialised.  A CSR graph always holds its
// normalised lists and their transpose.
struct sa_graph_s {
    int64_t T = 0;
    int kind = 0;           // 0 structured, 1 CSR
    int32_t W = 0;          // structured: window; CSR: verified band (0 = none)
    int32_t n_off = 0;      // structured: distances >= W and < T
    int64_t offs[SA_MAX_OFFSETS] = {0};  // descending
    int64_t nnz = 0;
    int materialized = 0;
    int64_t *rowptr = nullptr;
    int32_t *colidx = nullptr;
    int64_t *rev_rowptr = nullptr;
    int32_t *rev_colidx = nullptr;
    int32_t max_resid = 0;      // max edges outside the band over rows
    int32_t gprefix = 0;        // CSR: every row i holds keys 0 .. min(gprefix, i + 1) - 1
    int32_t max_resid_rev = 0;  // max transpose edges outside the band over keys
    int device = 0;
};

// Everything a kernel needs to enumerate N(i) and its transpose.
struct GraphView {
    int64_t T;
    int32_t kind;
    int32_t W;      // window (structured) or band (CSR)
    int32_t n_off;
    int64_t offs[SA_MAX_OFFSETS];  // descending
    const int64_t *rowptr;
    const int32_t *colidx;
    const int64_t *rev_rowptr;
    const int32_t *rev_colidx;
};

GraphView make_view(const sa_graph_s *g);

// Launch accounting, optional per-kernel event timing, the device error word.
void sa_count_launch(int n = 1);
void sa_prof_begin(const char *kernel, cudaStream_t s);
void sa_prof_end(cudaStream_t s);
#define SA_LAUNCH(name, s, ...)        \
    do {                               \
        sa_prof_begin(name, s);        \
        __VA_ARGS__;                   \
        sa_prof_end(s);                \
        sa_count_launch();             \
    } while (0)
int *sa_device_error_word();  // device address of this device's error word
int sa_link_pass_mode();      // sparse_attn_set_link_pass's setting


#define SA_DEVERR_TIMEOUT 1
#define SA_DEVERR_BOUNDS 2

// Closed forms of the structured graph (host and device).
__host__ __device__ inline int64_t sg_window_prefix(int64_t i, int64_t W) {
    // sum_{i' < i} min(i' + 1, W)
    if (i <= W) return i * (i + 1) / 2;
    return W * (W + 1) / 2 + (i - W) * W;
}

__host__ __device__ inline int64_t sg_rowptr(int64_t i, int64_t W, int n_off, const int64_t *offs) {
    int64_t r = sg_window_prefix(i, W);
    for (int a = 0; a < n_off; ++a) r += (i > offs[a]) ? (i - offs[a]) : 0;
    return r;
}

__host__ __device__ inline int64_t sg_degree(int64_t i, int64_t W, int n_off, const int64_t *offs) {
    int64_t d = (i + 1 < W) ? i + 1 : W;
    for (int a = 0; a < n_off; ++a) d += (offs[a] <= i) ? 1 : 0;
    return d;
}

__host__ __device__ inline int64_t sg_rev_rowptr(int64_t j, int64_t T, int64_t W, int n_off,
                                                 const int64_t *offs) {
    // sum_{j' < j} [ min(T - j', W) + #{o : j' + o < T} ]
    int64_t lim = T - W + 1;
    if (lim < 0) lim = 0;
    int64_t a = j < lim ? j : lim;  // keys j' < a have a full window of queries
    int64_t r = a * W + (j - a) * T - (a + j - 1) * (j - a) / 2;
    for (int b = 0; b < n_off; ++b) {
        int64_t c = T - offs[b];
        if (c < 0) c = 0;
        r += j < c ? j : c;
    }
    return r;
}

__host__ __device__ inline int64_t sg_in_degree(int64_t j, int64_t T, int64_t W, int n_off,
                                                const int64_t *offs) {
    int64_t d = (T - j < W) ? T - j : W;
    for (int b = 0; b < n_off; ++b) d += (j + offs[b] < T) ? 1 : 0;
    return d;
}

// Distance links of a structured graph that fall inside the span of keys the
// band blocks of a 128-row tile cover anyway (ceil((W + 127) / blk) blocks of
// blk keys starting at the first window key): such a link o is one more kept
// key per row inside those blocks, and is taken out of the gathered links.
// Writes the folded links (ascending, at most max_fold) to fold[], the others
// (descending) to rest[] and returns the span of the band blocks, We = W or
// the longest folded link + 1 (the blocks then start at key i - We + 1).
inline int32_t sa_fold_links(const sa_graph_s *g, int blk, int max_fold, int32_t *fold,
                             int *n_fold, int64_t *rest, int *n_rest) {
    *n_fold = 0;
    *n_rest = 0;
    int32_t We = g->W;
    const int64_t span = (int64_t)blk * ((g->W + 127 + blk - 1) / blk) - 127;
    for (int x = g->n_off - 1; x >= 0; --x) {  // ascending
        const int64_t o = g->offs[x];
        if (g->kind == 0 && o < span && *n_fold < max_fold) {
            fold[(*n_fold)++] = (int32_t)o;
            We = (int32_t)o + 1;
        }
    }
    for (int x = 0; x < g->n_off; ++x) {
        const int64_t o = g->offs[x];
        bool folded = false;
        for (int y = 0; y < *n_fold; ++y) folded |= (fold[y] == o);
        if (!folded) rest[(*n_rest)++] = o;
    }
    return We;
}

// Number of SMs of the current device (cached per device).
cudaError_t sa_sm_count(int *n);

// Opt a kernel into `bytes` of dynamic shared memory, once per (kernel, device).
cudaError_t sa_smem_optin(const void *kernel, int bytes);

// CUDA error helpers (host)
// Record the failing CUDA call (file:line, expression, error string) for
// sparse_attn_last_error_message().
void sa_record_cuda_error(cudaError_t e, const char *where);
#define SA_STR2(x) #x
#define SA_STR(x) SA_STR2(x)
#define SA_CUDA_TRY(expr)                                                         \
    do {                                                                          \
        cudaError_t _e = (expr);                                                  \
        if (_e != cudaSuccess) {                                                  \
            sa_record_cuda_error(_e, __FILE__ ":" SA_STR(__LINE__) ": " #expr);   \
            return SA_ERR_CUDA;                                                   \
        }                                                                         \
    } while (0)

// Internal launchers (graph.cu)
sa_status sa_graph_materialize_structured(sa_graph_s *g, cudaStream_t s);
sa_status sa_graph_from_csr(sa_graph_s *g, const int64_t *rowptr, const int32_t *colidx,
                            int64_t nnz, int32_t band, cudaStream_t s);

// Internal launchers (attn_gather.cu): every edge on CUDA cores.
sa_status sa_gather_fwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                        const GraphView &gv, float scale, sa_tensor *out, float *lse,
                        cudaStream_t s);
// Every argument check of the backward (nothing is launched).
sa_status sa_bwd_check_args(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                            const sa_tensor *out, const float *lse, const sa_tensor *dout,
                            sa_graph g, float scale, const sa_tensor *dq, const sa_tensor *dk,
                            const sa_tensor *dv);
// Backward with caller-placed scratch: Delta (4 bytes per query row) and an
// optional distance-edge cache (null: recompute); argument checks included.
sa_status sa_bwd_with_scratch(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                              const sa_tensor *out, const float *lse, const sa_tensor *dout,
                              sa_graph g, float scale, sa_tensor *dq, sa_tensor *dk,
                              sa_tensor *dv, float *delta, void *edge_cache, void *stream);
sa_status sa_gather_bwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                        const sa_tensor *out, const float *lse, const sa_tensor *dout,
                        const GraphView &gv, float scale, sa_tensor *dq, sa_tensor *dk,
                        sa_tensor *dv, float *delta, cudaStream_t s);

// Internal launchers (attn_dist.cu): learned-coordinate scoring, every edge
// on CUDA cores.  a, c: fp32 [B, H, T, 3]; v, out, dout, dv: [B, H, T, D].
sa_status sa_dist_fwd(const sa_tensor *a, const sa_tensor *c, const sa_tensor *v,
                      const GraphView &g, float scale, sa_tensor *out, float *lse,
                      cudaStream_t s);
sa_status sa_dist_bwd(const sa_tensor *a, const sa_tensor *c, const sa_tensor *v,
                      const sa_tensor *o, const float *lse, const sa_tensor *dout,
                      const GraphView &g, float scale, sa_tensor *da, sa_tensor *dc,
                      sa_tensor *dv, float *delta, cudaStream_t s);

// Internal launcher (attn_decode.cu): one query per (b, h) against a cache.
// q, out: [B, H, 1, D]; k, v: [B, Hkv, Tmax, D]; pos: device int64 [B].
sa_status sa_decode(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                    const int64_t *pos, const GraphView &g, float scale, sa_tensor *out,
                    float *lse, cudaStream_t s);
