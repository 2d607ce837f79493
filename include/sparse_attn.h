/*
 * sparse_attn.h -- C ABI of the B200 (sm_100a) sparse-graph causal attention
 * library (libsparse_attn.so).
 *
 * The operation.  Every query position i of a sequence attends only to a
 * fixed, causal neighbour set N(i), the same for every batch row and head,
 * and the softmax runs over exactly those keys:
 *     s_ij   = scale * (q_i . k_j)                 for j in N(i)
 *     out_i  = sum_j softmax_j(s_ij) v_j
 *     lse_i  = ln sum_j exp(s_ij)                  (natural log)
 * The T x T score matrix is never formed.
 *  - N(i) for a structured graph: the token itself, its W-1 nearest
 *    predecessors, and the positions i - 2^k (page "SpatialLM-Mini sped up
 *    training with a 16K context by 2.47x on an RTX 3050", section "How
 *    tokens choose whom to listen to"); the window keeps j <= i with
 *    i - j < W (page "MiniGPT (Part 6)", section "A mask is not enough",
 *    first listing).  Scores are scaled before the softmax (same section,
 *    chunked_swa listing).
 *  - N(i) as arbitrary CSR lists: tokens are nodes, the mask gives the edges
 *    (page "Longer Attention Span: Increasing Transformer Context Length with
 *    Sparse Graph Processing Techniques", Abstract).
 * The backward recomputes the probabilities from lse and is deterministic:
 * dQ by the forward lists, dK/dV by the transpose (reverse) lists, no float
 * atomics.
 *
 * Conventions for every call:
 *  - Tensors are contiguous [B, H, T, D] (sa_tensor), D in {32, 64, 128},
 *    dtype bf16 or fp32; q, k, v, out, dout, dq, dk, dv of one call share
 *    B, H, T, D and dtype.  lse is fp32 [B, H, T].  Device pointers must be
 *    16-byte aligned.  The caller owns every tensor buffer.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  All
 *    work is enqueued on it; fwd and bwd never synchronise the host.
 *  - Arguments are checked on the host before anything is launched; a
 *    non-SA_OK status means nothing was enqueued.  Errors of work already
 *    enqueued surface as SA_ERR_CUDA on a later call, or through
 *    sparse_attn_check_device().  No C++ exception crosses this ABI.
 *  - One graph serves all B*H slices of a call.  Its T must equal the
 *    tensors' T.  A graph may be used from several streams at once once its
 *    build has completed on the build stream.
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SA_OK = 0,
    SA_ERR_INVALID_ARG = 1,    /* null pointer, shape or dtype mismatch, bad size */
    SA_ERR_INVALID_GRAPH = 2,  /* look-ahead / negative key, malformed rowptr,
                                  band_hint not contained in every row */
    SA_ERR_UNSUPPORTED = 3,    /* valid but outside what the kernels implement */
    SA_ERR_OOM = 4,            /* a graph allocation failed */
    SA_ERR_CUDA = 5,           /* a CUDA runtime error (possibly from earlier work) */
    SA_ERR_DEVICE_TIMEOUT = 6  /* a kernel's bounded wait ran out (see check_device) */
} sa_status;

typedef enum { SA_BF16 = 0, SA_FP32 = 1 } sa_dtype;

/* A contiguous [B, H, T, D] tensor in device memory.  `dtype` is an sa_dtype. */
typedef struct {
    void *ptr;
    int32_t dtype;
    int64_t B, H, T, D;
} sa_tensor;

/* Opaque graph handle, owned by the library; release with graph_destroy. */
typedef struct sa_graph_s *sa_graph;

/* ---------------------------------------------------------------- graphs */

/* Build the structured graph: window of W keys including self, plus the
 * distance links i - 2^k for each k in dil_exps[0..n_dil) (host array; any
 * order, repeats ignored, 0 <= k <= 62).  A link that reaches before
 * position 0 is dropped; a link inside the window is the same edge and is
 * counted once.  T >= 1, 1 <= W.  The kernels use this graph implicitly from
 * (W, distances); with materialize != 0 the CSR lists and their transpose are
 * also written to library-owned device memory (allocated stream-ordered on
 * `stream`) so that graph_export can copy them out (T < 2^31, nnz < 2^31
 * needed then).  Never synchronises the host.  *out receives the handle. */
sa_status sparse_attn_graph_build_structured(int64_t T, int32_t W, const int32_t *dil_exps,
                                             int32_t n_dil, int32_t materialize, void *stream,
                                             sa_graph *out);

/* Build a graph from caller CSR lists in DEVICE memory: rowptr int64[T+1]
 * (rowptr[0] = 0, non-decreasing, rowptr[T] = nnz), colidx int32[nnz].  Rows
 * may be unsorted and hold repeats; each row is sorted ascending and
 * deduplicated (page "Longer Attention Span ...": the mask is an edge set).
 * A key j > i or j < 0, or a malformed rowptr, gives SA_ERR_INVALID_GRAPH.
 * band_hint = Wb > 0 states that every row i contains the whole window
 * {max(0, i-Wb+1) .. i}; it is verified (SA_ERR_INVALID_GRAPH if false) and
 * lets those edges run on the dense band tiles.  band_hint = 0: every edge
 * runs on the gather kernels.  The transpose lists are built too (stable:
 * queries ascending).  The caller's arrays are only read and may be freed
 * after the call returns.  Synchronises `stream` three times (to read the
 * validation result, the deduplicated entry count and the final checks).
 * Its temporaries (28 bytes per input entry) and the graph's lists come from
 * a library-owned stream-ordered memory pool per device that keeps up to
 * 4 GiB between builds (the first build in a process maps it).  T < 2^31,
 * nnz < 2^31. */
sa_status sparse_attn_graph_build_csr(int64_t T, const int64_t *rowptr, const int32_t *colidx,
                                      int64_t nnz, int32_t band_hint, void *stream,
                                      sa_graph *out);

/* Edge count of the graph (deduplicated) and of its transpose (equal). */
sa_status sparse_attn_graph_nnz(sa_graph g, int64_t *nnz, int64_t *rev_nnz);

/* Copy the normalised lists into caller-owned DEVICE buffers: rowptr
 * int64[T+1], colidx int32[nnz] (each row ascending), rev_rowptr int64[T+1],
 * rev_colidx int32[nnz] (each list of queries ascending).  Any pointer may be
 * NULL to skip it.  A structured graph must have been built with
 * materialize != 0 (else SA_ERR_INVALID_ARG). */
sa_status sparse_attn_graph_export(sa_graph g, int64_t *rowptr, int32_t *colidx,
                                   int64_t *rev_rowptr, int32_t *rev_colidx, void *stream);

/* Free the graph (synchronises the device before freeing its memory). */
sa_status sparse_attn_graph_destroy(sa_graph g);

/* ------------------------------------------------------------- attention */

/* Forward.  out has q's dtype (rounded to nearest even from fp32
 * accumulation); lse is fp32 [B, H, T], natural log; an empty row gives
 * out = 0 and lse = -inf.  scale must be finite.  No workspace. */
sa_status sparse_attn_fwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v, sa_graph g,
                          float scale, sa_tensor *out, float *lse, void *stream);

/* Bytes of device workspace sparse_attn_bwd needs for these shapes and this
 * graph: 4 * B * H * T (Delta_i = dO_i . out_i in fp32) and, for a
 * structured graph with n distance links, 8 * n * B * H * T more (the
 * probability and dS of every distance edge, computed once by the dQ pass and
 * reused by the dK/dV pass), each part rounded up to 256 bytes. */
size_t sparse_attn_bwd_workspace_size(const sa_tensor *q, sa_graph g);

/* Backward of sparse_attn_fwd for the upstream gradient dout.  out and lse
 * are the forward's results.  dq, dk, dv are written in full (no
 * accumulation into them).  `workspace` is caller-owned device memory of at
 * least sparse_attn_bwd_workspace_size() bytes, 256-byte aligned.  Results
 * are bitwise reproducible run to run. */
sa_status sparse_attn_bwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                          const sa_tensor *out, const float *lse, const sa_tensor *dout, sa_graph g,
                          float scale, sa_tensor *dq, sa_tensor *dk, sa_tensor *dv,
                          void *workspace, size_t ws_bytes, void *stream);

/* Backward that allocates nothing and takes no workspace, for callers that
 * cannot allocate device memory at the call site: a host running under a
 * fixed device-memory plan (every byte reserved up front), or code inside an
 * allocator hook, where allocating again would re-enter the allocator.  The
 * pages have no counterpart of this call; it is a deployment convenience.
 * Same arguments as sparse_attn_bwd minus the workspace, and the same results
 * up to rounding: without room for the distance-edge cache its dK/dV pass
 * recomputes p and dS of the distance links (bitwise reproducible run to run
 * on its own).  Its scratch (Delta, 4 bytes per query row) is a fixed device
 * array of SA_NOALLOC_MAX_ROWS floats inside the library: every GPU that
 * loads the library holds it (4 MiB) until the process exits.  Arguments
 * are checked as in sparse_attn_bwd (SA_ERR_INVALID_ARG / _UNSUPPORTED);
 * then B*H*T above SA_NOALLOC_MAX_ROWS returns SA_ERR_UNSUPPORTED.  Either
 * way nothing is enqueued.  Every call on a device shares the array (it
 * keeps the last call's contents, none of which must start at zero), so
 * calls whose work overlaps on the GPU race: serialise them (one stream, or
 * events).  Every call looks up the array's device address in the current
 * context (cudaGetSymbolAddress); the first call on a device may also make
 * the driver load the library's device code, so make that first call before
 * any stream capture. */
#define SA_NOALLOC_MAX_ROWS (1 << 20)
sa_status sparse_attn_bwd_noalloc(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                                  const sa_tensor *out, const float *lse, const sa_tensor *dout,
                                  sa_graph g, float scale, sa_tensor *dq, sa_tensor *dk,
                                  sa_tensor *dv, void *stream);

/* ------------------------------------------------------------------ decode */

/* One new query per batch row and head against a KV cache, over the same
 * graph (page "SpatialLM-Mini ...", section "What to check before adopting
 * it in your project", notes the missing KV cache and unmeasured generation
 * speed).  q and out: [B, H, 1, D]; k_cache, v_cache: [B, Hkv, Tmax, D] with
 * Hkv dividing H (query head h reads cache head h / (H / Hkv): grouped-query
 * attention, page "MiniGPT (Part 6)", introduction); same dtype and D as q.
 * pos: DEVICE int64 [B], the query's position in batch row b -- its own key
 * and value must already be stored at cache row pos[b].  The query attends
 * to N(pos[b]) of graph g (g's T >= Tmax), exactly as row pos[b] of
 * sparse_attn_fwd would.  lse: fp32 [B, H].  A pos[b] outside [0, Tmax)
 * (only known on the device) gives out = 0, lse = -inf for that row and
 * flags the device error word (sparse_attn_check_device then reports
 * SA_ERR_CUDA); nothing faults.  No workspace, no host synchronisation. */
sa_status sparse_attn_decode(const sa_tensor *q, const sa_tensor *k_cache,
                             const sa_tensor *v_cache, const int64_t *pos, sa_graph g,
                             float scale, sa_tensor *out, float *lse, void *stream);

/* -------------------------------------------- learned-coordinate scoring */

/* The same neighbour graph with the edge weight taken from learnable
 * coordinates instead of a dot product (page "SpatialLM-Mini sped up
 * training with a 16K context by 2.47x on an RTX 3050", section "How tokens
 * choose whom to listen to": each token gets a three-dimensional query and
 * key coordinate, and the shorter their distance the higher the weight).
 * The page leaves the extra learnable adjustments unspecified; the form
 * computed is
 *     s_ij  = -scale * |a_i - c_j|^2            for j in N(i)
 *     out_i = sum_j softmax_j(s_ij) v_j,   lse_i = ln sum_j exp(s_ij).
 * a (query coordinates) and c (key coordinates) are fp32 [B, H, T, 3]
 * (sa_tensor with D = 3, dtype SA_FP32, same B, H, T as v); v and out are
 * bf16 or fp32 [B, H, T, D], D in {32, 64, 128}; lse fp32 [B, H, T].  Every
 * edge runs on CUDA cores (a score is three FMAs).  No workspace. */
sa_status sparse_attn_dist_fwd(const sa_tensor *a, const sa_tensor *c, const sa_tensor *v,
                               sa_graph g, float scale, sa_tensor *out, float *lse, void *stream);

/* Workspace of sparse_attn_dist_bwd: 4 * B * H * T bytes (Delta), rounded up
 * to 256 bytes.  `v` gives the shape. */
size_t sparse_attn_dist_bwd_workspace_size(const sa_tensor *v, sa_graph g);

/* Backward of sparse_attn_dist_fwd for upstream gradient dout: da, dc
 * (fp32 [B, H, T, 3]) and dv (v's dtype) are written in full.  Recomputes
 * the probabilities from lse; two kernels with disjoint outputs (da by the
 * forward lists, dc and dv by the transpose lists), no atomics, bitwise
 * reproducible.  workspace: caller-owned device memory, 256-byte aligned. */
sa_status sparse_attn_dist_bwd(const sa_tensor *a, const sa_tensor *c, const sa_tensor *v,
                               const sa_tensor *out, const float *lse, const sa_tensor *dout,
                               sa_graph g, float scale, sa_tensor *da, sa_tensor *dc,
                               sa_tensor *dv, void *workspace, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------ utilities */

/* Human-readable name of a status. */
const char *sparse_attn_status_string(sa_status s);

/* Kernel selection for fwd/bwd (process-wide; default SA_PATH_AUTO):
 *  SA_PATH_AUTO   bf16 with D in {32, 64, 128} and a band (W >= 1) runs the
 *                 tcgen05 band kernels: the window on the tensor cores, the
 *                 other edges as diagonal blocks on the CUDA cores of the same
 *                 kernels (D = 32 on the D = 64 tiles, rows zero-extended);
 *                 everything else runs the gather kernels alone.
 *  SA_PATH_GATHER every edge on the gather kernels (CUDA cores). */
typedef enum { SA_PATH_AUTO = 0, SA_PATH_GATHER = 1 } sa_path;
sa_status sparse_attn_set_path(int32_t path);

/* Long distance links of a structured graph (process-wide; default
 * SA_LINKS_AUTO).  The band-kernel forward can take the links of at least
 * 2^13 rows (when all such links are multiples of 2^13, e.g. powers of two)
 * in a second pass that runs the tiles in an order keeping their K/V rows in
 * L2 ("Longer Attention Span ...", Abstract: single-GPU sequences of 160 M
 * tokens), merged into out and lse by the online-softmax rule.  Results are
 * the same up to rounding (pass 1's out is read back in the input dtype).
 *  SA_LINKS_AUTO     two passes when K and V hold 2 GiB or more in total and
 *                    1 GiB or more per (batch, head) slice, and
 *                    at least three such links exist (below that one pass was
 *                    measured faster on B200)
 *  SA_LINKS_SPLIT    two passes whenever such a link exists
 *  SA_LINKS_ONE_PASS never
 * Returns SA_ERR_INVALID_ARG for any other value. */
typedef enum { SA_LINKS_AUTO = 0, SA_LINKS_SPLIT = 1, SA_LINKS_ONE_PASS = 2 } sa_links_mode;
sa_status sparse_attn_set_link_pass(int32_t mode);

/* Synchronise `stream`, then read and clear the library's device error word:
 * SA_ERR_DEVICE_TIMEOUT if a kernel gave up a bounded wait since the last
 * check, SA_ERR_CUDA on a CUDA error, else SA_OK. */
sa_status sparse_attn_check_device(void *stream);

/* Diagnostic for the failure path above (the pages have no counterpart):
 * enqueue on `stream` one warp that waits, with the attention kernels'
 * bounded wait, on a barrier nothing completes, giving up after limit_ns
 * (1 ms .. 2 s, else SA_ERR_INVALID_ARG).  It faults nothing: the next
 * sparse_attn_check_device(stream) returns SA_ERR_DEVICE_TIMEOUT, clears the
 * word, and the context stays usable. */
sa_status sparse_attn_selftest_wait_timeout(int64_t limit_ns, void *stream);

/* Description of the last CUDA failure this thread saw inside the library
 * (the failing call and CUDA's error name and string), "" if none.  The
 * pointer stays valid until the thread's next failing call. */
const char *sparse_attn_last_error_message(void);

/* Number of kernel launches this library has enqueued on the calling host
 * thread's device since process start (for launch accounting). */
int64_t sparse_attn_launch_count(void);

/* Per-kernel timing for benchmarks.  profile_begin(1) makes every later
 * launch of this library record a CUDA event pair on its launch stream;
 * profile_end synchronises the device, stops recording and writes, for each
 * distinct kernel (at most max_kernels), its name (NUL-terminated, at most
 * name_len bytes, into names + k * name_len), its launch count and its total
 * event-timed milliseconds.  Returns the number of distinct kernels, or -1
 * on a CUDA error. */
sa_status sparse_attn_profile_begin(int32_t enable);
int32_t sparse_attn_profile_end(char *names, int32_t name_len, int32_t *launches, double *total_ms,
                                int32_t max_kernels);

#ifdef __cplusplus
}
#endif
#endif /* SPARSE_ATTN_H */
