// capi.cu -- the extern "C" entry points of libsparse_attn: argument checks
// on the host, graph handles, and dispatch to the kernels.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "sa_internal.cuh"
#include "sa_band.cuh"
#include "tc_common.cuh"

namespace {

std::atomic<int64_t> g_launches{0};
std::atomic<int> g_path{SA_PATH_AUTO};
std::atomic<int> g_links{SA_LINKS_AUTO};

// One error word per device, written by kernels whose waits are bounded.
__device__ int g_device_error = 0;

cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// One warp waits on an mbarrier that nothing arrives on, through the same
// bounded wait the attention kernels use: after limit_ns it records
// SA_DEVERR_TIMEOUT in the error word and returns.
__global__ void selftest_wait_kernel(int *err, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t mb;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        tc::mbar_init(tc::smem_u32(&mb), 1);
        abort_flag = 0;
        tc::fence_barrier_init();
    }
    __syncthreads();
    tc::mbar_wait(tc::smem_u32(&mb), 0, &abort_flag, err, SA_DEVERR_TIMEOUT, limit_ns);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sa_status check_tensor(const sa_tensor *t, const sa_tensor *ref) {
    if (!t || !t->ptr) return SA_ERR_INVALID_ARG;
    if (!aligned16(t->ptr)) return SA_ERR_INVALID_ARG;
    if (t->dtype != SA_BF16 && t->dtype != SA_FP32) return SA_ERR_INVALID_ARG;
    if (t->B < 1 || t->H < 1 || t->T < 1 || t->D < 1) return SA_ERR_INVALID_ARG;
    if (ref && (t->B != ref->B || t->H != ref->H || t->T != ref->T || t->D != ref->D ||
                t->dtype != ref->dtype))
        return SA_ERR_INVALID_ARG;
    return SA_OK;
}

// k (and v, dk, dv): q's B, T, D and dtype, with a head count that divides
// q's (grouped-query attention: query head h reads key/value head
// h / (H / Hkv)).
sa_status check_kv(const sa_tensor *t, const sa_tensor *q) {
    sa_status st = check_tensor(t, nullptr);
    if (st != SA_OK) return st;
    if (t->B != q->B || t->T != q->T || t->D != q->D || t->dtype != q->dtype)
        return SA_ERR_INVALID_ARG;
    if (q->H % t->H != 0) return SA_ERR_INVALID_ARG;
    return SA_OK;
}

sa_status check_common(const sa_tensor *q, sa_graph g) {
    if (!g) return SA_ERR_INVALID_ARG;
    sa_status st = check_tensor(q, nullptr);
    if (st != SA_OK) return st;
    if (q->T != g->T) return SA_ERR_INVALID_ARG;
    if (q->D != 32 && q->D != 64 && q->D != 128) return SA_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
    if (dev != g->device) return SA_ERR_INVALID_ARG;
    return SA_OK;
}

}  // namespace

void sa_count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

namespace {
thread_local std::string t_last_error;
}

void sa_record_cuda_error(cudaError_t e, const char *where) {
    const char *f = where ? strrchr(where, '/') : nullptr;
    t_last_error = std::string(f ? f + 1 : (where ? where : "?")) + ": " + cudaGetErrorName(e) +
                   " (" + cudaGetErrorString(e) + ")";
}

cudaError_t sa_sm_count(int *n) {
    static std::mutex mu;
    static int cached[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 0 && dev < 64 && cached[dev] > 0) {
        *n = cached[dev];
        return cudaSuccess;
    }
    e = cudaDeviceGetAttribute(n, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess && dev >= 0 && dev < 64) cached[dev] = *n;
    return e;
}

cudaError_t sa_smem_optin(const void *kernel, int bytes) {
    static std::mutex mu;
    static std::vector<std::pair<const void *, int>> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    for (auto &d : done)
        if (d.first == kernel && d.second == dev) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.emplace_back(kernel, dev);
    return e;
}

namespace {
struct ProfRecord {
    const char *name;
    cudaEvent_t a, b;
};
std::atomic<int> g_prof_on{0};
std::vector<ProfRecord> g_prof;
std::mutex g_prof_mu;
thread_local const char *t_prof_name = nullptr;
thread_local cudaEvent_t t_prof_start = nullptr;
}  // namespace

void sa_prof_begin(const char *kernel, cudaStream_t s) {
    if (!g_prof_on.load(std::memory_order_relaxed)) return;
    t_prof_name = kernel;
    if (cudaEventCreate(&t_prof_start) == cudaSuccess) cudaEventRecord(t_prof_start, s);
    else t_prof_start = nullptr;
}

void sa_prof_end(cudaStream_t s) {
    if (!g_prof_on.load(std::memory_order_relaxed) || !t_prof_start) return;
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return;
    cudaEventRecord(e, s);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof.push_back({t_prof_name, t_prof_start, e});
    t_prof_start = nullptr;
}

int *sa_device_error_word() {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    return static_cast<int *>(p);
}

GraphView make_view(const sa_graph_s *g) {
    GraphView v{};
    v.T = g->T;
    v.kind = g->kind;
    v.W = g->W;
    v.n_off = g->n_off;
    for (int a = 0; a < SA_MAX_OFFSETS; ++a) v.offs[a] = a < g->n_off ? g->offs[a] : 0;
    v.rowptr = g->rowptr;
    v.colidx = g->colidx;
    v.rev_rowptr = g->rev_rowptr;
    v.rev_colidx = g->rev_colidx;
    return v;
}

int sa_link_pass_mode() { return g_links.load(); }

extern "C" {

const char *sparse_attn_status_string(sa_status s) {
    switch (s) {
        case SA_OK: return "ok";
        case SA_ERR_INVALID_ARG: return "invalid argument";
        case SA_ERR_INVALID_GRAPH: return "invalid graph";
        case SA_ERR_UNSUPPORTED: return "unsupported";
        case SA_ERR_OOM: return "out of device memory";
        case SA_ERR_CUDA: return "CUDA error";
        case SA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

sa_status sparse_attn_set_path(int32_t path) {
    if (path != SA_PATH_AUTO && path != SA_PATH_GATHER) return SA_ERR_INVALID_ARG;
    g_path.store(path);
    return SA_OK;
}

sa_status sparse_attn_set_link_pass(int32_t mode) {
    if (mode != SA_LINKS_AUTO && mode != SA_LINKS_SPLIT && mode != SA_LINKS_ONE_PASS)
        return SA_ERR_INVALID_ARG;
    g_links.store(mode);
    return SA_OK;
}

int64_t sparse_attn_launch_count(void) { return g_launches.load(); }

const char *sparse_attn_last_error_message(void) { return t_last_error.c_str(); }

sa_status sparse_attn_profile_begin(int32_t enable) {
    g_prof_on.store(enable ? 1 : 0);
    return SA_OK;
}

int32_t sparse_attn_profile_end(char *names, int32_t name_len, int32_t *launches, double *total_ms,
                                int32_t max_kernels) {
    g_prof_on.store(0);
    bool ok = cudaDeviceSynchronize() == cudaSuccess;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    std::vector<std::string> keys;
    std::vector<int32_t> cnt;
    std::vector<double> ms;
    for (auto &r : g_prof) {
        float t = 0.f;
        if (ok && cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) ok = false;
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
        std::string n(r.name ? r.name : "?");
        size_t k = 0;
        while (k < keys.size() && keys[k] != n) ++k;
        if (k == keys.size()) {
            keys.push_back(n);
            cnt.push_back(0);
            ms.push_back(0.0);
        }
        cnt[k] += 1;
        ms[k] += t;
    }
    g_prof.clear();
    if (!ok) return -1;
    int32_t n = (int32_t)std::min<size_t>(keys.size(), (size_t)std::max(max_kernels, 0));
    for (int32_t k = 0; k < n; ++k) {
        if (names && name_len > 0) {
            size_t m = std::min<size_t>(keys[k].size(), (size_t)name_len - 1);
            memcpy(names + (size_t)k * name_len, keys[k].data(), m);
            names[(size_t)k * name_len + m] = 0;
        }
        if (launches) launches[k] = cnt[k];
        if (total_ms) total_ms[k] = ms[k];
    }
    return n;
}

sa_status sparse_attn_selftest_wait_timeout(int64_t limit_ns, void *stream) {
    if (limit_ns < 1000000 || limit_ns > 2000000000) return SA_ERR_INVALID_ARG;
    int *err = sa_device_error_word();
    if (!err) return SA_ERR_CUDA;
    cudaStream_t s = as_stream(stream);
    SA_LAUNCH("selftest_wait", s, selftest_wait_kernel<<<1, 32, 0, s>>>(err, (uint64_t)limit_ns));
    SA_CUDA_TRY(cudaGetLastError());
    return SA_OK;
}

sa_status sparse_attn_check_device(void *stream) {
    cudaStream_t s = as_stream(stream);
    SA_CUDA_TRY(cudaStreamSynchronize(s));
    int h = 0;
    SA_CUDA_TRY(cudaMemcpyFromSymbol(&h, g_device_error, sizeof(int)));
    if (h) {
        int z = 0;
        SA_CUDA_TRY(cudaMemcpyToSymbol(g_device_error, &z, sizeof(int)));
        return (h & SA_DEVERR_TIMEOUT) ? SA_ERR_DEVICE_TIMEOUT : SA_ERR_CUDA;
    }
    return SA_OK;
}

sa_status sparse_attn_graph_build_structured(int64_t T, int32_t W, const int32_t *dil_exps,
                                             int32_t n_dil, int32_t materialize, void *stream,
                                             sa_graph *out) {
    if (!out) return SA_ERR_INVALID_ARG;
    *out = nullptr;
    if (T < 1 || W < 1 || n_dil < 0 || (n_dil > 0 && !dil_exps)) return SA_ERR_INVALID_ARG;
    std::vector<int64_t> offs;
    for (int32_t a = 0; a < n_dil; ++a) {
        int32_t k = dil_exps[a];
        if (k < 0 || k > 62) return SA_ERR_INVALID_ARG;
        int64_t o = (int64_t)1 << k;
        if (o >= W && o < T) offs.push_back(o);  // shorter links lie in the window
    }
    std::sort(offs.begin(), offs.end(), [](int64_t a, int64_t b) { return a > b; });
    offs.erase(std::unique(offs.begin(), offs.end()), offs.end());
    if ((int)offs.size() > SA_MAX_OFFSETS) return SA_ERR_UNSUPPORTED;
    sa_graph_s *g = new (std::nothrow) sa_graph_s();
    if (!g) return SA_ERR_OOM;
    if (cudaGetDevice(&g->device) != cudaSuccess) {
        delete g;
        return SA_ERR_CUDA;
    }
    g->T = T;
    g->kind = 0;
    g->W = (int64_t)W > T ? (int32_t)T : W;
    g->n_off = (int32_t)offs.size();
    for (int a = 0; a < g->n_off; ++a) g->offs[a] = offs[a];
    g->nnz = sg_rowptr(T, g->W, g->n_off, g->offs);
    g->max_resid = g->n_off;
    g->max_resid_rev = g->n_off;
    if (materialize) {
        if (T >= (int64_t)1 << 31 || g->nnz >= (int64_t)1 << 31) {
            delete g;
            return SA_ERR_UNSUPPORTED;
        }
        sa_status st = sa_graph_materialize_structured(g, as_stream(stream));
        if (st != SA_OK) {
            sparse_attn_graph_destroy(g);
            return st;
        }
    }
    *out = g;
    return SA_OK;
}

sa_status sparse_attn_graph_build_csr(int64_t T, const int64_t *rowptr, const int32_t *colidx,
                                      int64_t nnz, int32_t band_hint, void *stream,
                                      sa_graph *out) {
    if (!out) return SA_ERR_INVALID_ARG;
    *out = nullptr;
    if (T < 1 || !rowptr || nnz < 0 || (nnz > 0 && !colidx) || band_hint < 0)
        return SA_ERR_INVALID_ARG;
    if (T >= (int64_t)1 << 31 || nnz >= (int64_t)1 << 31) return SA_ERR_UNSUPPORTED;
    sa_graph_s *g = new (std::nothrow) sa_graph_s();
    if (!g) return SA_ERR_OOM;
    if (cudaGetDevice(&g->device) != cudaSuccess) {
        delete g;
        return SA_ERR_CUDA;
    }
    g->T = T;
    g->kind = 1;
    g->W = (int64_t)band_hint > T ? (int32_t)T : band_hint;
    sa_status st = sa_graph_from_csr(g, rowptr, colidx, nnz, g->W, as_stream(stream));
    if (st != SA_OK) {
        sparse_attn_graph_destroy(g);
        return st;
    }
    *out = g;
    return SA_OK;
}

sa_status sparse_attn_graph_nnz(sa_graph g, int64_t *nnz, int64_t *rev_nnz) {
    if (!g) return SA_ERR_INVALID_ARG;
    if (nnz) *nnz = g->nnz;
    if (rev_nnz) *rev_nnz = g->nnz;
    return SA_OK;
}

sa_status sparse_attn_graph_export(sa_graph g, int64_t *rowptr, int32_t *colidx,
                                   int64_t *rev_rowptr, int32_t *rev_colidx, void *stream) {
    if (!g) return SA_ERR_INVALID_ARG;
    if (!g->materialized) return SA_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    const size_t rp = sizeof(int64_t) * (size_t)(g->T + 1), ci = sizeof(int32_t) * (size_t)g->nnz;
    if (rowptr) SA_CUDA_TRY(cudaMemcpyAsync(rowptr, g->rowptr, rp, cudaMemcpyDeviceToDevice, s));
    if (colidx && ci) SA_CUDA_TRY(cudaMemcpyAsync(colidx, g->colidx, ci, cudaMemcpyDeviceToDevice, s));
    if (rev_rowptr)
        SA_CUDA_TRY(cudaMemcpyAsync(rev_rowptr, g->rev_rowptr, rp, cudaMemcpyDeviceToDevice, s));
    if (rev_colidx && ci)
        SA_CUDA_TRY(cudaMemcpyAsync(rev_colidx, g->rev_colidx, ci, cudaMemcpyDeviceToDevice, s));
    return SA_OK;
}

sa_status sparse_attn_graph_destroy(sa_graph g) {
    if (!g) return SA_ERR_INVALID_ARG;
    cudaError_t e = cudaSuccess;
    if (g->rowptr || g->colidx || g->rev_rowptr || g->rev_colidx) e = cudaDeviceSynchronize();
    if (g->rowptr) cudaFree(g->rowptr);
    if (g->colidx) cudaFree(g->colidx);
    if (g->rev_rowptr) cudaFree(g->rev_rowptr);
    if (g->rev_colidx) cudaFree(g->rev_colidx);
    delete g;
    return e == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

sa_status sparse_attn_fwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v, sa_graph g,
                          float scale, sa_tensor *out, float *lse, void *stream) {
    sa_status st = check_common(q, g);
    if (st != SA_OK) return st;
    if ((st = check_kv(k, q)) != SA_OK || (st = check_tensor(v, k)) != SA_OK ||
        (st = check_tensor(out, q)) != SA_OK)
        return st;
    if (!lse || !aligned16(lse) || !std::isfinite(scale)) return SA_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    const GraphView gv = make_view(g);
    // (the band forward masks through the scale's sign: a zero scale, which
    // makes every kept score 0, takes the gather kernels)
    if (g_path.load() == SA_PATH_AUTO && scale != 0.f && sa_band_fwd_supported(q, g))
        return sa_band_fwd(q, k, v, g, gv, scale, out, lse, s);
    return sa_gather_fwd(q, k, v, gv, scale, out, lse, s);
}

// Workspace layout: Delta (fp32 per query row), then, for a structured graph
// with distance links, the (p, dS) pair of every distance edge (8 bytes per
// link per query row), each part 256-byte aligned.
static size_t delta_bytes(const sa_tensor *q) {
    const size_t n = sizeof(float) * (size_t)(q->B * q->H * q->T);
    return (n + 255) & ~(size_t)255;
}
static size_t edge_cache_bytes(const sa_tensor *q, sa_graph g) {
    if (!g || g->kind != 0 || g->n_off < 1) return 0;
    const size_t n = 2 * sizeof(float) * (size_t)g->n_off * (size_t)(q->B * q->H * q->T);
    return (n + 255) & ~(size_t)255;
}

size_t sparse_attn_bwd_workspace_size(const sa_tensor *q, sa_graph g) {
    if (!q || q->B < 1 || q->H < 1 || q->T < 1) return 0;
    return delta_bytes(q) + edge_cache_bytes(q, g);
}

}  // extern "C"

// C++ linkage: not part of the C ABI.
sa_status sa_bwd_check_args(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                            const sa_tensor *out, const float *lse, const sa_tensor *dout,
                            sa_graph g, float scale, const sa_tensor *dq, const sa_tensor *dk,
                            const sa_tensor *dv) {
    sa_status st = check_common(q, g);
    if (st != SA_OK) return st;
    if ((st = check_kv(k, q)) != SA_OK) return st;
    const sa_tensor *qs[] = {out, dout, dq};
    for (const sa_tensor *t : qs)
        if ((st = check_tensor(t, q)) != SA_OK) return st;
    const sa_tensor *ks[] = {v, dk, dv};
    for (const sa_tensor *t : ks)
        if ((st = check_tensor(t, k)) != SA_OK) return st;
    if (!lse || !aligned16(lse) || !std::isfinite(scale)) return SA_ERR_INVALID_ARG;
    return SA_OK;
}

sa_status sa_bwd_with_scratch(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                              const sa_tensor *out, const float *lse, const sa_tensor *dout,
                              sa_graph g, float scale, sa_tensor *dq, sa_tensor *dk,
                              sa_tensor *dv, float *delta, void *edge_cache, void *stream) {
    sa_status st = sa_bwd_check_args(q, k, v, out, lse, dout, g, scale, dq, dk, dv);
    if (st != SA_OK) return st;
    cudaStream_t s = as_stream(stream);
    const GraphView gv = make_view(g);
    if (g_path.load() == SA_PATH_AUTO && sa_band_bwd_supported(q, k, g))
        return sa_band_bwd(q, k, v, out, lse, dout, g, gv, scale, dq, dk, dv, delta, edge_cache,
                           s);
    return sa_gather_bwd(q, k, v, out, lse, dout, gv, scale, dq, dk, dv, delta, s);
}

extern "C" {

sa_status sparse_attn_bwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                          const sa_tensor *out, const float *lse, const sa_tensor *dout, sa_graph g,
                          float scale, sa_tensor *dq, sa_tensor *dk, sa_tensor *dv,
                          void *workspace, size_t ws_bytes, void *stream) {
    sa_status st = check_common(q, g);
    if (st != SA_OK) return st;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
        ws_bytes < sparse_attn_bwd_workspace_size(q, g))
        return SA_ERR_INVALID_ARG;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    void *edge_cache = edge_cache_bytes(q, g) ? ws + delta_bytes(q) : nullptr;
    return sa_bwd_with_scratch(q, k, v, out, lse, dout, g, scale, dq, dk, dv,
                               reinterpret_cast<float *>(ws), edge_cache, stream);
}

}  // extern "C"

// ------------------------------------------------ learned-coordinate scoring

namespace {

// a, c: fp32 [B, H, T, 3] with v's B, H, T; v: bf16/fp32 [B, H, T, D].
sa_status check_dist(const sa_tensor *a, const sa_tensor *c, const sa_tensor *v, sa_graph g) {
    sa_status st = check_common(v, g);
    if (st != SA_OK) return st;
    if ((st = check_tensor(a, nullptr)) != SA_OK || (st = check_tensor(c, a)) != SA_OK) return st;
    if (a->dtype != SA_FP32 || a->D != 3) return SA_ERR_INVALID_ARG;
    if (a->B != v->B || a->H != v->H || a->T != v->T) return SA_ERR_INVALID_ARG;
    return SA_OK;
}

size_t dist_delta_bytes(const sa_tensor *v) {
    const size_t n = sizeof(float) * (size_t)(v->B * v->H * v->T);
    return (n + 255) & ~(size_t)255;
}

}  // namespace

extern "C" {

sa_status sparse_attn_dist_fwd(const sa_tensor *a, const sa_tensor *c, const sa_tensor *v,
                               sa_graph g, float scale, sa_tensor *out, float *lse,
                               void *stream) {
    sa_status st = check_dist(a, c, v, g);
    if (st != SA_OK) return st;
    if ((st = check_tensor(out, v)) != SA_OK) return st;
    if (!lse || !aligned16(lse) || !std::isfinite(scale)) return SA_ERR_INVALID_ARG;
    return sa_dist_fwd(a, c, v, make_view(g), scale, out, lse, as_stream(stream));
}

size_t sparse_attn_dist_bwd_workspace_size(const sa_tensor *v, sa_graph) {
    if (!v || v->B < 1 || v->H < 1 || v->T < 1) return 0;
    return dist_delta_bytes(v);
}

sa_status sparse_attn_dist_bwd(const sa_tensor *a, const sa_tensor *c, const sa_tensor *v,
                               const sa_tensor *out, const float *lse, const sa_tensor *dout,
                               sa_graph g, float scale, sa_tensor *da, sa_tensor *dc,
                               sa_tensor *dv, void *workspace, size_t ws_bytes, void *stream) {
    sa_status st = check_dist(a, c, v, g);
    if (st != SA_OK) return st;
    if ((st = check_tensor(out, v)) != SA_OK || (st = check_tensor(dout, v)) != SA_OK ||
        (st = check_tensor(dv, v)) != SA_OK || (st = check_tensor(da, a)) != SA_OK ||
        (st = check_tensor(dc, a)) != SA_OK)
        return st;
    if (!lse || !aligned16(lse) || !std::isfinite(scale)) return SA_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
        ws_bytes < dist_delta_bytes(v))
        return SA_ERR_INVALID_ARG;
    return sa_dist_bwd(a, c, v, out, lse, dout, make_view(g), scale, da, dc, dv,
                       static_cast<float *>(workspace), as_stream(stream));
}

}  // extern "C"

// ------------------------------------------------------------------ decode

extern "C" sa_status sparse_attn_decode(const sa_tensor *q, const sa_tensor *k_cache,
                                        const sa_tensor *v_cache, const int64_t *pos,
                                        sa_graph g, float scale, sa_tensor *out, float *lse,
                                        void *stream) {
    if (!g) return SA_ERR_INVALID_ARG;
    sa_status st = check_tensor(q, nullptr);
    if (st != SA_OK) return st;
    if ((st = check_tensor(k_cache, nullptr)) != SA_OK ||
        (st = check_tensor(v_cache, k_cache)) != SA_OK || (st = check_tensor(out, q)) != SA_OK)
        return st;
    if (q->T != 1) return SA_ERR_INVALID_ARG;
    if (k_cache->B != q->B || k_cache->D != q->D || k_cache->dtype != q->dtype)
        return SA_ERR_INVALID_ARG;
    if (q->H % k_cache->H != 0) return SA_ERR_INVALID_ARG;
    if (k_cache->T > g->T) return SA_ERR_INVALID_ARG;
    if (q->D != 32 && q->D != 64 && q->D != 128) return SA_ERR_UNSUPPORTED;
    if (!pos || (reinterpret_cast<uintptr_t>(pos) & 7u) != 0) return SA_ERR_INVALID_ARG;
    if (!lse || !aligned16(lse) || !std::isfinite(scale)) return SA_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
    if (dev != g->device) return SA_ERR_INVALID_ARG;
    return sa_decode(q, k_cache, v_cache, pos, make_view(g), scale, out, lse, as_stream(stream));
}
