// bwd_noalloc.cu -- sparse_attn_bwd_noalloc: the backward without any
// caller workspace.  Its only scratch (Delta_i = dO_i . out_i, fp32, one
// value per query row) lives in a fixed device array defined in this file.
//
// For callers that cannot allocate device memory at the call site: a host
// that runs under a fixed device-memory plan (every byte reserved up front,
// where growing or fragmenting the pool mid-request is not allowed), or code
// that runs inside an allocator hook, where allocating again would re-enter
// the allocator.  Such callers still pass their inputs and outputs.
//
// The array is module-scope: every GPU that loads the library holds
// SA_NOALLOC_MAX_ROWS * 4 bytes of it until the process exits, and every call
// on a device shares it.  Calls whose work overlaps on the GPU race on it.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "sa_internal.cuh"

namespace {

__device__ __align__(256) float g_noalloc_delta[SA_NOALLOC_MAX_ROWS];

constexpr int kMaxDevices = 64;
float *g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of the array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
sa_status noalloc_scratch(float **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_delta) != cudaSuccess || !p) return SA_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<float *>(p);
    }
    *out = g_noalloc_ptr[dev];
    return SA_OK;
}

}  // namespace

extern "C" sa_status sparse_attn_bwd_noalloc(const sa_tensor *q, const sa_tensor *k,
                                             const sa_tensor *v, const sa_tensor *out,
                                             const float *lse, const sa_tensor *dout, sa_graph g,
                                             float scale, sa_tensor *dq, sa_tensor *dk,
                                             sa_tensor *dv, void *stream) {
    if (!q || q->B < 1 || q->H < 1 || q->T < 1) return SA_ERR_INVALID_ARG;
    if (q->B * q->H * q->T > (int64_t)SA_NOALLOC_MAX_ROWS) return SA_ERR_UNSUPPORTED;
    float *scratch = nullptr;
    sa_status st = noalloc_scratch(&scratch);
    if (st != SA_OK) return st;
    // Delta is written in full by the dQ pass before the dK/dV pass reads it,
    // so nothing in the array has to start at zero.  Without room for the
    // distance-edge cache the dK/dV pass recomputes p and dS.
    return sa_bwd_with_scratch(q, k, v, out, lse, dout, g, scale, dq, dk, dv, scratch, nullptr,
                               stream);
}
