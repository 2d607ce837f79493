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

#include "sa_internal.cuh"

namespace {

__device__ __align__(256) float g_noalloc_delta[SA_NOALLOC_MAX_ROWS];

// Device address of the array in the current context.  In host code the
// array's name is only a host-side stand-in, so the address is looked up
// with the device current.  It is looked up again on every call (cheap once
// the module is loaded) rather than cached, so that a reset device or a
// different context never receives a stale address.
sa_status noalloc_scratch(float **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_delta);
    if (e != cudaSuccess || !p) {
        sa_record_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol,
                             "bwd_noalloc: cudaGetSymbolAddress");
        return SA_ERR_CUDA;
    }
    *out = static_cast<float *>(p);
    return SA_OK;
}

}  // namespace

extern "C" sa_status sparse_attn_bwd_noalloc(const sa_tensor *q, const sa_tensor *k,
                                             const sa_tensor *v, const sa_tensor *out,
                                             const float *lse, const sa_tensor *dout, sa_graph g,
                                             float scale, sa_tensor *dq, sa_tensor *dk,
                                             sa_tensor *dv, void *stream) {
    // every argument is checked first (a bad one is SA_ERR_INVALID_ARG
    // whatever its size), then the size against the array
    sa_status st = sa_bwd_check_args(q, k, v, out, lse, dout, g, scale, dq, dk, dv);
    if (st != SA_OK) return st;
    // rows = B * H * T, compared step by step so that no product overflows
    const int64_t kMax = SA_NOALLOC_MAX_ROWS;
    if (q->B > kMax || q->H > kMax / q->B || q->T > kMax / (q->B * q->H))
        return SA_ERR_UNSUPPORTED;
    float *scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != SA_OK) return st;
    // Delta is written in full by the dQ pass before the dK/dV pass
    // reads it, so nothing in the array has to start at zero.  Without room
    // for the distance-edge cache the dK/dV pass recomputes p and dS.
    return sa_bwd_with_scratch(q, k, v, out, lse, dout, g, scale, dq, dk, dv, scratch, nullptr,
                               stream);
}
