// attn_band.cu -- placeholder until the tcgen05 band kernels land.
#include "sa_band.cuh"

bool sa_band_fwd_supported(const sa_tensor *, const sa_graph_s *) { return false; }
bool sa_band_bwd_supported(const sa_tensor *, const sa_graph_s *) { return false; }
sa_status sa_band_fwd(const sa_tensor *, const sa_tensor *, const sa_tensor *, const sa_graph_s *,
                      const GraphView &, float, sa_tensor *, float *, cudaStream_t) {
    return SA_ERR_UNSUPPORTED;
}
sa_status sa_band_bwd(const sa_tensor *, const sa_tensor *, const sa_tensor *, const sa_tensor *,
                      const float *, const sa_tensor *, const sa_graph_s *, const GraphView &, float,
                      sa_tensor *, sa_tensor *, sa_tensor *, float *, cudaStream_t) {
    return SA_ERR_UNSUPPORTED;
}
