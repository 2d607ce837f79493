// sa_band.cuh -- the tcgen05 band-tile path (window edges on tensor cores,
// the remaining edges gathered in the same kernel).
#pragma once
#include "sa_internal.cuh"

bool sa_band_fwd_supported(const sa_tensor *q, const sa_graph_s *g);
bool sa_band_bwd_supported(const sa_tensor *q, const sa_tensor *k, const sa_graph_s *g);
sa_status sa_band_fwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                      const sa_graph_s *g, const GraphView &gv, float scale, sa_tensor *out,
                      float *lse, cudaStream_t s);
sa_status sa_band_bwd(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                      const sa_tensor *out, const float *lse, const sa_tensor *dout,
                      const sa_graph_s *g, const GraphView &gv, float scale, sa_tensor *dq,
                      sa_tensor *dk, sa_tensor *dv, float *delta, void *pds, cudaStream_t s);
// The long distance links of a structured graph as a second forward pass over
// (out, lse) (attn_links.cu): offs (descending) are multiples of `span` rows.
sa_status sa_link_pass(const sa_tensor *q, const sa_tensor *k, const sa_tensor *v,
                       const int64_t *offs, int n_off, int64_t span, float scale, sa_tensor *out,
                       float *lse, cudaStream_t s);
