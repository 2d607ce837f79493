// tmap.cuh -- host-side TMA tensor maps for contiguous [B*H, T, D] bf16
// tensors (3-D: x = D, y = T, z = B*H), 128-byte swizzle, zero fill outside
// the tensor.  cuTensorMapEncodeTiled is fetched from the driver at run time.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

bool sa_tmap_bf16_3d(CUtensorMap *m, const void *base, uint64_t D, uint64_t T, uint64_t BH,
                     uint32_t box_rows);

