// sa_rows.cuh -- the per-warp loader of "diagonal" slots shared by the three
// tcgen05 band kernels.
//
// A diagonal slot of a 128-row tile holds one gathered row pair (K and V in
// the forward and dQ passes, Q and dO in the dK/dV pass) for every tile row:
// row r of the slot is the neighbour, in that slot, of the tile's row r (a
// distance link, or one entry of a CSR list).  Each of the four compute warps
// of a pipeline owns 32 tile rows and copies its own rows with 16-byte
// cp.async copies into a DS-stage ring in shared memory, in the 128-byte
// swizzled layout TMA writes (64-column halves), so that thread r can read its
// row with the same addressing as a TMA-loaded tile.  No other role takes
// part and no mbarrier is involved: the warps of a pipeline progress
// independently, each keeping DS slots of copies in flight.
//
// Row indices are read QA slots ahead of their copies through a register
// queue, so that no copy waits on an index load; optionally each slot is also
// prefetched into L2 one iteration after its index load (DS + QA - 1 slots
// ahead of its use), for rows that miss L2.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "tc_common.cuh"

namespace rows {

constexpr int kQA = 4;  // index loads run this many slots ahead of their copies

// Run the diagonal slots 0 .. nd-1 of the calling warp.
//   ring_a, ring_b: shared addresses of stage 0 of the two row rings (each
//                   stage a 128-row tile of D bf16 columns, `stage_bytes` apart)
//   src_a, src_b:   the two source tensors
//   slot_base(d):   element offset of slot d's source slice (warp-uniform)
//   key_of(d):      this lane's tile row's source row for slot d, -1 if none
//                   (d may exceed nd - 1: return -1 then)
//   body(d, st):    the compute of slot d on stage st (every lane's copies of
//                   slot d have landed)
// All 32 lanes must call it with the same nd.
template <int D, int DS, typename SlotBase, typename KeyOf, typename Body>
__device__ __forceinline__ void warp_slots(int nd, uint32_t ring_a, uint32_t ring_b,
                                           uint32_t stage_bytes, const __nv_bfloat16 *src_a,
                                           const __nv_bfloat16 *src_b, bool l2_prefetch,
                                           int lane, int wq, SlotBase slot_base, KeyOf key_of,
                                           Body body) {
    constexpr int CPR = D / 8, RPI = 32 / CPR;  // 16-byte chunks per row, rows per instruction
    const int cl = lane % CPR, xl = lane / CPR;
    auto issue = [&](int st, int d, int32_t key) {
        const uint32_t da = ring_a + (uint32_t)st * stage_bytes;
        const uint32_t db = ring_b + (uint32_t)st * stage_bytes;
        const size_t base = (size_t)slot_base(d) + (size_t)(cl * 8);
#pragma unroll
        for (int it = 0; it < CPR; ++it) {
            const int x = it * RPI + xl;
            const int32_t kx = __shfl_sync(0xffffffffu, key, x);
            if (kx >= 0) {
                const uint32_t off = (uint32_t)((cl >> 3) * (128 * 128)) +
                                     tc::sw128_off((uint32_t)(32 * wq + x), (uint32_t)(cl & 7));
                const size_t src = base + (size_t)kx * D;
                tc::cp_async16(da + off, src_a + src);
                tc::cp_async16(db + off, src_b + src);
            }
        }
        tc::cp_async_commit();
    };
    auto prefetch = [&](int d, int32_t key) {
        if (key >= 0) {
            const size_t src = (size_t)slot_base(d) + (size_t)key * D;
#pragma unroll
            for (int x = 0; x < (D + 63) / 64; ++x) {
                tc::prefetch_l2(src_a + src + 64 * x);
                tc::prefetch_l2(src_b + src + 64 * x);
            }
        }
    };
#pragma unroll
    for (int s = 0; s < DS; ++s) issue(s, s, key_of(s));
    int32_t kq[kQA];  // kq[x]: key of slot d + DS + x at iteration d
#pragma unroll
    for (int s = 0; s < kQA; ++s) kq[s] = key_of(DS + s);
    if (l2_prefetch) {
#pragma unroll
        for (int s = 0; s < kQA - 1; ++s) prefetch(DS + s, kq[s]);
    }
    for (int d = 0; d < nd; ++d) {
        const int st = d % DS;
        if (l2_prefetch) prefetch(d + DS + kQA - 1, kq[kQA - 1]);
        tc::cp_async_wait<DS - 1>();  // slot d has landed (this lane's copies)
        __syncwarp();                 // ... and every lane's
        body(d, st);
        __syncwarp();                 // every lane is done with the stage: refill it
        issue(st, d + DS, kq[0]);
#pragma unroll
        for (int s = 0; s < kQA - 1; ++s) kq[s] = kq[s + 1];
        kq[kQA - 1] = key_of(d + DS + kQA);
    }
    tc::cp_async_wait<0>();  // nothing stays in flight past the slots
}

}  // namespace rows
