// Window permutation of Q/K/V and its inverse ("RainFusion2.0" section 3.3,
// first frame moved to the end per section 3.4).
//
// Both directions are row gathers of d bf16 values (128 or 256 bytes per
// row), HBM-bound.  A warp handles 32 rows per iteration: each lane first
// computes the closed-form source row of one of those rows, then the warp
// copies the 32 rows with 16-byte vector loads (all issued before the
// stores, 8 KB in flight per warp for d = 128), rows fetched by shuffling the
// source index from the lane that computed it.
#pragma once
#include "geometry.cuh"

namespace rf2 {

template <int D, bool kForward>
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4* __restrict__ in,
                                                           uint4* __restrict__ out, PermGeo g,
                                                           int64_t total_rows)
{
    constexpr int C = D / 8;          // 16-byte chunks per row
    constexpr int R = 32 / C;         // rows covered by one warp-wide load
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int cidx = lane % C;
    const int rsub = lane / C;

    for (int64_t row0 = warp * 32; row0 < total_rows; row0 += nwarps * 32) {
        const int64_t myrow = row0 + lane;
        int64_t src = 0;
        if (myrow < total_rows) {
            const int64_t bh = myrow / g.N;
            const int32_t p = (int32_t)(myrow - bh * g.N);
            const int32_t s = kForward ? perm_src(g, p) : perm_dst(g, p);
            src = bh * g.N + s;
        }
        uint4 v[C];
        #pragma unroll
        for (int k = 0; k < C; ++k) {
            const int r = k * R + rsub;
            const int64_t srow = __shfl_sync(0xffffffffu, src, r);
            if (row0 + r < total_rows) v[k] = __ldcs(in + srow * C + cidx);
        }
        #pragma unroll
        for (int k = 0; k < C; ++k) {
            const int r = k * R + rsub;
            if (row0 + r < total_rows) out[(row0 + r) * C + cidx] = v[k];
        }
    }
}

}  // namespace rf2
