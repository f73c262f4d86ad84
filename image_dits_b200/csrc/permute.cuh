// Window permutation of Q/K/V and its inverse ("RainFusion2.0" section 3.3,
// first frame moved to the end per section 3.4).
//
// Both directions are row gathers of d bf16 values (128 or 256 bytes per
// row), HBM-bound.  A warp handles a batch of rows per iteration: each lane
// first computes the closed-form source row of one of them, then the warp
// copies the batch with 16-byte vector loads (all issued before the
// stores), rows fetched by shuffling the source index from the lane that
// computed it.  Loads and stores are marked streaming (each byte is touched
// once).
#pragma once
#include "geometry.cuh"

namespace rf2 {

#ifndef RF2_PERMUTE_ROWS
#define RF2_PERMUTE_ROWS 16
#endif
#ifndef RF2_PERMUTE_MINB
#define RF2_PERMUTE_MINB 4
#endif

// A warp moves kRows rows per iteration: lanes compute the source rows of the
// batch (one each), then every lane loads its 16-byte pieces of all kRows
// rows before storing any.
template <int D, bool kForward>
__global__ void __launch_bounds__(256, RF2_PERMUTE_MINB) permute_rows_kernel(const uint4* __restrict__ in,
                                                                             uint4* __restrict__ out, PermGeo g,
                                                                             int64_t total_rows)
{
    constexpr int C = D / 8;          // 16-byte chunks per row
    constexpr int R = 32 / C;         // rows covered by one warp-wide load
    constexpr int kRows = RF2_PERMUTE_ROWS;
    constexpr int kLoads = kRows / R;
    static_assert(kRows % R == 0 && kRows <= 32, "rows per iteration");
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int cidx = lane % C;
    const int rsub = lane / C;

    for (int64_t row0 = warp * kRows; row0 < total_rows; row0 += nwarps * kRows) {
        int64_t src = 0;
        if (lane < kRows && row0 + lane < total_rows) {
            const int64_t myrow = row0 + lane;
            const int64_t bh = myrow / g.N;
            const int32_t p = (int32_t)(myrow - bh * g.N);
            const int32_t s = kForward ? perm_src(g, p) : perm_dst(g, p);
            src = bh * g.N + s;
            if (RF2_CHECKED && !in_range(s >= 0 && s < g.N)) src = -1;     // checked build: reported, skipped
        }
        uint4 v[kLoads];
        bool ok[kLoads];
        #pragma unroll
        for (int k = 0; k < kLoads; ++k) {
            const int r = k * R + rsub;
            const int64_t srow = __shfl_sync(0xffffffffu, src, r);
            ok[k] = row0 + r < total_rows && (!RF2_CHECKED || srow >= 0);
            if (ok[k]) v[k] = __ldcs(in + srow * C + cidx);
        }
        #pragma unroll
        for (int k = 0; k < kLoads; ++k) {
            const int r = k * R + rsub;
            if (ok[k]) __stcs(out + (row0 + r) * C + cidx, v[k]);
        }
    }
}

}  // namespace rf2
