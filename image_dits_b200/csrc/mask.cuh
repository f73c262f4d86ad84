// Online block-mask prediction ("RainFusion2.0" section 3.2, eqs. (5)-(8), and
// the first-frame sink of section 3.4).
//
// block_mean_kernel   q^_i / k^_j = mean over the valid rows of each 64-token
//                     block (eqs. (5)-(6)).  Blocks are 64 contiguous rows of
//                     the permuted tensors, so this is a segmented reduction
//                     over contiguous memory: one warp per block, 16-byte
//                     loads, fp32 accumulation, HBM-bound.
// select_kernel       S^_ij = q^_i . k^_j / sqrt(d) for R query blocks of one
//                     head against every key block (fp32 FMA from shared
//                     memory, eq. (7)), then per row the n largest scores
//                     (eq. (8)) by a 4-pass 8-bit radix select on
//                     order-preserving uint32 keys (equal scores: lower j),
//                     union the sink columns, and write the row as an
//                     ascending CSR list.  Sink rows keep every column.
#pragma once
#include "geometry.cuh"

namespace rf2 {

__device__ __forceinline__ void bf16x8_accumulate(const uint4 v, float (&acc)[8])
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    #pragma unroll
    for (int k = 0; k < 4; ++k) {
        acc[2 * k] += __uint_as_float(w[k] << 16);
        acc[2 * k + 1] += __uint_as_float(w[k] & 0xffff0000u);
    }
}

// means: [2][BH][Tb][D] fp32 (0 = queries, 1 = keys).
template <int D>
__global__ void __launch_bounds__(256) block_mean_kernel(const uint4* __restrict__ qp,
                                                         const uint4* __restrict__ kp,
                                                         float* __restrict__ means, int32_t N,
                                                         int32_t Tb, int64_t BH)
{
    constexpr int C = D / 8;
    constexpr int R = 32 / C;
    const int lane = threadIdx.x & 31;
    const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t per_tensor = BH * Tb;
    if (w >= 2 * per_tensor) return;
    const int which = (int)(w / per_tensor);
    const int64_t rem = w - which * per_tensor;
    const int64_t bh = rem / Tb;
    const int32_t i = (int32_t)(rem - bh * Tb);
    const int32_t rows = min(kBlock, N - i * kBlock);
    const uint4* src = (which ? kp : qp) + (bh * N + (int64_t)i * kBlock) * C;

    float acc[8];
    #pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.f;
    const int cidx = lane % C;
    const int r0 = lane / C;
    if (rows == kBlock) {
        #pragma unroll 8
        for (int r = r0; r < kBlock; r += R) bf16x8_accumulate(__ldcs(src + r * C + cidx), acc);
    } else {
        for (int r = r0; r < rows; r += R) bf16x8_accumulate(__ldcs(src + r * C + cidx), acc);
    }
    #pragma unroll
    for (int off = C; off < 32; off <<= 1)
        #pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], off);
    if (lane < C) {
        const float fr = (float)rows;
        float4* dst = reinterpret_cast<float4*>(means + ((int64_t)which * per_tensor + rem) * D) + 2 * cidx;
        dst[0] = make_float4(acc[0] / fr, acc[1] / fr, acc[2] / fr, acc[3] / fr);
        dst[1] = make_float4(acc[4] / fr, acc[5] / fr, acc[6] / fr, acc[7] / fr);
    }
}

// Order-preserving map float -> uint32 (larger float, larger key).
__device__ __forceinline__ uint32_t float_order_key(float f)
{
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kSelThreads = 256;
constexpr int kSelKeysPerChunk = 64;

template <int D, int R>
struct SelectSmem {
    static constexpr int KSTRIDE = D + 4;       // padded row of a key-mean chunk (floats)
    static size_t bytes(int Tb)
    {
        return sizeof(float) * (size_t)R * D                                  // query means
             + sizeof(float) * (size_t)kSelKeysPerChunk * KSTRIDE             // key-mean chunk
             + sizeof(uint32_t) * (size_t)R * Tb                              // score keys
             + sizeof(uint32_t) * 256 * (kSelThreads / 32);                   // histograms
    }
};

// Grid: (ceil(Tb / R), BH).  Block: 256 threads.
template <int D, int R>
__global__ void __launch_bounds__(kSelThreads) select_kernel(const float* __restrict__ means,
                                                             int32_t* __restrict__ row_start,
                                                             int32_t* __restrict__ row_count,
                                                             int32_t* __restrict__ col_idx,
                                                             MaskGeo mg, int64_t BH, float inv_sqrt_d)
{
    using SM = SelectSmem<D, R>;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    float* qs = reinterpret_cast<float*>(smem_raw);                       // [R][D]
    float* ks = qs + R * D;                                               // [64][D+4]
    uint32_t* keys = reinterpret_cast<uint32_t*>(ks + kSelKeysPerChunk * SM::KSTRIDE);  // [R][Tb]
    uint32_t* hist_all = keys + (size_t)R * mg.Tb;                        // [8][256]

    const int Tb = mg.Tb;
    const int64_t bh = blockIdx.y;
    const int i0 = blockIdx.x * R;
    const int nrows = min(R, Tb - i0);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const float* qm = means + (bh * Tb) * D;
    const float* km = means + (BH * Tb + bh * Tb) * D;

    // Rows of this tile that need scoring (sink rows keep every column).
    const int n_score_rows = max(0, min(nrows, mg.sink_first - i0));
    const bool keep_all = mg.n_keep >= Tb;

    if (n_score_rows > 0 && !keep_all) {
        for (int e = tid; e < R * D / 4; e += kSelThreads) {
            const int r = (e * 4) / D;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < n_score_rows) v = reinterpret_cast<const float4*>(qm + (int64_t)i0 * D)[e];
            reinterpret_cast<float4*>(qs)[e] = v;
        }
        // Thread layout for scoring: key kk = tid % 64, rows rg*(R/4) .. +R/4.
        constexpr int RPT = R / 4;
        const int kk = tid % kSelKeysPerChunk;
        const int rg = tid / kSelKeysPerChunk;
        for (int j0 = 0; j0 < Tb; j0 += kSelKeysPerChunk) {
            __syncthreads();
            const int nk = min(kSelKeysPerChunk, Tb - j0);
            for (int e = tid; e < kSelKeysPerChunk * D / 4; e += kSelThreads) {
                const int kr = (e * 4) / D;
                const int kc = (e * 4) % D;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (kr < nk) v = reinterpret_cast<const float4*>(km + (int64_t)(j0 + kr) * D)[kc / 4];
                *reinterpret_cast<float4*>(ks + kr * SM::KSTRIDE + kc) = v;
            }
            __syncthreads();
            float acc[RPT];
            #pragma unroll
            for (int r = 0; r < RPT; ++r) acc[r] = 0.f;
            const float* krow = ks + kk * SM::KSTRIDE;
            #pragma unroll 4
            for (int c = 0; c < D; c += 4) {
                const float4 kv = *reinterpret_cast<const float4*>(krow + c);
                #pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const float4 qv = *reinterpret_cast<const float4*>(qs + (rg * RPT + r) * D + c);
                    acc[r] = fmaf(qv.x, kv.x, acc[r]);
                    acc[r] = fmaf(qv.y, kv.y, acc[r]);
                    acc[r] = fmaf(qv.z, kv.z, acc[r]);
                    acc[r] = fmaf(qv.w, kv.w, acc[r]);
                }
            }
            if (kk < nk) {
                #pragma unroll
                for (int r = 0; r < RPT; ++r)
                    keys[(size_t)(rg * RPT + r) * Tb + j0 + kk] = float_order_key(acc[r] * inv_sqrt_d);
            }
        }
        __syncthreads();
    }

    uint32_t* hist = hist_all + warp * 256;
    for (int r = warp; r < nrows; r += kSelThreads / 32) {
        const int i = i0 + r;
        const int64_t rs = row_offset(mg, bh, i);
        const int64_t row_id = bh * Tb + i;
        int32_t* out = col_idx + rs;
        if (i >= mg.sink_first || keep_all) {
            for (int j = lane; j < Tb; j += 32) out[j] = j;
            if (lane == 0) { row_start[row_id] = (int32_t)rs; row_count[row_id] = Tb; }
            continue;
        }
        const uint32_t* rk = keys + (size_t)r * Tb;
        // Radix select of the n-th largest key, 8 bits at a time from the top.
        uint32_t prefix = 0, pmask = 0;
        int remaining = mg.n_keep;
        #pragma unroll 1
        for (int shift = 24; shift >= 0; shift -= 8) {
            #pragma unroll
            for (int b = 0; b < 8; ++b) hist[lane * 8 + b] = 0;
            __syncwarp();
            for (int j = lane; j < Tb; j += 32) {
                const uint32_t k = rk[j];
                if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
            }
            __syncwarp();
            // Lane l owns bins 255-8l .. 248-8l (descending).
            uint32_t cnt[8];
            uint32_t local = 0;
            #pragma unroll
            for (int b = 0; b < 8; ++b) { cnt[b] = hist[255 - (lane * 8 + b)]; local += cnt[b]; }
            uint32_t incl = local;
            #pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            const uint32_t excl = incl - local;
            const bool here = (excl < (uint32_t)remaining) && ((uint32_t)remaining <= incl);
            const uint32_t ballot = __ballot_sync(0xffffffffu, here);
            const int src_lane = __ffs(ballot) - 1;
            uint32_t bin = 0, before = 0;
            if (lane == src_lane) {
                uint32_t run = excl;
                #pragma unroll
                for (int b = 0; b < 8; ++b) {
                    if (run + cnt[b] >= (uint32_t)remaining) { bin = 255 - (lane * 8 + b); before = run; break; }
                    run += cnt[b];
                }
            }
            bin = __shfl_sync(0xffffffffu, bin, src_lane);
            before = __shfl_sync(0xffffffffu, before, src_lane);
            remaining -= (int)before;
            prefix |= bin << shift;
            pmask |= 255u << shift;
            __syncwarp();
        }
        // prefix is the threshold key; `remaining` keys equal to it are kept,
        // the lowest-indexed ones first.
        const uint32_t thr = prefix;
        int eq_left = remaining;
        int written = 0;
        for (int j0 = 0; j0 < Tb; j0 += 32) {
            const int j = j0 + lane;
            const uint32_t k = (j < Tb) ? rk[j] : 0u;
            const bool eq = (j < Tb) && (k == thr);
            const uint32_t eq_ballot = __ballot_sync(0xffffffffu, eq);
            const int eq_rank = __popc(eq_ballot & ((1u << lane) - 1u));
            const bool sel = (j < Tb) && (k > thr || (eq && eq_rank < eq_left) || j >= mg.sink_first);
            eq_left -= __popc(eq_ballot);
            const uint32_t sel_ballot = __ballot_sync(0xffffffffu, sel);
            if (sel) out[written + __popc(sel_ballot & ((1u << lane) - 1u))] = j;
            written += __popc(sel_ballot);
        }
        if (lane == 0) { row_start[row_id] = (int32_t)rs; row_count[row_id] = written; }
    }
}

}  // namespace rf2
