// Online block-mask prediction ("RainFusion2.0" section 3.2, eqs. (5)-(8), and
// the first-frame sink of section 3.4).
//
// block_mean_kernel   q^_i / k^_j = mean over the valid rows of each 64-token
//                     block (eqs. (5)-(6)).  Blocks are 64 contiguous rows of
//                     the permuted tensors, so this is a segmented reduction
//                     over contiguous memory: one warp per block, 16-byte
//                     loads, fp32 accumulation, HBM-bound.
// score_tc_kernel     S^_ij = q^_i . k^_j / sqrt(d) (eq. (7)) for a group of
//                     heads on the tensor cores (tcgen05 kind::tf32, three
//                     hi/lo products for fp32 accuracy), into a score buffer
//                     that stays in L2 between the two kernels.
// select_from_scores_kernel
//                     per row the n largest scores (eq. (8)) by a 4-pass
//                     8-bit radix select on order-preserving uint32 keys
//                     (equal scores: lower j), union the sink columns, and
//                     write the row as an ascending CSR list.  Sink rows keep
//                     every column.
// select_probe_kernel the same selection with the row's keys in registers
//                     (a few counting probes, then an exact rank of the last
//                     <= 32 candidates), used for rows of up to 512 key blocks.
// select_cdf_kernel   the CDF-threshold alternative to top-n (see below).
#pragma once
#include "geometry.cuh"
#include "ptx.cuh"

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

// Output: the block means as a tf32 split, hi = tf32(mean) (low 13 mantissa
// bits zero) and lo = mean - hi, each [2][BH][Tb][D] fp32 (0 = queries,
// 1 = keys), ready for the tensor-core score kernel.
template <int D>
__global__ void __launch_bounds__(256) block_mean_kernel(const uint4* __restrict__ qp,
                                                         const uint4* __restrict__ kp,
                                                         float* __restrict__ means_hi, float* __restrict__ means_lo,
                                                         int32_t N, int32_t Tb, int64_t BH)
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
        const int64_t at = ((int64_t)which * per_tensor + rem) * D + 8 * cidx;
        float m[8], h[8];
        #pragma unroll
        for (int k = 0; k < 8; ++k) { m[k] = acc[k] / fr; h[k] = to_tf32(m[k]); }
        float4* dh = reinterpret_cast<float4*>(means_hi + at);
        float4* dl = reinterpret_cast<float4*>(means_lo + at);
        dh[0] = make_float4(h[0], h[1], h[2], h[3]);
        dh[1] = make_float4(h[4], h[5], h[6], h[7]);
        dl[0] = make_float4(m[0] - h[0], m[1] - h[1], m[2] - h[2], m[3] - h[3]);
        dl[1] = make_float4(m[4] - h[4], m[5] - h[5], m[6] - h[6], m[7] - h[7]);
    }
}

// Permutation of Q and K fused with the block means (the "permute + pooling"
// step): warp w takes 64-row blocks of the permuted output of both tensors
// (blocks 0 .. BH*Tb-1 of Q, then those of K), copies each block's rows in
// batches of 16 rows (8 at d = 128) as permute_rows_kernel does, and
// accumulates the block's column sums in registers in the same row order as
// block_mean_kernel, so the means (and the masks predicted from them) are
// bit-identical to the unfused path.  Saves re-reading Qp and Kp.
#ifndef RF2_POOL_SUB
#define RF2_POOL_SUB 8
#endif
#ifndef RF2_POOL_MINB
#define RF2_POOL_MINB 4
#endif

template <int D>
__global__ void __launch_bounds__(256, D == 128 ? RF2_POOL_MINB : 4) permute_pool_kernel(
    const uint4* __restrict__ q, const uint4* __restrict__ k, uint4* __restrict__ qp, uint4* __restrict__ kp,
    PermGeo g, int32_t Tb, int64_t BH, float* __restrict__ means_hi, float* __restrict__ means_lo)
{
    constexpr int C = D / 8;          // 16-byte chunks per row
    constexpr int R = 32 / C;         // rows covered by one warp-wide load
    constexpr int kSub = D == 128 ? RF2_POOL_SUB : 16;   // rows per batch
    constexpr int kLoads = kSub / R;
    static_assert(kBlock % kSub == 0 && kSub % R == 0 && kSub <= 32, "rows per batch");
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int cidx = lane % C;
    const int rsub = lane / C;
    const int64_t per_tensor = BH * Tb;
    const int32_t N = g.N;
    for (int64_t blk = warp; blk < 2 * per_tensor; blk += nwarps) {
        const int which = (int)(blk / per_tensor);
        const int64_t rem = blk - which * per_tensor;
        const int64_t bh = rem / Tb;
        const int32_t i = (int32_t)(rem - bh * Tb);
        const uint4* in = (which ? k : q) + bh * N * C + cidx;
        uint4* out = (which ? kp : qp) + (bh * N + (int64_t)i * kBlock) * C + cidx;
        const int32_t rows = min(kBlock, N - i * kBlock);
        float acc[8];
        #pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = 0.f;
        #pragma unroll 1
        for (int r0 = 0; r0 < rows; r0 += kSub) {
            int32_t src = 0;
            if (lane < kSub && r0 + lane < rows) {
                src = perm_src(g, i * kBlock + r0 + lane);
                if (RF2_CHECKED && !in_range(src >= 0 && src < N)) src = -1;   // checked build: reported, skipped
            }
            uint4 v[kLoads];
            bool ok[kLoads];
            #pragma unroll
            for (int u = 0; u < kLoads; ++u) {
                const int r = u * R + rsub;
                const int32_t srow = __shfl_sync(0xffffffffu, src, r);
                ok[u] = r0 + r < rows && (!RF2_CHECKED || srow >= 0);
                if (ok[u]) v[u] = __ldcs(in + (int64_t)srow * C);
            }
            #pragma unroll
            for (int u = 0; u < kLoads; ++u) {
                const int r = r0 + u * R + rsub;
                if (ok[u]) {
                    __stcs(out + r * C, v[u]);
                    bf16x8_accumulate(v[u], acc);
                }
            }
        }
        #pragma unroll
        for (int off = C; off < 32; off <<= 1)
            #pragma unroll
            for (int c = 0; c < 8; ++c) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], off);
        if (lane < C) {
            const float fr = (float)rows;
            const int64_t at = ((int64_t)which * per_tensor + rem) * D + 8 * cidx;
            float m[8], h[8];
            #pragma unroll
            for (int c = 0; c < 8; ++c) { m[c] = acc[c] / fr; h[c] = to_tf32(m[c]); }
            float4* dh = reinterpret_cast<float4*>(means_hi + at);
            float4* dl = reinterpret_cast<float4*>(means_lo + at);
            dh[0] = make_float4(h[0], h[1], h[2], h[3]);
            dh[1] = make_float4(h[4], h[5], h[6], h[7]);
            dl[0] = make_float4(m[0] - h[0], m[1] - h[1], m[2] - h[2], m[3] - h[3]);
            dl[1] = make_float4(m[4] - h[4], m[5] - h[5], m[6] - h[6], m[7] - h[7]);
        }
    }
}

// Order-preserving map float -> uint32 (larger float, larger key).
__device__ __forceinline__ uint32_t float_order_key(float f)
{
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kSelThreads = 256;

// The r-th largest (1 <= r <= cnt) of keys[0..cnt), all of which share the
// high bits common to kmin and kmax (bounds of the keys, not necessarily
// attained), by one warp: 8-bit radix digits from just below those common
// bits (hist: 256 words of this warp's shared memory).  Returns the key;
// `remaining` receives how many keys equal to it are among the r largest.
__device__ __forceinline__ uint32_t radix_kth(const uint32_t* keys, int cnt, int r, uint32_t kmin, uint32_t kmax,
                                              uint32_t* hist, int lane, int& remaining)
{
    const int common = __clz(kmin ^ kmax);                  // 32 when kmin == kmax
    uint32_t pmask = (common >= 32) ? 0xffffffffu : ~(0xffffffffu >> common);
    uint32_t prefix = kmax & pmask;
    remaining = r;
    const int top = 32 - common;                            // undetermined low bits
    #pragma unroll 1
    for (int lo = top - 8; lo > -8; lo -= 8) {
        const int shift = (lo < 0) ? 0 : lo;                // the last digit may overlap fixed bits

        #pragma unroll
        for (int b = 0; b < 8; ++b) hist[lane * 8 + b] = 0;
        __syncwarp();
        // Lanes hitting the same bin add once (the scores of a row are
        // concentrated, so a warp's 32 keys often share one or two bins).
        for (int j0 = 0; j0 < cnt; j0 += 32) {
            const int j = j0 + lane;
            const uint32_t k = (j < cnt) ? keys[j] : 0u;
            const bool hit = (j < cnt) && ((k & pmask) == prefix);
            const uint32_t bin = hit ? ((k >> shift) & 255u) : 256u;
            const uint32_t peers = __match_any_sync(0xffffffffu, bin);
            if (hit && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
        }
        __syncwarp();
        // Lane l owns bins 255-8l .. 248-8l (descending).
        uint32_t cnt8[8];
        uint32_t local = 0;
        #pragma unroll
        for (int b = 0; b < 8; ++b) { cnt8[b] = hist[255 - (lane * 8 + b)]; local += cnt8[b]; }
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
                if (run + cnt8[b] >= (uint32_t)remaining) { bin = 255 - (lane * 8 + b); before = run; break; }
                run += cnt8[b];
            }
        }
        bin = __shfl_sync(0xffffffffu, bin, src_lane);
        before = __shfl_sync(0xffffffffu, before, src_lane);
        remaining -= (int)before;
        prefix |= bin << shift;
        pmask |= 255u << shift;
        __syncwarp();
    }
    return prefix;
}

// Writes row i: the keys above thr, the lowest-indexed `eq_left` keys equal to
// it, and every sink column, in ascending order at the row's closed-form offset.
__device__ __forceinline__ void write_row(const uint32_t* rk, const MaskGeo& mg, int64_t bh, int i, int lane,
                                          uint32_t thr, int eq_left, int32_t* row_start, int32_t* row_count,
                                          int32_t* col_idx)
{
    const int Tb = mg.Tb;
    const int64_t rs = row_offset(mg, bh, i);
    const int64_t row_id = bh * Tb + i;
    int32_t* out = col_idx + rs;
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
        if (sel) csr_put(out, written + __popc(sel_ballot & ((1u << lane) - 1u)), j, rs, mg.col_capacity);
        written += __popc(sel_ballot);
    }
    if (lane == 0) { row_start[row_id] = (int32_t)rs; row_count[row_id] = written; }
}

// Selection of one non-sink or sink row i of head bh from its T_b score keys
// (order-preserving uint32), by one warp: the n-th largest key by radix_kth
// over the whole row (its digits start below the bits common to the row's
// min and max key), then write_row.  Sink rows (and keep = 1) keep every
// column.
__device__ __forceinline__ void select_row(const uint32_t* rk, uint32_t* hist, const MaskGeo& mg, int64_t bh, int i,
                                           int lane, int32_t* row_start, int32_t* row_count, int32_t* col_idx,
                                           bool keep_all)
{
    const int Tb = mg.Tb;
    if (i >= mg.sink_first || keep_all) {
        const int64_t rs = row_offset(mg, bh, i);
        const int64_t row_id = bh * Tb + i;
        int32_t* out = col_idx + rs;
        for (int j = lane; j < Tb; j += 32) csr_put(out, j, j, rs, mg.col_capacity);
        if (lane == 0) { row_start[row_id] = (int32_t)rs; row_count[row_id] = Tb; }
        return;
    }
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int j = lane; j < Tb; j += 32) { const uint32_t k = rk[j]; kmin = min(kmin, k); kmax = max(kmax, k); }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    int remaining;
    const uint32_t thr = radix_kth(rk, Tb, mg.n_keep, kmin, kmax, hist, lane, remaining);
    write_row(rk, mg, bh, i, lane, thr, remaining, row_start, row_count, col_idx);
}

#ifndef RF2_SELECT_SAMPLED
#define RF2_SELECT_SAMPLED 1
#endif
constexpr int kSelCand = 512;                               // candidate keys per warp (words)

// Top-n of a long row from a sample (same threshold and ties as select_row):
// 64 keys, one from each of 64 equal stripes of the row, are sorted (warp bitonic sort, two per
// lane); the n-th largest key is bracketed between the sample keys ranked
// pos - 8 and pos + 8 (pos = its expected rank in the sample: about 2.5
// standard deviations of a sample quantile either side); one pass counts the
// keys above the bracket and gathers the keys inside it, and radix_kth ranks
// the gathered keys.  When the bracket misses the n-th key or holds more than
// kSelCand keys, the row goes through select_row.
__device__ __forceinline__ void select_row_sampled(const uint32_t* rk, uint32_t* hist, uint32_t* cand,
                                                   const MaskGeo& mg, int64_t bh, int i, int lane,
                                                   int32_t* row_start, int32_t* row_count, int32_t* col_idx,
                                                   bool keep_all)
{
    const int Tb = mg.Tb, n = mg.n_keep;
    if (i >= mg.sink_first || keep_all || Tb < 256) {
        select_row(rk, hist, mg, bh, i, lane, row_start, row_count, col_idx, keep_all);
        return;
    }
    // sample e = 2*lane + s: one position in stripe e of the row's 64 equal
    // stripes, at an offset drawn from (row, e) (stratified sampling: a fixed
    // stride follows the scores' smooth structure and biases the quantile);
    // then sorted descending in e
    auto pick = [&](int e) -> int {
        const int s0 = (e * Tb) >> 6, s1 = ((e + 1) * Tb) >> 6;          // stripe [s0, s1), s1 > s0
        const uint32_t h = (uint32_t)(i * 0x9E3779B1u) ^ (uint32_t)(e * 0x85EBCA77u);
        return s0 + (int)((h ^ (h >> 15)) % (uint32_t)(s1 - s0));
    };
    uint32_t v0 = rk[pick(2 * lane)], v1 = rk[pick(2 * lane + 1)];
    #pragma unroll
    for (int k = 2; k <= 64; k <<= 1) {
        #pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const bool desc = ((2 * lane) & k) == 0;          // same for both elements of the lane
            if (j == 1) {
                const uint32_t a = max(v0, v1), b = min(v0, v1);
                v0 = desc ? a : b;
                v1 = desc ? b : a;
            } else {
                const uint32_t o0 = __shfl_xor_sync(0xffffffffu, v0, j >> 1);
                const uint32_t o1 = __shfl_xor_sync(0xffffffffu, v1, j >> 1);
                const bool keep_max = (((2 * lane) & j) == 0) == desc;
                v0 = keep_max ? max(v0, o0) : min(v0, o0);
                v1 = keep_max ? max(v1, o1) : min(v1, o1);
            }
        }
    }
    auto sample_at = [&](int e) -> uint32_t {
        const uint32_t a = __shfl_sync(0xffffffffu, v0, e >> 1);
        const uint32_t b = __shfl_sync(0xffffffffu, v1, e >> 1);
        return (e & 1) ? b : a;
    };
    const int pos = (int)(((int64_t)n * 64) / Tb);
    const uint32_t hi = sample_at(max(0, pos - 8));
    const uint32_t lo = sample_at(min(63, pos + 8));       // lo <= hi
    int c_gt = 0, c_in = 0;
    for (int j0 = 0; j0 < Tb; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t k = (j < Tb) ? rk[j] : 0u;
        const bool gt = (j < Tb) && k > hi;
        const bool in = (j < Tb) && k <= hi && k >= lo;
        const uint32_t bi = __ballot_sync(0xffffffffu, in);
        const int at = c_in + __popc(bi & ((1u << lane) - 1u));
        if (in && at < kSelCand) cand[at] = k;
        c_gt += __popc(__ballot_sync(0xffffffffu, gt));
        c_in += __popc(bi);
    }
    __syncwarp();
    if (!(c_gt < n && n <= c_gt + c_in && c_in <= kSelCand)) {
        select_row(rk, hist, mg, bh, i, lane, row_start, row_count, col_idx, keep_all);
        return;
    }
    int remaining;
    const uint32_t thr = radix_kth(cand, c_in, n - c_gt, lo, hi, hist, lane, remaining);
    write_row(rk, mg, bh, i, lane, thr, remaining, row_start, row_count, col_idx);
    __syncwarp();
}

// ------------------------------------------------------------------------
// Pooled scores on the tensor cores (eq. (7)): S^ = q^ k^T / sqrt(d) for a
// group of heads, as tcgen05 kind::tf32 products of the hi/lo split written
// by block_mean_kernel: q.k = hi.hi + hi.lo + lo.hi, leaving about 2^-21
// |q||k| of error, far inside the 1e-5 tie band of the selection.
// Work item = (head, 128 query blocks); persistent CTAs take items i,
// i + gridDim.x, ...  An item walks its key blocks in chunks of 256 (one
// M128 x N256 accumulator) and d in slices of 32; each stage holds the query
// slice (hi, lo) and the key slice (hi, lo).
// Roles (256 threads): warps 0 and 1 issue the TMA loads (hi and lo parts:
// one thread's TMA stream is served serially); warp 2 issues the MMAs into
// one of two 256-column TMEM accumulators; warps 4-7 move a finished
// accumulator to S^ in global memory, scaled by 1/sqrt(d), while the next
// chunk is multiplied.
template <int D>
struct ScoreCfg {
    static constexpr int KC = D / 32;                  // 32-float (128-byte) slices of d
    static constexpr int NCH = 256;                    // keys per accumulator
    static constexpr uint32_t A_TILE = 128 * 128;      // 128 rows x 32 floats
    static constexpr uint32_t B_TILE = NCH * 128;      // 256 rows x 32 floats
    static constexpr uint32_t STAGE = 2 * A_TILE + 2 * B_TILE;   // [A hi][A lo][B hi][B lo]
    static constexpr uint32_t SMEM = 1024 + 2 * STAGE + 128;
    static constexpr int THREADS = 256;
};

template <int D>
__global__ void __launch_bounds__(ScoreCfg<D>::THREADS, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo,
                const __grid_constant__ CUtensorMap tm_hi_b, const __grid_constant__ CUtensorMap tm_lo_b,
                float* __restrict__ S, int32_t Tb, int32_t ld_s, int64_t BH, int64_t h0, int32_t G,
                float inv_sqrt_d, int* status)
{
    using Cfg = ScoreCfg<D>;
    constexpr int KC = Cfg::KC;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_u32 - raw_u32);
    // barriers: full[2], empty[2], acc_full[2], acc_empty[2], drain
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + 2 * Cfg::STAGE);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9);
    int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
    uint64_t* full = bars;
    uint64_t* empty = bars + 2;
    uint64_t* acc_full = bars + 4;
    uint64_t* acc_empty = bars + 6;
    uint64_t* drain = bars + 8;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int mtiles = (Tb + 127) / 128;
    const int nchunks = (Tb + Cfg::NCH - 1) / Cfg::NCH;
    const int items = G * mtiles;
    const int my_items = (blockIdx.x < items) ? (items - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&full[i]), 2);                 // hi and lo producers
            mbar_init(smem_u32(&empty[i]), 1);
            mbar_init(smem_u32(&acc_full[i]), 1);
            mbar_init(smem_u32(&acc_empty[i]), 128);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    volatile int* abort = abort_flag;

    if (warp == 0 || warp == 1) {
        if (lane == 0) {
            // warp 0: hi parts, warp 1: lo parts.  Rows of the block-mean maps:
            // queries of all heads first, then keys.
            const CUtensorMap* ta = (warp == 0) ? &tm_hi : &tm_lo;
            const CUtensorMap* tb = (warp == 0) ? &tm_hi_b : &tm_lo_b;
            int step = 0;
            int issued[2] = {-1, -1};
            bool ok = true;
            for (int it = 0; ok && it < my_items; ++it) {
                const int item = blockIdx.x + it * gridDim.x;
                const int64_t bh = h0 + item / mtiles;
                const int m0 = (item % mtiles) * 128;
                const int qrow = (int)(bh * Tb) + m0;
                const int krow0 = (int)(BH * Tb + bh * Tb);
                for (int n = 0; ok && n < nchunks; ++n)
                    for (int c = 0; c < KC; ++c, ++step) {
                        const int b = step & 1;
                        const int use = step >> 1;
                        if (use > 0 && !mbar_wait(smem_u32(&empty[b]), (use - 1) & 1, abort, status)) { ok = false; break; }
                        const uint32_t st = base_u32 + b * Cfg::STAGE;
                        mbar_arrive_expect_tx(smem_u32(&full[b]), Cfg::A_TILE + Cfg::B_TILE);
                        tma_load_2d(st + warp * Cfg::A_TILE, ta, smem_u32(&full[b]), c * 32, qrow);
                        tma_load_2d(st + 2 * Cfg::A_TILE + warp * Cfg::B_TILE, tb, smem_u32(&full[b]), c * 32,
                                    krow0 + n * Cfg::NCH);
                        issued[b] = use;
                    }
            }
            for (int b = 0; b < 2; ++b)
                if (issued[b] >= 0) mbar_wait_drain(smem_u32(&full[b]), issued[b] & 1);
        }
    } else if (warp == 2) {
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_tf32_f32(128, Cfg::NCH);
            int step = 0, chunk = 0;
            bool ok = true;
            for (int it = 0; ok && it < my_items; ++it)
                for (int n = 0; ok && n < nchunks; ++n, ++chunk) {
                    const int a = chunk & 1;
                    if (chunk >= 2 && !mbar_wait(smem_u32(&acc_empty[a]), ((chunk >> 1) - 1) & 1, abort, status)) { ok = false; break; }
                    const uint32_t d_tmem = tmem + Cfg::NCH * a;
                    for (int c = 0; c < KC; ++c, ++step) {
                        const int b = step & 1;
                        if (!mbar_wait(smem_u32(&full[b]), (step >> 1) & 1, abort, status)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t st = base_u32 + b * Cfg::STAGE;
                        const uint32_t a_hi = st, a_lo = st + Cfg::A_TILE;
                        const uint32_t b_hi = st + 2 * Cfg::A_TILE, b_lo = b_hi + Cfg::B_TILE;
                        #pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {              // 8 floats = 32 bytes per K step
                            const uint32_t off = ks * 32;
                            const uint32_t first = (c == 0 && ks == 0) ? 0u : 1u;
                            mma_ss_tf32(d_tmem, smem_desc_sw128(a_hi + off, 16, 1024), smem_desc_sw128(b_hi + off, 16, 1024), IDESC, first);
                            mma_ss_tf32(d_tmem, smem_desc_sw128(a_hi + off, 16, 1024), smem_desc_sw128(b_lo + off, 16, 1024), IDESC, 1u);
                            mma_ss_tf32(d_tmem, smem_desc_sw128(a_lo + off, 16, 1024), smem_desc_sw128(b_hi + off, 16, 1024), IDESC, 1u);
                        }
                        mma_commit(smem_u32(&empty[b]));
                    }
                    if (ok) mma_commit(smem_u32(&acc_full[a]));
                }
            mma_commit(smem_u32(drain));
            mbar_wait_drain(smem_u32(drain), 0);
        }
    } else if (warp >= 4) {
        // epilogue warps 4-7: TMEM lane quarter = warp % 4, so row = 32 * (warp % 4) + lane
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        bool ok = true;
        int chunk = 0;
        for (int it = 0; ok && it < my_items; ++it) {
            const int item = blockIdx.x + it * gridDim.x;
            const int64_t hl = item / mtiles;                  // head within the group
            const int i = (item % mtiles) * 128 + row;
            float* dst = S + (hl * Tb + i) * (int64_t)ld_s;
            for (int n = 0; n < nchunks; ++n, ++chunk) {
                const int a = chunk & 1;
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&acc_full[a]), (chunk >> 1) & 1, abort, status));
                if (!ok) break;
                tc_fence_after();
                const uint32_t taddr = tmem + lane_addr + Cfg::NCH * a;
                #pragma unroll 1
                for (int c0 = 0; c0 < Cfg::NCH; c0 += 32) {
                    const int j0 = n * Cfg::NCH + c0;
                    if (j0 >= Tb) break;                        // uniform over the warp
                    uint32_t r[32];
                    tmem_ld32(taddr + c0, r);
                    tmem_wait_ld();
                    if (i < Tb) {
                        if (j0 + 32 <= Tb) {
                            #pragma unroll
                            for (int q = 0; q < 8; ++q)
                                reinterpret_cast<float4*>(dst + j0)[q] = make_float4(
                                    __uint_as_float(r[4 * q]) * inv_sqrt_d, __uint_as_float(r[4 * q + 1]) * inv_sqrt_d,
                                    __uint_as_float(r[4 * q + 2]) * inv_sqrt_d, __uint_as_float(r[4 * q + 3]) * inv_sqrt_d);
                        } else {
                            #pragma unroll
                            for (int q = 0; q < 32; ++q)
                                if (j0 + q < Tb) dst[j0 + q] = __uint_as_float(r[q]) * inv_sqrt_d;
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(smem_u32(&acc_empty[a]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------------
// Top-n per row + sink + CSR (eq. (8), section 3.4) from precomputed scores:
// R rows of one head per CTA (256 threads), the rows' scores loaded as
// order-preserving keys into shared memory, then one warp per row: 4-pass
// 8-bit radix select of the n-th largest key (equal scores: lower j), and an
// ascending ballot-ordered CSR write including every sink column.
template <int R>
__global__ void __launch_bounds__(kSelThreads) select_from_scores_kernel(const float* __restrict__ S, int32_t ld_s,
                                                                         int32_t* __restrict__ row_start,
                                                                         int32_t* __restrict__ row_count,
                                                                         int32_t* __restrict__ col_idx, MaskGeo mg,
                                                                         int64_t h0)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int Tb = mg.Tb;
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw);            // [R][Tb]
    uint32_t* hist_all = keys + (size_t)R * Tb;                          // [8][256], then [8][kSelCand]
    const int64_t hl = blockIdx.y;                                        // head within the group
    const int64_t bh = h0 + hl;
    const int i0 = blockIdx.x * R;
    const int nrows = min(R, Tb - i0);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const bool keep_all = mg.n_keep >= Tb;
    const int n_score_rows = keep_all ? 0 : max(0, min(nrows, mg.sink_first - i0));
    // the rows' scores as keys: 16-byte loads (rows are ld_s = T_b rounded up
    // to 4 floats apart), all rows of the CTA in flight together
    const int nq = (Tb + 3) >> 2;
    for (int idx = tid; idx < n_score_rows * nq; idx += kSelThreads) {
        const int r = idx / nq, q4 = idx - r * nq;
        const float4 f = *reinterpret_cast<const float4*>(S + (hl * Tb + i0 + r) * (int64_t)ld_s + 4 * q4);
        uint32_t* dst = keys + (size_t)r * Tb + 4 * q4;
        const int j = 4 * q4;
        dst[0] = float_order_key(f.x);
        if (j + 1 < Tb) dst[1] = float_order_key(f.y);
        if (j + 2 < Tb) dst[2] = float_order_key(f.z);
        if (j + 3 < Tb) dst[3] = float_order_key(f.w);
    }
    __syncthreads();
    uint32_t* hist = hist_all + warp * 256;
    uint32_t* cand = hist_all + (kSelThreads / 32) * 256 + warp * kSelCand;
    for (int r = warp; r < nrows; r += kSelThreads / 32) {
        if (RF2_SELECT_SAMPLED)
            select_row_sampled(keys + (size_t)r * Tb, hist, cand, mg, bh, i0 + r, lane, row_start, row_count, col_idx,
                               keep_all);
        else
            select_row(keys + (size_t)r * Tb, hist, mg, bh, i0 + r, lane, row_start, row_count, col_idx, keep_all);
    }
}

// Inverse of float_order_key.
__device__ __forceinline__ float order_key_float(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Top-n selection, keys in registers, few counting probes: the threshold key
// (the n-th largest) is bracketed by keys lo < hi with #{key >= lo} >= n >
// #{key >= hi}; each probe counts the keys at or above one candidate key
// (KPL compares per lane and a warp sum).  Probes alternate between a guess
// interpolated in score value from the bracket's counts (scores are smooth,
// so a few probes narrow the bracket to a handful of keys) and a plain key
// bisection (which bounds the probe count).  Once at most 32 keys lie in the
// bracket they are gathered and ranked exactly with one warp-wide bitonic
// sort.  Equal keys go to the lowest j; output as in select_row.
template <int KPL>
__global__ void __launch_bounds__(kSelThreads) select_probe_kernel(const float* __restrict__ S, int32_t ld_s,
                                                                   int32_t* __restrict__ row_start,
                                                                   int32_t* __restrict__ row_count,
                                                                   int32_t* __restrict__ col_idx, MaskGeo mg,
                                                                   int64_t h0)
{
    __shared__ uint32_t cand_all[kSelThreads];
    const int Tb = mg.Tb;
    const int lane = threadIdx.x & 31;
    uint32_t* cand = cand_all + (threadIdx.x & ~31);
    const int64_t hl = blockIdx.y;
    const int64_t bh = h0 + hl;
    const int i = blockIdx.x * (kSelThreads / 32) + (threadIdx.x >> 5);
    if (i >= Tb) return;                                   // whole warp
    const int64_t rs = row_offset(mg, bh, i);
    const int64_t row_id = bh * Tb + i;
    int32_t* out = col_idx + rs;
    if (i >= mg.sink_first || mg.n_keep >= Tb) {
        for (int j = lane; j < Tb; j += 32) csr_put(out, j, j, rs, mg.col_capacity);
        if (lane == 0) { row_start[row_id] = (int32_t)rs; row_count[row_id] = Tb; }
        return;
    }
    const float* src = S + (hl * Tb + i) * (int64_t)ld_s;
    uint32_t key[KPL];
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    #pragma unroll
    for (int u = 0; u < KPL; ++u) {
        const int j = u * 32 + lane;
        key[u] = (j < Tb) ? float_order_key(src[j]) : 0u;
        if (j < Tb) { kmin = min(kmin, key[u]); kmax = max(kmax, key[u]); }
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    const int n = mg.n_keep;
    auto count_ge = [&](uint32_t K) -> int {
        int c = 0;
        #pragma unroll
        for (int u = 0; u < KPL; ++u) c += (u * 32 + lane < Tb) && (key[u] >= K);
        return __reduce_add_sync(0xffffffffu, c);
    };
    // bracket: [lo, hi) with count_ge(lo) = c_lo >= n > c_hi = count_ge(hi)
    uint64_t lo = kmin, hi = (uint64_t)kmax + 1;
    int c_lo = Tb, c_hi = 0;
    #pragma unroll 1
    for (int it = 0; it < 80 && c_lo - c_hi > 32 && hi - lo > 1; ++it) {
        uint64_t mid;
        if ((it & 1) == 0) {
            const float vlo = order_key_float((uint32_t)lo), vhi = order_key_float((uint32_t)(hi - 1));
            // the bracket's keys below the n-th largest, as a fraction of the
            // bracket: place the guess that far up the bracket's value range
            const float f = ((float)(c_lo - n) + 0.5f) / (float)(c_lo - c_hi);
            mid = float_order_key(vlo + f * (vhi - vlo));
        } else {
            mid = lo + ((hi - lo) >> 1);
        }
        if (mid <= lo) mid = lo + 1;
        if (mid >= hi) mid = hi - 1;
        const int c = count_ge((uint32_t)mid);
        if (c >= n) { lo = mid; c_lo = c; }
        else { hi = mid; c_hi = c; }
    }
    uint32_t thr;
    if (hi - lo <= 1) {
        thr = (uint32_t)lo;
    } else {
        // at most 32 keys in [lo, hi): gather them and rank them exactly
        int base = 0;
        #pragma unroll
        for (int u = 0; u < KPL; ++u) {
            const bool in = (u * 32 + lane < Tb) && key[u] >= (uint32_t)lo && (uint64_t)key[u] < hi;
            const uint32_t b = __ballot_sync(0xffffffffu, in);
            if (in) cand[base + __popc(b & ((1u << lane) - 1u))] = key[u];
            base += __popc(b);
        }
        __syncwarp();
        uint32_t v = (lane < base) ? cand[lane] : 0u;       // 0 sorts below every candidate
        // bitonic sort, descending over the 32 lanes
        #pragma unroll
        for (int k = 2; k <= 32; k <<= 1) {
            #pragma unroll
            for (int jj = k >> 1; jj > 0; jj >>= 1) {
                const uint32_t o = __shfl_xor_sync(0xffffffffu, v, jj);
                const bool desc = ((lane & k) == 0);
                const bool lower = ((lane & jj) == 0);
                v = (lower == desc) ? max(v, o) : min(v, o);
            }
        }
        thr = __shfl_sync(0xffffffffu, v, n - c_hi - 1);      // rank n - c_hi within the bracket
        __syncwarp();
    }
    int gt = 0;
    #pragma unroll
    for (int u = 0; u < KPL; ++u) gt += (u * 32 + lane < Tb) && (key[u] > thr);
    gt = __reduce_add_sync(0xffffffffu, gt);
    int eq_left = n - gt;                                  // keys equal to thr that are kept
    int written = 0;
    #pragma unroll
    for (int u = 0; u < KPL; ++u) {
        const int j = u * 32 + lane;
        if (u * 32 >= Tb) break;                           // uniform
        const uint32_t k = key[u];
        const bool eq = (j < Tb) && (k == thr);
        const uint32_t eq_ballot = __ballot_sync(0xffffffffu, eq);
        const int eq_rank = __popc(eq_ballot & ((1u << lane) - 1u));
        const bool sel = (j < Tb) && (k > thr || (eq && eq_rank < eq_left) || j >= mg.sink_first);
        eq_left -= __popc(eq_ballot);
        const uint32_t sel_ballot = __ballot_sync(0xffffffffu, sel);
        if (sel) csr_put(out, written + __popc(sel_ballot & ((1u << lane) - 1u)), j, rs, mg.col_capacity);
        written += __popc(sel_ballot);
    }
    if (lane == 0) { row_start[row_id] = (int32_t)rs; row_count[row_id] = written; }
}

// CDF-threshold selection ("RainFusion2.0" section 2, online adaptive
// patterns: the best key blocks of a row are kept until the cumulative
// softmax of its pooled scores reaches tau), the sink of section 3.4 added on
// top.  One warp per row, the row's order keys and weights in shared memory:
//   w_j = 2^((S_j - max) log2 e)  and  Z = sum_j w_j  (fp32; each lane sums its
//   columns in ascending order, then an xor butterfly, so every lane holds the
//   same bits),
//   K* = the largest key with W(>= K*) >= tau Z, found by bisection over the
//   row's key range (W(>= K) summed the same way),
//   kept = {key > K*} plus the first c blocks of key K* in ascending j, c the
//   smallest count with W(> K*) + c w(K*) >= tau Z.
// This is the shortest prefix of the (score desc, j asc) order whose mass
// reaches tau.  Rows use the full capacity T_b (make_mask_geo with
// n_keep = T_b), so row offsets stay closed-form.
__device__ __forceinline__ float warp_sum_same(float v)
{
    #pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

template <int R>
__global__ void __launch_bounds__(32 * R) select_cdf_kernel(const float* __restrict__ S, int32_t ld_s,
                                                            int32_t* __restrict__ row_start,
                                                            int32_t* __restrict__ row_count,
                                                            int32_t* __restrict__ col_idx, MaskGeo mg, int64_t h0,
                                                            float tau)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int Tb = mg.Tb;
    const int lane = threadIdx.x & 31;
    const int r = threadIdx.x >> 5;
    const int64_t hl = blockIdx.y;
    const int64_t bh = h0 + hl;
    const int i = blockIdx.x * R + r;
    if (i >= Tb) return;                                   // whole warp
    uint32_t* key = reinterpret_cast<uint32_t*>(smem_raw) + (size_t)r * Tb;
    float* w = reinterpret_cast<float*>(smem_raw) + (size_t)R * Tb + (size_t)r * Tb;
    const int64_t rs = row_offset(mg, bh, i);
    const int64_t row_id = bh * Tb + i;
    int32_t* out = col_idx + rs;
    if (i >= mg.sink_first) {
        for (int j = lane; j < Tb; j += 32) csr_put(out, j, j, rs, mg.col_capacity);
        if (lane == 0) { row_start[row_id] = (int32_t)rs; row_count[row_id] = Tb; }
        return;
    }
    const float* src = S + (hl * Tb + i) * (int64_t)ld_s;
    float mx = -INFINITY;
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int j = lane; j < Tb; j += 32) {
        const float v = src[j];
        const uint32_t k = float_order_key(v);
        key[j] = k;
        mx = fmaxf(mx, v);
        kmin = min(kmin, k);
        kmax = max(kmax, k);
    }
    #pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    float z = 0.f;
    for (int j = lane; j < Tb; j += 32) {
        const float v = src[j];
        const float wj = exp2f((v - mx) * 1.4426950408889634f);
        w[j] = wj;
        z += wj;
    }
    z = warp_sum_same(z);
    const float target = tau * z;
    __syncwarp();
    auto mass_ge = [&](uint32_t K) -> float {
        float a = 0.f;
        for (int j = lane; j < Tb; j += 32) a += (key[j] >= K) ? w[j] : 0.f;
        return warp_sum_same(a);
    };
    uint32_t lo = kmin, hi = kmax;                         // mass_ge(kmin) = z >= target
    while (lo < hi) {
        const uint32_t mid = lo + (uint32_t)(((uint64_t)hi - lo + 1) >> 1);
        if (mass_ge(mid) >= target) lo = mid;
        else hi = mid - 1;
    }
    const uint32_t thr = lo;
    const float w_gt = (thr == 0xffffffffu) ? 0.f : mass_ge(thr + 1);
    int n_eq = 0;
    float w_eq = 0.f;
    for (int j0 = 0; j0 < Tb; j0 += 32) {
        const int j = j0 + lane;
        const bool eq = (j < Tb) && key[j] == thr;
        const uint32_t b = __ballot_sync(0xffffffffu, eq);
        if (b && w_eq == 0.f) w_eq = __shfl_sync(0xffffffffu, eq ? w[j] : 0.f, __ffs(b) - 1);
        n_eq += __popc(b);
    }
    int c = 1;
    if (n_eq > 1 && w_eq > 0.f) {
        c = (int)ceilf((target - w_gt) / w_eq);
        c = max(1, min(n_eq, c));
        while (c > 1 && w_gt + (float)(c - 1) * w_eq >= target) --c;
        while (c < n_eq && w_gt + (float)c * w_eq < target) ++c;
    }
    int eq_left = c;
    int written = 0;
    for (int j0 = 0; j0 < Tb; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t k = (j < Tb) ? key[j] : 0u;
        const bool eq = (j < Tb) && (k == thr);
        const uint32_t eq_ballot = __ballot_sync(0xffffffffu, eq);
        const int eq_rank = __popc(eq_ballot & ((1u << lane) - 1u));
        const bool sel = (j < Tb) && (k > thr || (eq && eq_rank < eq_left) || j >= mg.sink_first);
        eq_left -= __popc(eq_ballot);
        const uint32_t sel_ballot = __ballot_sync(0xffffffffu, sel);
        if (sel) csr_put(out, written + __popc(sel_ballot & ((1u << lane) - 1u)), j, rs, mg.col_capacity);
        written += __popc(sel_ballot);
    }
    if (lane == 0) { row_start[row_id] = (int32_t)rs; row_count[row_id] = written; }
}

}  // namespace rf2
