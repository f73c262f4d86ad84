// Block-sparse FlashAttention forward on tcgen05 ("RainFusion2.0" section 3.1:
// eqs. (1)-(4) with the block mask M; Q_i K_j^T and P_ij V_j skipped when
// M_ij = 0).
//
// Work unit: one CTA computes two adjacent 64-row query blocks (2p, 2p+1) of
// one (batch, head) as a single M = 128 tile (a cta_group::1 tcgen05 MMA runs
// at full rate only at M = 128; M = 64 runs at half rate).  It visits the
// sorted union of the two blocks' CSR rows (built as bitmaps, so rows need
// not even be sorted); each union entry carries one "kept" bit per query
// block, and the rows of a block that did not keep key block j get no
// probability mass from it (P exactly 0), so every row sees exactly its own
// kept blocks.
//
// A step covers two union entries (128 keys): S = Q [K_a; K_b]^T is one
// M128 x N128 product (an N = 64 product leaves a third of the tensor pipe
// idle), then O += P [V_a; V_b].
//
// Roles (256 threads, two CTAs per SM so that one CTA's softmax overlaps the
// other's MMAs):
//   warps 0-3  softmax + epilogue: thread r owns query row r = TMEM lane r
//              and its full 128-column score row
//   warp 4     MMA issuer (one thread)
//   warp 5     TMA: Q once, then K of the step's first key block
//   warp 6     TMA: K of the step's second key block
//   warp 7     TMA: V of both key blocks
// (one thread's TMA stream is served serially, so loads are spread over three
// issuing warps).  Shared memory: Q 32 KB and one 32 KB K and V stage, all
// 128-byte swizzled.  TMEM: O (d fp32 columns) and one 128-column S buffer;
// P (bf16) is written over the first 64 columns of S and read by the PV
// product straight from TMEM.  Per CTA the chain is S_t -> softmax_t -> PV_t
// -> S_{t+1}; the tensor pipe serves the other CTA in between.
//
// Softmax (eqs. (2)-(4)) in fp32, log2 domain, per thread: pass 1 loads the
// row's scores 32 columns at a time for the block max; pass 2 reloads them
// (the next chunk's load in flight while the current one is exponentiated),
// writes P in bf16 and accumulates the row sum.  The running max m is raised
// (and O rescaled in TMEM) only when a step's max exceeds it by more than 8
// (a factor 256); O and l always use the same m, so O / l is unchanged.  O
// can be rescaled without waiting: PV_{t-1} was issued before S_t, so it has
// completed once S_t has.  kExpEmu of every 32 exponentials per chunk run on
// the FMA pipe (exp2_poly) instead of the SFU.
//
// Every wait on an mbarrier is bounded (ptx.cuh): on a timeout the CTA
// raises a shared abort flag, every role leaves its loop, in-flight TMA loads
// and MMAs are drained (again with a time limit), TMEM is freed and the
// device status word records RF2_ERR_TIMEOUT.
#pragma once
#include "geometry.cuh"
#include "ptx.cuh"

#ifndef RF2_EXP2_EMU
#define RF2_EXP2_EMU 0
#endif

namespace rf2 {

template <int D>
struct AttnCfg {
    static constexpr int KCH = D / 64;                     // 128-byte column chunks per row
    static constexpr uint32_t Q_CHUNK = 128 * 128;         // one 64-column chunk of Q (128 rows)
    static constexpr uint32_t Q_BYTES = Q_CHUNK * KCH;
    static constexpr uint32_t K_CHUNK = 128 * 128;         // one chunk of the K stage: 128 key rows
    static constexpr uint32_t KV_STAGE = 128 * D * 2;      // two 64-key blocks
    static constexpr uint32_t V_BLOCK = 64 * D * 2;        // one key block of V: [chunk][64 rows]
    static constexpr uint32_t TM_O = 0;
    static constexpr uint32_t TM_S = 128;
    static constexpr uint32_t TM_COLS = 256;
    static constexpr int THREADS = 256;
    static constexpr int MMA_WARP = 4;
    static constexpr int KA_WARP = 5;
    static constexpr int KB_WARP = 6;
    static constexpr int V_WARP = 7;
    // Shared memory: [align slack][Q][K stage][V stage][union list][control]
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + KV_STAGE;
    static constexpr uint32_t OFF_LIST = OFF_V + KV_STAGE;
    static constexpr uint32_t CONTROL_BYTES = 256;
    __host__ __device__ static size_t list_bytes(int Tb) { return ((size_t)Tb * 4 + 15) & ~(size_t)15; }
    __host__ __device__ static size_t smem_bytes(int Tb) { return 1024 + OFF_LIST + list_bytes(Tb) + CONTROL_BYTES; }
};

struct __align__(16) AttnCtl {
    uint64_t q_full;
    uint64_t k_full, k_empty;
    uint64_t v_full, v_empty;
    uint64_t s_full, p_full;
    uint64_t o_final, drain;
    uint32_t tmem_base;
    int32_t list_len;
    int32_t abort;
};
static_assert(sizeof(AttnCtl) <= 256, "control block must fit CONTROL_BYTES");

struct AttnArgs {
    const int32_t* row_start;
    const int32_t* row_count;
    const int32_t* col_idx;
    uint16_t* op;           // bf16 bits [BH, N, D]
    float* lse;             // [BH, N] or null
    int* status;            // device status word
    int32_t N;
    int32_t Tb;
    int32_t pairs;          // ceil(Tb / 2)
    int32_t sink_pairs;     // pairs holding a sink block: scheduled first in each head
    float scale_log2;       // log2(e) / sqrt(D)
};

// 32 scores of one row -> 16 packed bf16 pairs of P = 2^(s*sl2 - m), adding
// the fp32 probabilities to sum4.  `nvalid` < 32 masks the tail columns.
#ifndef RF2_EXP_PACKED
#define RF2_EXP_PACKED 1
#endif

template <bool kMasked>
__device__ __forceinline__ void exp_chunk(const uint32_t (&s)[32], float sl2, float neg_mu, int nvalid,
                                          uint32_t (&pk)[16], float (&sum4)[4])
{
    if (RF2_EXP_PACKED) {
        // x = s*sl2 - m and the row sums two lanes at a time (fma/add.f32x2)
        const float2 sc = make_float2(sl2, sl2), mu = make_float2(neg_mu, neg_mu);
        float2 acc[2] = {make_float2(sum4[0], sum4[1]), make_float2(sum4[2], sum4[3])};
        #pragma unroll
        for (int c = 0; c < 32; c += 2) {
            const float2 x = ffma2(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), sc, mu);
            float2 p = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            if (kMasked) {
                p.x = (c < nvalid) ? p.x : 0.f;
                p.y = (c + 1 < nvalid) ? p.y : 0.f;
            }
            acc[(c >> 1) & 1] = fadd2(acc[(c >> 1) & 1], p);
            pk[c >> 1] = pack_bf16x2(p.x, p.y);
        }
        sum4[0] = acc[0].x; sum4[1] = acc[0].y; sum4[2] = acc[1].x; sum4[3] = acc[1].y;
        return;
    }
    #pragma unroll
    for (int c = 0; c < 32; c += 2) {
        const float x0 = fmaf(__uint_as_float(s[c]), sl2, neg_mu);
        const float x1 = fmaf(__uint_as_float(s[c + 1]), sl2, neg_mu);
        float p0 = (c < RF2_EXP2_EMU) ? exp2_poly(x0) : ex2_approx(x0);
        float p1 = (c + 1 < RF2_EXP2_EMU) ? exp2_poly(x1) : ex2_approx(x1);
        if (kMasked) {
            p0 = (c < nvalid) ? p0 : 0.f;
            p1 = (c + 1 < nvalid) ? p1 : 0.f;
        }
        sum4[(c >> 1) & 3] += p0 + p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
    }
}

template <bool kMasked>
__device__ __forceinline__ float max_chunk(const uint32_t (&s)[32], int nvalid, float acc)
{
    float m4[4] = {acc, -INFINITY, -INFINITY, -INFINITY};
    #pragma unroll
    for (int c = 0; c < 32; ++c) {
        const float v = __uint_as_float(s[c]);
        m4[c & 3] = fmaxf(m4[c & 3], (!kMasked || c < nvalid) ? v : -INFINITY);
    }
    return fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
}

template <int D>
__global__ void __launch_bounds__(AttnCfg<D>::THREADS, 2)
block_sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_kc,
                         const __grid_constant__ CUtensorMap tm_v, const AttnArgs args)
{
    using Cfg = AttnCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_u32 - raw_u32);
    int32_t* list = reinterpret_cast<int32_t*>(base + Cfg::OFF_LIST);
    AttnCtl* ctl = reinterpret_cast<AttnCtl*>(base + Cfg::OFF_LIST + Cfg::list_bytes(args.Tb));

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int Tb = args.Tb;

    // ---- work item: (bh, pair); sink pairs of a head first (they are the longest)
    const int64_t bh = blockIdx.x / args.pairs;
    const int u = (int)(blockIdx.x - bh * args.pairs);
    const int pair = (u < args.sink_pairs) ? (args.pairs - 1 - u) : (u - args.sink_pairs);
    const int qb0 = 2 * pair;
    const bool has_b = (qb0 + 1) < Tb;

    // ---- set-up: barriers, TMEM, union of the two CSR rows
    if (tid == 0) {
        mbar_init(smem_u32(&ctl->q_full), 1);
        mbar_init(smem_u32(&ctl->k_full), 2);              // the two K producers arrive
        mbar_init(smem_u32(&ctl->k_empty), 1);
        mbar_init(smem_u32(&ctl->v_full), 1);
        mbar_init(smem_u32(&ctl->v_empty), 1);
        mbar_init(smem_u32(&ctl->s_full), 1);
        mbar_init(smem_u32(&ctl->p_full), 128);
        mbar_init(smem_u32(&ctl->o_final), 1);
        mbar_init(smem_u32(&ctl->drain), 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == Cfg::KA_WARP && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_kc);
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ctl->tmem_base), Cfg::TM_COLS);
        tmem_relinquish();
    }
    // Union of the two CSR rows as bitmaps (one bit per key block and query
    // block), built in the still unused K stage, then compacted in ascending
    // order: a word's entries start at the popcount of all earlier words.
    const int W = (Tb + 31) >> 5;                          // <= 128 words
    uint32_t* bmA = reinterpret_cast<uint32_t*>(base + Cfg::OFF_K);
    uint32_t* bmB = bmA + W;
    int32_t* word_off = reinterpret_cast<int32_t*>(bmB + W);
    for (int w = tid; w < 2 * W; w += Cfg::THREADS) bmA[w] = 0u;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    const int64_t rA = bh * Tb + qb0;
    {
        const int lenA = min(max(args.row_count[rA], 0), Tb);
        const int32_t* srcA = args.col_idx + args.row_start[rA];
        for (int e = tid; e < lenA; e += Cfg::THREADS) {
            const int32_t j = srcA[e];
            if (j >= 0 && j < Tb) atomicOr(&bmA[j >> 5], 1u << (j & 31));
        }
        if (has_b) {
            const int lenB = min(max(args.row_count[rA + 1], 0), Tb);
            const int32_t* srcB = args.col_idx + args.row_start[rA + 1];
            for (int e = tid; e < lenB; e += Cfg::THREADS) {
                const int32_t j = srcB[e];
                if (j >= 0 && j < Tb) atomicOr(&bmB[j >> 5], 1u << (j & 31));
            }
        }
    }
    __syncthreads();
    if (warp == 0) {
        int cnt[4];
        int local = 0;
        #pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int w = lane * 4 + k;
            cnt[k] = (w < W) ? __popc(bmA[w] | bmB[w]) : 0;
            local += cnt[k];
        }
        int incl = local;
        #pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        int run = incl - local;
        #pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int w = lane * 4 + k;
            if (w < W) word_off[w] = run;
            run += cnt[k];
        }
        if (lane == 31) ctl->list_len = incl;
    }
    __syncthreads();
    for (int w = tid; w < W; w += Cfg::THREADS) {
        const uint32_t a = bmA[w], b = bmB[w];
        uint32_t m = a | b;
        int pos = word_off[w];
        while (m) {
            const int bit = __ffs(m) - 1;
            m &= m - 1;
            list[pos++] = (w * 32 + bit) | (int32_t)(((a >> bit) & 1u) << 30) | (int32_t)(((b >> bit) & 1u) << 31);
        }
    }
    __syncthreads();
    const int L = ctl->list_len;
    const int T = (L + 1) >> 1;                            // steps of two key blocks
    volatile int* abort = &ctl->abort;

    // Key block of entry e (a missing second entry of the last step repeats
    // the first one: valid data whose kept bits are 0).
    auto block_of = [&](int e) -> int { return min((e < L ? list[e] : list[e - 1]) & 0x3fffffff, Tb - 1); };

    if (warp == Cfg::KA_WARP || warp == Cfg::KB_WARP) {
        // ------------------------------------------------ TMA: K of one key block per step
        if (lane == 0) {
            fence_proxy_async_smem();   // the stage held the row bitmaps (generic accesses)
            const int g = (warp == Cfg::KA_WARP) ? 0 : 1;
            int issued = -1;
            if (g == 0) {
                mbar_arrive_expect_tx(smem_u32(&ctl->q_full), Cfg::Q_BYTES);
                tma_load_4d(base_u32 + Cfg::OFF_Q, &tm_q, smem_u32(&ctl->q_full), 0, qb0 * 64, 0, (int)bh);
            }
            for (int t = 0; t < T; ++t) {
                if (t > 0 && !mbar_wait(smem_u32(&ctl->k_empty), (t - 1) & 1, abort, args.status)) break;
                const int j = block_of(2 * t + g);
                const uint32_t dst = base_u32 + Cfg::OFF_K + g * 64 * 128;
                mbar_arrive_expect_tx(smem_u32(&ctl->k_full), Cfg::KV_STAGE / 2);
                for (int c = 0; c < Cfg::KCH; ++c)
                    tma_load_3d(dst + c * Cfg::K_CHUNK, &tm_kc, smem_u32(&ctl->k_full), c * 64, j * 64, (int)bh);
                issued = t;
            }
            // Drain: no TMA may still be writing shared memory when the CTA exits.
            if (g == 0) mbar_wait_drain(smem_u32(&ctl->q_full), 0);
            if (issued >= 0) mbar_wait_drain(smem_u32(&ctl->k_full), issued & 1);
        }
    } else if (warp == Cfg::V_WARP) {
        // ------------------------------------------------ TMA: V of both key blocks
        if (lane == 0) {
            fence_proxy_async_smem();
            int issued = -1;
            for (int t = 0; t < T; ++t) {
                if (t > 0 && !mbar_wait(smem_u32(&ctl->v_empty), (t - 1) & 1, abort, args.status)) break;
                const uint32_t dst = base_u32 + Cfg::OFF_V;
                mbar_arrive_expect_tx(smem_u32(&ctl->v_full), Cfg::KV_STAGE);
                for (int g = 0; g < 2; ++g)
                    tma_load_4d(dst + g * Cfg::V_BLOCK, &tm_v, smem_u32(&ctl->v_full), 0, block_of(2 * t + g) * 64,
                                0, (int)bh);
                issued = t;
            }
            if (issued >= 0) mbar_wait_drain(smem_u32(&ctl->v_full), issued & 1);
        }
    } else if (warp == Cfg::MMA_WARP) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0);
            constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, 1);
            const uint32_t q_s = base_u32 + Cfg::OFF_Q;
            const uint32_t k_s = base_u32 + Cfg::OFF_K;
            const uint32_t v_s = base_u32 + Cfg::OFF_V;
            bool ok = (T == 0) || mbar_wait(smem_u32(&ctl->q_full), 0, abort, args.status);
            tc_fence_after();
            for (int t = 0; ok && t < T; ++t) {
                const uint32_t par = t & 1;
                if (!mbar_wait(smem_u32(&ctl->k_full), par, abort, args.status)) break;
                tc_fence_after();
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk & 3) * 32;          // 16 bf16 = 32 bytes per K step
                    const uint64_t a = smem_desc_sw128(q_s + (kk >> 2) * Cfg::Q_CHUNK + off, 16, 1024);
                    const uint64_t b = smem_desc_sw128(k_s + (kk >> 2) * Cfg::K_CHUNK + off, 16, 1024);
                    mma_ss(tmem + Cfg::TM_S, a, b, IDESC_S, kk > 0 ? 1u : 0u);
                }
                mma_commit(smem_u32(&ctl->s_full));
                mma_commit(smem_u32(&ctl->k_empty));
                if (!mbar_wait(smem_u32(&ctl->p_full), par, abort, args.status)) break;
                if (!mbar_wait(smem_u32(&ctl->v_full), par, abort, args.status)) break;
                tc_fence_after();
                #pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    // 16 keys per K step: steps 0-3 in block a, 4-7 in block b
                    const uint64_t b = smem_desc_sw128(v_s + (kk >> 2) * Cfg::V_BLOCK + (kk & 3) * 2048, 64 * 128, 1024);
                    mma_ts(tmem + Cfg::TM_O, tmem + Cfg::TM_S + kk * 8, b, IDESC_O, (t > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(smem_u32(&ctl->v_empty));
                if (t == T - 1) mma_commit(smem_u32(&ctl->o_final));
            }
            // Drain: every MMA this thread issued has completed before TMEM is freed.
            mma_commit(smem_u32(&ctl->drain));
            mbar_wait_drain(smem_u32(&ctl->drain), 0);
        }
    } else {
        // ------------------------------------------------ softmax + epilogue (warps 0-3)
        const int row = tid;                       // 0..127 = TMEM lane
        const int half = row >> 6;                 // which query block of the pair
        const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
        const uint32_t s_row = tmem + lane_addr + Cfg::TM_S;
        const float sl2 = args.scale_log2;
        float m_run = -INFINITY;
        float l_run = 0.f;
        bool ok = true;
        for (int t = 0; t < T; ++t) {
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl->s_full), t & 1, abort, args.status));
            if (!ok) break;
            tc_fence_after();
            // kept flags and valid key counts of the step's two key blocks (uniform over the warp)
            bool kept[2];
            int nv[2];
            #pragma unroll
            for (int g = 0; g < 2; ++g) {
                const int e = 2 * t + g;
                const int32_t ent = (e < L) ? list[e] : 0;
                kept[g] = (e < L) && ((ent >> (30 + half)) & 1);
                nv[g] = min(64, args.N - (ent & 0x3fffffff) * 64);
            }
            // pass 1: row max over the kept blocks
            float mx = -INFINITY;
            #pragma unroll
            for (int g = 0; g < 2; ++g) {
                if (!kept[g]) continue;
                uint32_t a[32], b[32];
                tmem_ld32(s_row + 64 * g, a);
                tmem_ld32(s_row + 64 * g + 32, b);
                tmem_wait_ld();
                reg_fence(a);
                reg_fence(b);
                if (nv[g] == 64) {
                    mx = max_chunk<false>(a, 64, mx);
                    mx = max_chunk<false>(b, 64, mx);
                } else {
                    mx = max_chunk<true>(a, nv[g], mx);
                    mx = max_chunk<true>(b, nv[g] - 32, mx);
                }
            }
            const float mb = mx * sl2;                     // scale > 0: max commutes
            const bool need = (m_run != -INFINITY) && (mb > m_run + 8.0f);
            if (__any_sync(0xffffffffu, need)) {
                // Rescale O: PV_{t-1} was issued before S_t, so it is complete.
                float f = 1.f;
                if (need) { f = ex2_approx(m_run - mb); l_run *= f; m_run = mb; }
                #pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_addr + Cfg::TM_O + c0, o);
                    tmem_wait_ld();
                    reg_fence(o);
                    #pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
                    tmem_st32(tmem + lane_addr + Cfg::TM_O + c0, o);
                }
            }
            if (m_run == -INFINITY) m_run = mb;
            const float neg_mu = (m_run == -INFINITY) ? 0.f : -m_run;
            // pass 2: P = 2^(s*sl2 - m) in bf16 over the first 64 columns of S,
            // chunk q of 32 scores -> 16 columns at 16q (behind every chunk read)
            float sum4[4] = {0.f, 0.f, 0.f, 0.f};
            #pragma unroll
            for (int g = 0; g < 2; ++g) {
                uint32_t pk[16];
                if (kept[g]) {
                    uint32_t a[32];
                    tmem_ld32(s_row + 64 * g, a);
                    tmem_wait_ld();
                    reg_fence(a);
                    uint32_t b[32];
                    tmem_ld32(s_row + 64 * g + 32, b);         // in flight during the first half
                    if (nv[g] == 64) exp_chunk<false>(a, sl2, neg_mu, 32, pk, sum4);
                    else exp_chunk<true>(a, sl2, neg_mu, nv[g], pk, sum4);
                    tmem_st16(s_row + 32 * g, pk);
                    tmem_wait_ld();
                    reg_fence(b);
                    if (nv[g] == 64) exp_chunk<false>(b, sl2, neg_mu, 32, pk, sum4);
                    else exp_chunk<true>(b, sl2, neg_mu, nv[g] - 32, pk, sum4);
                    tmem_st16(s_row + 32 * g + 16, pk);
                } else {
                    #pragma unroll
                    for (int c = 0; c < 16; ++c) pk[c] = 0u;
                    tmem_st16(s_row + 32 * g, pk);
                    tmem_st16(s_row + 32 * g + 16, pk);
                }
            }
            l_run += (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(smem_u32(&ctl->p_full));
        }
        // ---- epilogue: O / l -> bf16
        if (ok && T > 0)
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl->o_final), 0, abort, args.status));
        tc_fence_after();
        if (ok) {
            const int qb = qb0 + half;
            const int64_t tok = (int64_t)qb * 64 + (row & 63);
            const bool valid = (qb < Tb) && (tok < args.N);
            const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
            uint16_t* dst = args.op + ((int64_t)bh * args.N + tok) * D;
            #pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t o[32];
                if (T > 0) {
                    tmem_ld32(tmem + lane_addr + Cfg::TM_O + c0, o);
                    tmem_wait_ld();
                    reg_fence(o);
                } else {
                    #pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = 0u;
                }
                if (valid) {
                    uint32_t w[16];
                    #pragma unroll
                    for (int c = 0; c < 16; ++c)
                        w[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
                    uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
                    #pragma unroll
                    for (int c = 0; c < 4; ++c) d4[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                }
            }
            if (valid && args.lse) {
                args.lse[(int64_t)bh * args.N + tok] =
                    (l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TM_COLS);
    }
}

}  // namespace rf2
