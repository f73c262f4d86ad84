// Block-sparse FlashAttention forward on tcgen05 ("RainFusion2.0" section 3.1:
// eqs. (1)-(4) with the block mask M; Q_i K_j^T and P_ij V_j skipped when
// M_ij = 0).
//
// Work unit: one CTA computes two adjacent 64-row query blocks (2p, 2p+1) of
// one (batch, head) as a single M = 128 tile, the native row count of a
// cta_group::1 tcgen05 MMA.  The key blocks it visits are the sorted union of
// the two blocks' CSR rows (bitmap union, so rows need not even be sorted);
// each union entry carries one "kept" bit per query block, and the rows of a block that did not keep key block j are
// masked to -inf in the softmax (their P is exactly 0), so every row sees
// exactly its own kept blocks.
//
// Roles (192 threads):
//   warps 0-3  softmax + epilogue: thread r owns query row r, i.e. TMEM lane r
//   warp 4     TMA producer: Q once, then K_j and V_j tiles of every visited
//              key block into 2-stage rings (128-byte swizzled tiles)
//   warp 5     MMA issuer (one thread):  S_t = Q K_t^T  (SS, M128 N64, into
//              one of two TMEM S buffers) and O += P_t V_t (TS: P read from
//              TMEM where softmax wrote it over S_t, V from shared memory)
// TMEM: O (d fp32 columns) + two 64-column S/P buffers = 256 columns, so
// two CTAs fit on an SM and one's softmax overlaps the other's MMAs.
//
// Online softmax (eqs. (2)-(4)) in fp32 in the log2 domain.  The running max
// m is only raised when a block's max exceeds it by more than 8 (a factor
// 256), so O (in TMEM) is rarely rescaled; because O and l always use the
// same m, the final O / l is unchanged.  Scale, exp2 and sums are fp32; P is
// rounded to bf16 as the MMA operand.
//
// Every wait on an mbarrier is bounded (ptx.cuh): on a timeout the CTA
// raises a shared abort flag, every role leaves its loop, in-flight TMA loads
// and MMAs are drained (again with a time limit), TMEM is freed and the
// device status word records RF2_ERR_TIMEOUT.
#pragma once
#include "geometry.cuh"
#include "ptx.cuh"

namespace rf2 {

template <int D>
struct AttnCfg {
    static constexpr int BM = 128;
    static constexpr int BN = 64;
    static constexpr int KCH = D / 64;                 // 128-byte column chunks per row
    static constexpr int STAGES = 2;
    static constexpr uint32_t Q_CHUNK = BM * 128;      // bytes of one 64-column chunk of Q
    static constexpr uint32_t KV_CHUNK = BN * 128;
    static constexpr uint32_t Q_BYTES = Q_CHUNK * KCH;
    static constexpr uint32_t KV_BYTES = KV_CHUNK * KCH;
    static constexpr uint32_t TM_O = 0;
    static constexpr uint32_t TM_S = D;                // S/P buffer b at TM_S + 64*b
    static constexpr uint32_t TM_COLS = 256;
    static constexpr int THREADS = 192;
    static constexpr int PRODUCER_WARP = 4;
    static constexpr int MMA_WARP = 5;
    // Shared memory: [align slack][Q][K ring][V ring][union list (Tb words)][control]
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + STAGES * KV_BYTES;
    static constexpr uint32_t OFF_LIST = OFF_V + STAGES * KV_BYTES;
    static constexpr uint32_t CONTROL_BYTES = 256;
    // The list is padded to 16 bytes so the control block (mbarriers) stays aligned.
    __host__ __device__ static size_t list_bytes(int Tb) { return ((size_t)Tb * 4 + 15) & ~(size_t)15; }
    static size_t smem_bytes(int Tb) { return 1024 + OFF_LIST + list_bytes(Tb) + CONTROL_BYTES; }
};

struct __align__(16) AttnCtl {
    uint64_t q_full;
    uint64_t k_full[2], k_empty[2];
    uint64_t v_full[2], v_empty[2];
    uint64_t s_full[2], p_full[2];
    uint64_t o_done, o_final, drain;
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

template <int D>
__global__ void __launch_bounds__(AttnCfg<D>::THREADS, 2)
block_sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
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
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&ctl->k_full[s]), 1);
            mbar_init(smem_u32(&ctl->k_empty[s]), 1);
            mbar_init(smem_u32(&ctl->v_full[s]), 1);
            mbar_init(smem_u32(&ctl->v_empty[s]), 1);
            mbar_init(smem_u32(&ctl->s_full[s]), 1);
            mbar_init(smem_u32(&ctl->p_full[s]), 128);
        }
        mbar_init(smem_u32(&ctl->o_done), 1);
        mbar_init(smem_u32(&ctl->o_final), 1);
        mbar_init(smem_u32(&ctl->drain), 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == Cfg::PRODUCER_WARP && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ctl->tmem_base), Cfg::TM_COLS);
        tmem_relinquish();
    }
    // Union of the two CSR rows as bitmaps (one bit per key block and query
    // block), built in the still unused K/V rings, then compacted in
    // ascending order: a word's entries start at the popcount of all earlier
    // words of (A | B).
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
        // exclusive scan of per-word popcounts, 4 consecutive words per lane
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
        uint32_t u = a | b;
        int pos = word_off[w];
        while (u) {
            const int bit = __ffs(u) - 1;
            u &= u - 1;
            list[pos++] = (w * 32 + bit) | (int32_t)(((a >> bit) & 1u) << 30) | (int32_t)(((b >> bit) & 1u) << 31);
        }
    }
    __syncthreads();
    const int L = ctl->list_len;
    volatile int* abort = &ctl->abort;

    if (warp == Cfg::PRODUCER_WARP) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            fence_proxy_async_smem();   // the rings held the row bitmaps (generic accesses)
            const uint32_t q_s = base_u32 + Cfg::OFF_Q;
            mbar_arrive_expect_tx(smem_u32(&ctl->q_full), Cfg::Q_BYTES);
            for (int c = 0; c < Cfg::KCH; ++c)
                tma_load_3d(q_s + c * Cfg::Q_CHUNK, &tm_q, smem_u32(&ctl->q_full), c * 64, qb0 * 64, (int)bh);
            int issued_k[2] = {-1, -1}, issued_v[2] = {-1, -1};
            for (int t = 0; t < L; ++t) {
                const int s = t % Cfg::STAGES;
                const int use = t / Cfg::STAGES;
                const int j = min(list[t] & 0x3fffffff, Tb - 1);
                if (use > 0 && !mbar_wait(smem_u32(&ctl->k_empty[s]), (use - 1) & 1, abort, args.status)) break;
                const uint32_t k_s = base_u32 + Cfg::OFF_K + s * Cfg::KV_BYTES;
                mbar_arrive_expect_tx(smem_u32(&ctl->k_full[s]), Cfg::KV_BYTES);
                for (int c = 0; c < Cfg::KCH; ++c)
                    tma_load_3d(k_s + c * Cfg::KV_CHUNK, &tm_k, smem_u32(&ctl->k_full[s]), c * 64, j * 64, (int)bh);
                issued_k[s] = use;
                if (use > 0 && !mbar_wait(smem_u32(&ctl->v_empty[s]), (use - 1) & 1, abort, args.status)) break;
                const uint32_t v_s = base_u32 + Cfg::OFF_V + s * Cfg::KV_BYTES;
                mbar_arrive_expect_tx(smem_u32(&ctl->v_full[s]), Cfg::KV_BYTES);
                for (int c = 0; c < Cfg::KCH; ++c)
                    tma_load_3d(v_s + c * Cfg::KV_CHUNK, &tm_v, smem_u32(&ctl->v_full[s]), c * 64, j * 64, (int)bh);
                issued_v[s] = use;
            }
            // Drain: no TMA may still be writing shared memory when the CTA
            // exits.  Only this thread arms these barriers, so the phase of the
            // last load it issued is the one to wait for.
            mbar_wait_drain(smem_u32(&ctl->q_full), 0);
            for (int s = 0; s < Cfg::STAGES; ++s) {
                if (issued_k[s] >= 0) mbar_wait_drain(smem_u32(&ctl->k_full[s]), issued_k[s] & 1);
                if (issued_v[s] >= 0) mbar_wait_drain(smem_u32(&ctl->v_full[s]), issued_v[s] & 1);
            }
        }
    } else if (warp == Cfg::MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, 0);
            constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, 1);
            const uint32_t q_s = base_u32 + Cfg::OFF_Q;
            bool ok = (L == 0) || mbar_wait(smem_u32(&ctl->q_full), 0, abort, args.status);
            tc_fence_after();
            for (int t = 0; ok && t <= L; ++t) {
                if (t < L) {
                    const int s = t % Cfg::STAGES;
                    if (!mbar_wait(smem_u32(&ctl->k_full[s]), (t / Cfg::STAGES) & 1, abort, args.status)) break;
                    tc_fence_after();
                    const uint32_t k_s = base_u32 + Cfg::OFF_K + s * Cfg::KV_BYTES;
                    const uint32_t d_tmem = tmem + Cfg::TM_S + 64 * (t & 1);
                    #pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk & 3) * 32;   // 16 bf16 = 32 bytes per K step
                        const uint64_t a = smem_desc_sw128(q_s + (kk >> 2) * Cfg::Q_CHUNK + off, 16, 1024);
                        const uint64_t b = smem_desc_sw128(k_s + (kk >> 2) * Cfg::KV_CHUNK + off, 16, 1024);
                        mma_ss(d_tmem, a, b, IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(smem_u32(&ctl->s_full[t & 1]));
                    mma_commit(smem_u32(&ctl->k_empty[s]));
                }
                if (t >= 1) {
                    const int v = t - 1;
                    const int s = v % Cfg::STAGES;
                    if (!mbar_wait(smem_u32(&ctl->p_full[v & 1]), (v >> 1) & 1, abort, args.status)) break;
                    if (!mbar_wait(smem_u32(&ctl->v_full[s]), (v / Cfg::STAGES) & 1, abort, args.status)) break;
                    tc_fence_after();
                    const uint32_t v_s = base_u32 + Cfg::OFF_V + s * Cfg::KV_BYTES;
                    const uint32_t p_tmem = tmem + Cfg::TM_S + 64 * (v & 1);
                    #pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t b = smem_desc_sw128(v_s + kk * 2048, Cfg::KV_CHUNK, 1024);
                        mma_ts(tmem + Cfg::TM_O, p_tmem + kk * 8, b, IDESC_O, (v > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(smem_u32(&ctl->o_done));
                    mma_commit(smem_u32(&ctl->v_empty[s]));
                    if (v == L - 1) mma_commit(smem_u32(&ctl->o_final));
                }
            }
            // Drain: every MMA this thread issued has completed before TMEM is freed.
            mma_commit(smem_u32(&ctl->drain));
            mbar_wait_drain(smem_u32(&ctl->drain), 0);
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int row = tid;                       // 0..127 = TMEM lane
        const int half = row >> 6;                 // which query block of the pair
        const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
        const float sl2 = args.scale_log2;
        float m_run = -INFINITY;
        float l_run = 0.f;
        bool ok = true;
        for (int t = 0; t < L; ++t) {
            const int b = t & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl->s_full[b]), (t >> 1) & 1, abort, args.status));
            if (!ok) break;
            tc_fence_after();
            const int32_t e = list[t];
            const int j = e & 0x3fffffff;
            const bool kept = (e >> (30 + half)) & 1;        // uniform over the warp
            const uint32_t s_addr = tmem + lane_addr + Cfg::TM_S + 64 * b;
            uint32_t pk[32];
            if (kept) {
                uint32_t sr[64];
                tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                tmem_wait_ld();
                const int nvalid = min(64, args.N - j * 64);
                float smax = -INFINITY;
                #pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (c < nvalid) smax = fmaxf(smax, __uint_as_float(sr[c]));
                const float mb = smax * sl2;                  // scale > 0: max commutes
                const bool need = (m_run != -INFINITY) && (mb > m_run + 8.0f);
                if (__any_sync(0xffffffffu, need)) {
                    // O rescale: the PV product of step t-1 must be complete (t >= 1 here).
                    float f = 1.f;
                    if (need) { f = ex2_approx(m_run - mb); l_run *= f; m_run = mb; }
                    ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl->o_done), (t - 1) & 1, abort, args.status));
                    if (!ok) break;
                    tc_fence_after();
                    #pragma unroll 1
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t o[32];
                        tmem_ld32(tmem + lane_addr + Cfg::TM_O + c0, o);
                        tmem_wait_ld();
                        #pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
                        tmem_st32(tmem + lane_addr + Cfg::TM_O + c0, o);
                    }
                }
                if (m_run == -INFINITY) m_run = mb;
                const float neg_mu = (m_run == -INFINITY) ? 0.f : -m_run;
                float sum = 0.f;
                #pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    const float p0 = (c < nvalid) ? ex2_approx(fmaf(__uint_as_float(sr[c]), sl2, neg_mu)) : 0.f;
                    const float p1 = (c + 1 < nvalid) ? ex2_approx(fmaf(__uint_as_float(sr[c + 1]), sl2, neg_mu)) : 0.f;
                    sum += p0 + p1;
                    pk[c >> 1] = pack_bf16x2(p0, p1);
                }
                l_run += sum;
            } else {
                #pragma unroll
                for (int c = 0; c < 32; ++c) pk[c] = 0u;
            }
            tmem_st32(s_addr, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(smem_u32(&ctl->p_full[b]));
        }
        // ---- epilogue: O / l -> bf16
        if (ok && L > 0)
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
                if (L > 0) {
                    tmem_ld32(tmem + lane_addr + Cfg::TM_O + c0, o);
                    tmem_wait_ld();
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
