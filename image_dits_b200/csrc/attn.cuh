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
// A step is one union entry (64 keys): S_e = Q K_e^T is an M128 x N64
// product into one of two 64-column S buffers of TMEM, then O += P_e V_e.
// With two S buffers the product for entry e+1 runs while the softmax of
// entry e does, so the softmax warps find the next scores (nearly) ready
// instead of waiting for the PV and S products of a single-buffer chain; the
// N = 64 product runs at 2/3 of the N = 128 rate (M128 x N64 x K16: 48
// cycles against 64), which the overlap more than repays.
//
// Roles (256 threads, two CTAs per SM):
//   warps 0-3  softmax + epilogue: thread r owns query row r = TMEM lane r
//   warp 4     MMA issuer (one thread)
//   warp 5     TMA: K of the even entries (stage 0); Q is loaded once by
//              thread 0 as soon as the barriers exist
//   warp 6     TMA: K of the odd entries (stage 1)
//   warp 7     TMA: V of every entry (stage e mod 2)
// (one thread's TMA stream is served serially, so loads are spread over three
// issuing warps).  Shared memory: Q 32 KB, two 16 KB K stages and two 16 KB V
// stages, all 128-byte swizzled.  TMEM: O (d fp32 columns) and two 64-column
// S buffers; P (bf16) is written over the first 32 columns of its S buffer
// and read by the PV product straight from TMEM.  Issue order of the MMA
// thread: S_0, S_1, then per entry e: PV_e, S_{e+2} (S_{e+2} overwrites the
// buffer PV_e reads; the tensor pipe runs one thread's MMAs in order).  One
// completion barrier per product, as every tcgen05.commit (and every branch)
// between a thread's MMAs costs the issuing thread about 50 cycles: s_full[b]
// (S_e done: scores ready, K stage b free) and pv_done[b] (PV_e done: V stage
// b free, O holds entry e).
//
// Softmax (eqs. (2)-(4)) in fp32, log2 domain, per thread and entry: the 64
// scores are loaded once and P = 2^(s - m) is written in bf16 under the
// running max m as it stands, the row sum accumulated.  No max is taken
// unless the row has none yet or the entry's sum exceeds 2^24 (P stays a
// valid bf16 and O, l far inside fp32 below that); then m is raised to the
// entry's max, O rescaled in TMEM and P written again.  O and l always use
// the same m, so O / l is unchanged.  Before a rescale the warp
// waits for PV_{e-1} (barrier pv_done): S_e completing implies PV_{e-2}
// has, but PV_{e-1} may still run.
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
    static constexpr int KCH = D / 64;                     // 128-byte column chunks per row
    static constexpr uint32_t Q_CHUNK = 128 * 128;         // one 64-column chunk of Q (128 rows)
    static constexpr uint32_t Q_BYTES = Q_CHUNK * KCH;
    static constexpr uint32_t KB_CHUNK = 64 * 128;         // one 64-column chunk of a 64-key block
    static constexpr uint32_t KV_BLOCK = 64 * D * 2;       // one key block of K or V: [chunk][64 rows]
    static constexpr uint32_t TM_O = 0;
    static constexpr uint32_t TM_S = 128;                  // S buffer b at TM_S + 64 b
    static constexpr uint32_t TM_COLS = 256;
    static constexpr int THREADS = 256;
    static constexpr int MMA_WARP = 4;
    static constexpr int KA_WARP = 5;
    static constexpr int KB_WARP = 6;
    static constexpr int V_WARP = 7;
    // Shared memory: [align slack][Q][K stage 0, 1][V stage 0, 1][union list][control]
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + 2 * KV_BLOCK;
    static constexpr uint32_t OFF_LIST = OFF_V + 2 * KV_BLOCK;
    static constexpr uint32_t CONTROL_BYTES = 256;
    __host__ __device__ static size_t list_bytes(int Tb) { return ((size_t)Tb * 4 + 15) & ~(size_t)15; }
    __host__ __device__ static size_t smem_bytes(int Tb) { return 1024 + OFF_LIST + list_bytes(Tb) + CONTROL_BYTES; }
};

struct __align__(16) AttnCtl {
    uint64_t q_full;
    uint64_t k_full[2], v_full[2];
    uint64_t s_full[2], p_full[2], pv_done[2];
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
    int32_t sink_pairs;     // pairs holding a sink block (the last ones of a head): scheduled early
    float scale_log2;       // log2(e) / sqrt(D)
    int64_t col_capacity;   // checked build: bound of row_start + row_count (B*H*T_b^2)
};

// An entry's probability sum under a stale running max up to which its P is
// used as it is (P <= 2^24 in bf16, and O, l stay far inside fp32).
constexpr float kSumLimit = 16777216.f;

// 32 scores of one row -> 16 packed bf16 pairs of P = 2^(s*sl2 - m), adding
// the fp32 probabilities to sum4; x = s*sl2 - m and the sums run two lanes
// at a time (fma/add.f32x2).  `nvalid` < 32 masks the tail columns.
template <bool kMasked>
__device__ __forceinline__ void exp_chunk(const uint32_t (&s)[32], float sl2, float neg_mu, int nvalid,
                                          uint32_t (&pk)[16], float (&sum4)[4])
{
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
}

// max(acc, s[0..nvalid)) over one 32-score chunk, four independent chains.
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

    // ---- work item (bh, pair).  A head's sink pairs (full rows: the longest
    // items) are launched before its other pairs, so the CTAs in flight use
    // the K/V of about one head (L2-resident); for the last two heads both
    // heads' sink pairs come first, so the grid does not end on full rows.
    int64_t bh;
    int pair;
    {
        const int P = args.pairs, S = args.sink_pairs;
        const int64_t BH = gridDim.x / P;
        const int64_t x = blockIdx.x;
        const int64_t tail0 = (BH >= 2) ? (BH - 2) * P : 0;   // first block of the last two heads
        if (x < tail0 || BH < 2) {
            bh = x / P;
            const int u = (int)(x - bh * P);
            pair = (u < S) ? (P - 1 - u) : (u - S);
        } else {
            const int t = (int)(x - tail0);                    // 0 .. 2P - 1
            if (t < 2 * S) {
                bh = BH - 2 + t / S;
                pair = P - 1 - t % S;
            } else {
                const int v = t - 2 * S;                       // normal pairs of the two heads
                bh = BH - 2 + v / (P - S);
                pair = v % (P - S);
            }
        }
    }
    const int qb0 = 2 * pair;
    const bool has_b = (qb0 + 1) < Tb;
    const int64_t rA = bh * Tb + qb0;

    // The two CSR rows' extents and first entries (up to 2 x 256 per row),
    // read into registers before the set-up below so that their two dependent
    // round trips to memory overlap it.  (Checked build: a row outside the CSR
    // array, or a key block outside 0 .. T_b - 1, is reported and skipped.)
    auto row_len = [&](int64_t r) -> int {
        const int32_t cnt = args.row_count[r];
        const int len = min(max(cnt, 0), Tb);
        if (RF2_CHECKED && !in_range(cnt >= 0 && cnt <= Tb && args.row_start[r] >= 0 &&
                                     (int64_t)args.row_start[r] + cnt <= args.col_capacity))
            return 0;
        return len;
    };
    int lenA = 0, lenB = 0;
    const int32_t* srcA = args.col_idx;
    const int32_t* srcB = args.col_idx;
    int32_t first[4] = {-1, -1, -1, -1};               // entries tid and tid + 256 of rows A and B
    auto read_rows = [&]() {
        lenA = row_len(rA);
        srcA = args.col_idx + args.row_start[rA];
        if (has_b) {
            lenB = row_len(rA + 1);
            srcB = args.col_idx + args.row_start[rA + 1];
        }
        first[0] = (tid < lenA) ? srcA[tid] : -1;
        first[1] = (tid + Cfg::THREADS < lenA) ? srcA[tid + Cfg::THREADS] : -1;
        first[2] = (tid < lenB) ? srcB[tid] : -1;
        first[3] = (tid + Cfg::THREADS < lenB) ? srcB[tid + Cfg::THREADS] : -1;
    };
    if (warp != 0) read_rows();

    // ---- set-up: barriers, TMEM, union of the two CSR rows
    if (tid == 0) {
        mbar_init(smem_u32(&ctl->q_full), 1);
        #pragma unroll
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&ctl->k_full[b]), 1);
            mbar_init(smem_u32(&ctl->v_full[b]), 1);
            mbar_init(smem_u32(&ctl->s_full[b]), 1);
            mbar_init(smem_u32(&ctl->p_full[b]), 128);
            mbar_init(smem_u32(&ctl->pv_done[b]), 1);
        }
        mbar_init(smem_u32(&ctl->o_final), 1);
        mbar_init(smem_u32(&ctl->drain), 1);
        ctl->abort = 0;
        fence_mbar_init();
        // Q first: its load overlaps the set-up below (the Q region is not touched before)
        mbar_arrive_expect_tx(smem_u32(&ctl->q_full), Cfg::Q_BYTES);
        tma_load_4d(base_u32 + Cfg::OFF_Q, &tm_q, smem_u32(&ctl->q_full), 0, qb0 * 64, 0, (int)bh);
    }
    if (warp == Cfg::KA_WARP && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_kc);
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ctl->tmem_base), Cfg::TM_COLS);
        tmem_relinquish();
        read_rows();
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
    {
        auto set_bit = [&](uint32_t* bm, int32_t j) {
            if (in_range(j >= 0 && j < Tb) && j >= 0 && j < Tb) atomicOr(&bm[j >> 5], 1u << (j & 31));
        };
        if (tid < lenA) set_bit(bmA, first[0]);
        if (tid + Cfg::THREADS < lenA) set_bit(bmA, first[1]);
        if (tid < lenB) set_bit(bmB, first[2]);
        if (tid + Cfg::THREADS < lenB) set_bit(bmB, first[3]);
        for (int e = tid + 2 * Cfg::THREADS; e < lenA; e += Cfg::THREADS) set_bit(bmA, srcA[e]);
        for (int e = tid + 2 * Cfg::THREADS; e < lenB; e += Cfg::THREADS) set_bit(bmB, srcB[e]);
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
    volatile int* abort = &ctl->abort;

    // Key block of union entry e.
    auto block_of = [&](int e) -> int { return min(list[e] & 0x3fffffff, Tb - 1); };

    if (warp == Cfg::KA_WARP || warp == Cfg::KB_WARP) {
        // ------------------------------------------------ TMA: K of entries e = g, g + 2, ... into stage g
        if (lane == 0) {
            fence_proxy_async_smem();   // the K stages held the row bitmaps (generic accesses)
            const int g = (warp == Cfg::KA_WARP) ? 0 : 1;
            const uint32_t full = smem_u32(&ctl->k_full[g]);
            const uint32_t dst = base_u32 + Cfg::OFF_K + g * Cfg::KV_BLOCK;
            int issued = -1;
            for (int e = g, i = 0; e < L; e += 2, ++i) {
                // stage g is free once S_{e-2} is done
                if (i > 0 && !mbar_wait(smem_u32(&ctl->s_full[g]), (i - 1) & 1, abort, args.status)) break;
                const int j = block_of(e);
                mbar_arrive_expect_tx(full, Cfg::KV_BLOCK);
                for (int c = 0; c < Cfg::KCH; ++c)
                    tma_load_3d(dst + c * Cfg::KB_CHUNK, &tm_kc, full, c * 64, j * 64, (int)bh);
                issued = i;
            }
            // Drain: no TMA may still be writing shared memory when the CTA exits.
            if (g == 0) mbar_wait_drain(smem_u32(&ctl->q_full), 0);
            if (issued >= 0) mbar_wait_drain(full, issued & 1);
        }
    } else if (warp == Cfg::V_WARP) {
        // ------------------------------------------------ TMA: V of entry e into stage e mod 2
        if (lane == 0) {
            fence_proxy_async_smem();
            int issued = -1;                     // entries e <= issued were loaded
            for (int e = 0; e < L; ++e) {
                const int b = e & 1, i = e >> 1;
                // stage b is free once PV_{e-2} is done
                if (i > 0 && !mbar_wait(smem_u32(&ctl->pv_done[b]), (i - 1) & 1, abort, args.status)) break;
                mbar_arrive_expect_tx(smem_u32(&ctl->v_full[b]), Cfg::KV_BLOCK);
                tma_load_4d(base_u32 + Cfg::OFF_V + b * Cfg::KV_BLOCK, &tm_v, smem_u32(&ctl->v_full[b]), 0,
                            block_of(e) * 64, 0, (int)bh);
                issued = e;
            }
            // the last load of each stage: entries issued and issued - 1
            for (int e = max(issued - 1, 0); e <= issued; ++e)
                mbar_wait_drain(smem_u32(&ctl->v_full[e & 1]), (uint32_t)((e >> 1) & 1));
        }
    } else if (warp == Cfg::MMA_WARP) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, 0);
            constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, 1);
            // descriptors: only the start address (16-byte units, low 14 bits) changes
            const uint64_t dq = smem_desc_sw128(base_u32 + Cfg::OFF_Q, 16, 1024);
            const uint64_t dk = smem_desc_sw128(base_u32 + Cfg::OFF_K, 16, 1024);
            const uint64_t dv = smem_desc_sw128(base_u32 + Cfg::OFF_V, 64 * 128, 1024);
            // S_e = Q K_e^T into S buffer e mod 2
            auto issue_s = [&](int e) -> bool {
                const int b = e & 1;
                if (!mbar_wait(smem_u32(&ctl->k_full[b]), (e >> 1) & 1, abort, args.status)) return false;
                tc_fence_after();
                const uint64_t kb = dk + ((b * Cfg::KV_BLOCK) >> 4);
                #pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // 16 bf16 = 32 bytes per K step
                    const uint32_t off = ((kk >> 2) * Cfg::Q_CHUNK + (kk & 3) * 32) >> 4;
                    const uint32_t offk = ((kk >> 2) * Cfg::KB_CHUNK + (kk & 3) * 32) >> 4;
                    mma_ss(tmem + Cfg::TM_S + 64 * b, dq + off, kb + offk, IDESC_S, kk > 0 ? 1u : 0u);
                }
                mma_commit(smem_u32(&ctl->s_full[b]));
                return true;
            };
            bool ok = (L == 0) || mbar_wait(smem_u32(&ctl->q_full), 0, abort, args.status);
            tc_fence_after();
            for (int e = 0; ok && e < 2 && e < L; ++e) ok = issue_s(e);
            for (int e = 0; ok && e < L; ++e) {
                const int b = e & 1;
                const uint32_t par = (e >> 1) & 1;
                if (!mbar_wait(smem_u32(&ctl->p_full[b]), par, abort, args.status)) break;
                if (!mbar_wait(smem_u32(&ctl->v_full[b]), par, abort, args.status)) break;
                tc_fence_after();
                const uint64_t vb = dv + ((b * Cfg::KV_BLOCK) >> 4);
                #pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    // 16 keys per K step; V as the MN-major B operand (d chunks 8 KB apart)
                    mma_ts(tmem + Cfg::TM_O, tmem + Cfg::TM_S + 64 * b + kk * 8, vb + ((kk * 2048) >> 4), IDESC_O,
                           (e > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(smem_u32(&ctl->pv_done[b]));
                if (e == L - 1) mma_commit(smem_u32(&ctl->o_final));
                if (e + 2 < L) ok = issue_s(e + 2);
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
        const float sl2 = args.scale_log2;
        float m_run = -INFINITY;
        float l_run = 0.f;
        bool ok = true;
        for (int e = 0; e < L; ++e) {
            const int b = e & 1;
            const uint32_t s_row = tmem + lane_addr + Cfg::TM_S + 64 * b;
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl->s_full[b]), (e >> 1) & 1, abort, args.status));
            if (!ok) break;
            tc_fence_after();
            // kept flag and valid key count of the entry (uniform over the warp)
            const int32_t ent = list[e];
            const bool kept = (ent >> (30 + half)) & 1;
            const int nv = min(64, args.N - (ent & 0x3fffffff) * 64);
            float sum4[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pk[16];
            if (kept) {
                uint32_t a[32], c[32];
                tmem_ld32(s_row, a);
                tmem_ld32(s_row + 32, c);
                tmem_wait_ld();
                reg_fence(a);
                reg_fence(c);
                // P = 2^(s*sl2 - m) in bf16 over the first 32 columns of the buffer
                auto exps = [&](float neg_mu) {
                    #pragma unroll
                    for (int k = 0; k < 4; ++k) sum4[k] = 0.f;
                    if (nv == 64) exp_chunk<false>(a, sl2, neg_mu, 32, pk, sum4);
                    else exp_chunk<true>(a, sl2, neg_mu, nv, pk, sum4);
                    tmem_st16(s_row, pk);
                    if (nv == 64) exp_chunk<false>(c, sl2, neg_mu, 32, pk, sum4);
                    else exp_chunk<true>(c, sl2, neg_mu, nv - 32, pk, sum4);
                    tmem_st16(s_row + 16, pk);
                };
                // Fast path: the entry's probabilities under the running max as it
                // stands, with no max taken; it holds while their sum stays within
                // kSumLimit.  A row's first kept entry, or a sum above the limit
                // (or not finite), takes the entry's max instead, raises m (O
                // rescaled) and writes P again before the hand-off.
                bool slow = (m_run == -INFINITY);
                if (!slow) {
                    exps(-m_run);
                    slow = !((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]) <= kSumLimit);
                }
                if (__any_sync(0xffffffffu, slow)) {
                    float mb = m_run;
                    if (slow) {
                        float mx;
                        if (nv == 64) mx = max_chunk<false>(c, 32, max_chunk<false>(a, 32, -INFINITY));
                        else mx = max_chunk<true>(c, nv - 32, max_chunk<true>(a, nv, -INFINITY));
                        mb = mx * sl2;                     // scale > 0: max commutes
                    }
                    const bool resc = slow && (m_run != -INFINITY) && (mb > m_run);
                    if (__any_sync(0xffffffffu, resc)) {
                        // Rescale O once PV_{e-1} has completed (S_e done implies PV_{e-2} is).
                        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl->pv_done[(e - 1) & 1]),
                                                               (uint32_t)(((e - 1) >> 1) & 1), abort, args.status));
                        if (!ok) break;
                        tc_fence_after();
                        float f = 1.f;
                        if (resc) { f = ex2_approx(m_run - mb); l_run *= f; }
                        #pragma unroll 1
                        for (int c0 = 0; c0 < D; c0 += 32) {
                            uint32_t o[32];
                            tmem_ld32(tmem + lane_addr + Cfg::TM_O + c0, o);
                            tmem_wait_ld();
                            reg_fence(o);
                            #pragma unroll
                            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
                            tmem_st32(tmem + lane_addr + Cfg::TM_O + c0, o);
                        }
                    }
                    if (slow && (m_run == -INFINITY || mb > m_run)) m_run = mb;
                    exps(m_run == -INFINITY ? 0.f : -m_run);
                }
            } else {
                #pragma unroll
                for (int k = 0; k < 16; ++k) pk[k] = 0u;
                tmem_st16(s_row, pk);
                tmem_st16(s_row + 16, pk);
            }
            l_run += (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
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
