// Pooled scores and top-n selection for rows of a few thousand key blocks
// ("RainFusion2.0" section 3.2, eqs. (7)-(8), with the first-frame sink of
// section 3.4), without writing the score matrix.
//
// topn_codes_kernel: work item = (head, 128 query blocks).  The scores S^_ij =
// q^_i . k^_j of the item's rows come from the tensor cores (tcgen05
// kind::tf32, three hi/lo products: fp32 accuracy) in chunks of 128 key
// blocks, and each value is read out of TMEM exactly once by the thread that
// owns its row (TMEM lane = query block):
//  1. Bracket.  The row's scores against 64 sampled key blocks (one from each
//     of 64 equal stripes of the row, offset hashed from the item) come first;
//     sorted, their ranks pos -/+ 10 (pos = the n-th key's expected rank in
//     the sample) give a value bracket [lo, hi] that holds the n-th largest
//     score with high probability (widened by a quarter where it is clamped
//     at the end of the sample).
//  2. Codes.  Every score s becomes a 16-bit code floor(256 x), clamped to
//     0..65535, with x = 8 + 240 (s - lo) / (hi - lo): the bracket covers
//     coarse codes (the high byte) 8..247 in 240 steps of w = (hi - lo) / 240,
//     eight more steps on either side keep their order, and everything
//     further out shares code 0 or 65535.  The map is monotone, so a larger
//     code means a larger score.  The coarse and the fine (low) bytes go to
//     two workspace arrays (2 bytes per score instead of 4), with a histogram
//     of coarse >> 3 per row counted in registers on the way.
// topn_rows_kernel then selects from the codes, one thread per row, and lists
// the rare rows it cannot settle for topn_overflow_kernel (one CTA per row).
//
// The kept set is the top n under the order (score desc, j asc) of the
// tensor-core scores, except that keys of one 16-bit code (width w / 256) are
// ranked by j where that width is below 1e-6 (after the 1/sqrt(d) scale), and
// otherwise by an fp32 rescoring; keys whose scores differ by less than the
// tf32 hi/lo error (~1e-7) may be ranked either way.  All such keys lie inside
// the 1e-5 tie band of the selection.
#pragma once
#include "geometry.cuh"
#include "mask.cuh"
#include "ptx.cuh"

namespace rf2 {

template <int D>
struct TopnCfg {
    static constexpr int KC = D / 32;                   // 32-float (128-byte) slices of d
    static constexpr int NB = 128;                      // key blocks per accumulator chunk
    static constexpr int SAMPLE = 64;
    static constexpr uint32_t A_PART = 128 * 128;       // one slice of q^ (hi or lo): 128 rows x 128 B
    static constexpr uint32_t A_BYTES = KC * 2 * A_PART;
    static constexpr uint32_t B_PART = NB * 128;        // one slice of a k^ chunk (hi or lo)
    static constexpr uint32_t STAGE = 2 * B_PART;
    static constexpr int NSTAGE = 3;
    static constexpr uint32_t OFF_B = A_BYTES;
    static constexpr uint32_t OFF_CTL = OFF_B + NSTAGE * STAGE;
    static constexpr uint32_t TM_XCH = 2 * NB;          // TMEM columns of the brackets handed between the row sets
    static constexpr uint32_t SMEM = 1024 + OFF_CTL + 256;
    static constexpr int THREADS = 384;
    static constexpr int MAX_TB = 2048;                 // topn_overflow_kernel keeps a row's codes in registers
};

struct __align__(16) TopnCtl {
    uint64_t a_full, a_empty;
    uint64_t full[3], empty[3];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain;
    uint64_t xch_full[2];       // a bracket handed to the other row set
    uint32_t tmem_base;
    int32_t abort;
};
static_assert(sizeof(TopnCtl) <= 256, "control block");

// Per-row results of topn_codes_kernel that the selection kernels read.  Item
// it = (head, 128 query blocks); G = ceil(Tb / 32) groups of 32 key blocks.
//   codes  uint32 [items][8 G words][128 rows]: the coarse codes of a row's
//          keys, four per word, key 4 w + b in byte b of word w
//   fine   uint32, laid out as codes: the fine bytes
//   hist   uint32 [items][2 row sets][16][128 rows]: counts of code >> 3 over
//          the keys each set saw, bins 2 p (low half) and 2 p + 1 (high half)
//   width  float  [items][128 rows]: the value width of one code (unscaled)
struct TopnArgs {
    const float* means_hi;      // [2][BH][Tb][D] (queries, then keys)
    const float* means_lo;
    uint32_t* codes;
    uint32_t* fine;
    uint32_t* hist;
    float* width;
    int32_t* overflow;          // [0] = count, then rows with too many keys tied in their threshold code
    int32_t* row_start;
    int32_t* row_count;
    int32_t* col_idx;
    int* status;
    MaskGeo mg;
    int64_t BH;
    float tiny_width;           // code widths up to this are ties (unscaled score units)
    float tiny_width_fine;      // coarse widths up to this (256 tiny_width) make the fine codes ties
    float min_width;            // smallest bracket width (unscaled)
};

__host__ __device__ inline size_t topn_codes_words(int64_t items, int32_t Tb) { return (size_t)items * ((Tb + 31) / 32) * 128 * 8; }
__host__ __device__ inline size_t topn_overflow_words(int64_t rows) { return (size_t)rows + 1; }
__host__ __device__ inline size_t topn_hist_words(int64_t items) { return (size_t)items * 2 * 16 * 128; }

// Key block sampled from stripe e of S equal stripes of a row of Tb blocks,
// at an offset hashed from the item and the stripe.
__device__ __forceinline__ int topn_sample_col(uint32_t item, int e, int S, int Tb)
{
    const int s0 = (int)(((int64_t)e * Tb) / S), s1 = (int)(((int64_t)(e + 1) * Tb) / S);
    uint32_t h = item * 0x9E3779B1u ^ (uint32_t)e * 0x85EBCA77u;
    h ^= h >> 15;
    h *= 0x2C1B3C6Du;
    h ^= h >> 12;
    return s0 + (int)(h % (uint32_t)(s1 - s0));
}

// One bit per byte of w (bit i = byte i), taken from bit 7 of each byte of m.
__device__ __forceinline__ uint32_t byte_flags(uint32_t m)
{
    return ((((m >> 7) & 0x01010101u) * 0x00204081u) >> 21) & 0xFu;
}

// Bit i set iff byte i of w equals the byte replicated in y.
__device__ __forceinline__ uint32_t bytes_eq(uint32_t w, uint32_t y)
{
    const uint32_t x = w ^ y;
    const uint32_t nz = ((x & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | x;      // bit 7 of a byte: byte != 0
    return byte_flags(~nz);
}

// Bit i set iff byte i of w is >= the byte replicated in y (unsigned).
__device__ __forceinline__ uint32_t bytes_ge(uint32_t w, uint32_t y)
{
    const uint32_t H = 0x80808080u;
    const uint32_t d = (w | H) - (y & ~H);                // bit 7: low 7 bits of w >= those of y
    return byte_flags((w & ~y) | (~(w ^ y) & d));
}

// Byte k (0..31) of the eight words w[0..7], without indexing registers.
__device__ __forceinline__ uint32_t byte_of8(const uint32_t (&w)[8], int k)
{
    const int q = k >> 2;
    const uint32_t a01 = (q & 1) ? w[1] : w[0], a23 = (q & 1) ? w[3] : w[2];
    const uint32_t a45 = (q & 1) ? w[5] : w[4], a67 = (q & 1) ? w[7] : w[6];
    const uint32_t a03 = (q & 2) ? a23 : a01, a47 = (q & 2) ? a67 : a45;
    const uint32_t a = (q & 4) ? a47 : a03;
    return (a >> (8 * (k & 3))) & 255u;
}

// Scores and codes ("RainFusion2.0" section 3.2, eq. (7), on the tensor
// cores) for top-n selection; see the description at the top of this file.
// Roles (384 threads, one CTA per SM, persistent over items):
//   warps 0, 1   producers of the hi and lo parts: the item's q^ tile (TMA,
//                kept resident), the sampled k^ rows (one-row TMA boxes, two
//                rows per lane) and the k^ chunks (TMA)
//   warp 2       MMA issuer (one thread)
//   warps 4-7    row set 0, warps 8-11 row set 1: thread r of a set reads
//                TMEM lane r = query block m0 + r; the sets take alternate
//                accumulator chunks (chunk c goes to set c mod 2)
template <int D>
__global__ void __launch_bounds__(TopnCfg<D>::THREADS, 1)
topn_codes_kernel(const __grid_constant__ CUtensorMap tm_a_hi, const __grid_constant__ CUtensorMap tm_a_lo,
                  const __grid_constant__ CUtensorMap tm_b_hi, const __grid_constant__ CUtensorMap tm_b_lo,
                  const __grid_constant__ CUtensorMap tm_r_hi, const __grid_constant__ CUtensorMap tm_r_lo,
                  const TopnArgs args)
{
    using Cfg = TopnCfg<D>;
    constexpr int KC = Cfg::KC;
    constexpr int NB = Cfg::NB;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_u32 - raw_u32);
    TopnCtl* ctl = reinterpret_cast<TopnCtl*>(base + Cfg::OFF_CTL);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const MaskGeo mg = args.mg;
    const int Tb = mg.Tb;
    const int n = mg.n_keep;
    const int64_t BH = args.BH;
    const int mtiles = (Tb + 127) / 128;
    const int nch = (Tb + NB - 1) / NB;
    const int G = (Tb + 31) / 32;
    const int S = min(Cfg::SAMPLE, Tb);
    const int64_t items = BH * mtiles;
    const int my_items = (blockIdx.x < items) ? (int)((items - 1 - blockIdx.x) / gridDim.x) + 1 : 0;
    const int row_end = min(mg.sink_first, Tb);          // rows that select (the rest keep every block)
    auto needs_mma = [&](int m0) -> bool { return m0 < row_end && n < Tb; };

    if (tid == 0) {
        mbar_init(smem_u32(&ctl->a_full), 2);
        mbar_init(smem_u32(&ctl->a_empty), 1);
        for (int i = 0; i < Cfg::NSTAGE; ++i) {
            mbar_init(smem_u32(&ctl->full[i]), 2);
            mbar_init(smem_u32(&ctl->empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&ctl->acc_full[i]), 1);
            mbar_init(smem_u32(&ctl->acc_empty[i]), 128);
        }
        mbar_init(smem_u32(&ctl->drain), 1);
        mbar_init(smem_u32(&ctl->xch_full[0]), 128);
        mbar_init(smem_u32(&ctl->xch_full[1]), 128);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ctl->tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    volatile int* abort = &ctl->abort;

    if (warp == 0 || warp == 1) {
        // ------------------------------------------------ producers (warp 0: hi parts, warp 1: lo parts)
        const int part = warp;
        const CUtensorMap* ta = part ? &tm_a_lo : &tm_a_hi;
        const CUtensorMap* tb = part ? &tm_b_lo : &tm_b_hi;
        const CUtensorMap* tr = part ? &tm_r_lo : &tm_r_hi;
        int step = 0, a_use = 0, a_last = -1;
        int last_use[Cfg::NSTAGE] = {-1, -1, -1};
        bool last_tma[Cfg::NSTAGE] = {false, false, false};
        bool ok = true;
        for (int it = 0; ok && it < my_items; ++it) {
            const int64_t item = blockIdx.x + (int64_t)it * gridDim.x;
            const int64_t bh = item / mtiles;
            const int m0 = (int)(item % mtiles) * 128;
            if (!needs_mma(m0)) continue;
            const int krow0 = (int)(BH * Tb + bh * Tb);
            // sampled key blocks of rows lane and lane + 32 of the sample
            const int jA = (lane < S) ? topn_sample_col((uint32_t)item, lane, S, Tb) : 0;
            const int jB = (lane + 32 < S) ? topn_sample_col((uint32_t)item, lane + 32, S, Tb) : 0;
            if (a_use > 0 &&
                !__all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl->a_empty), (a_use - 1) & 1, abort, args.status))) {
                ok = false;
                break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(smem_u32(&ctl->a_full), KC * Cfg::A_PART);
                for (int c = 0; c < KC; ++c)
                    tma_load_2d(base_u32 + (2 * c + part) * Cfg::A_PART, ta, smem_u32(&ctl->a_full), c * 32,
                                (int)(bh * Tb + m0));
            }
            a_last = a_use++;
            // the sampled key blocks, one stage per slice of d: a one-row TMA box per
            // sampled block (the swizzle follows the destination address, so the
            // rows land in the same layout as a full box)
            for (int c = 0; c < KC; ++c, ++step) {
                const int st = step % Cfg::NSTAGE, use = step / Cfg::NSTAGE;
                if (use > 0 &&
                    !__all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl->empty[st]), (use - 1) & 1, abort, args.status))) {
                    ok = false;
                    break;
                }
                const uint32_t dst = base_u32 + Cfg::OFF_B + st * Cfg::STAGE + part * Cfg::B_PART;
                if (lane == 0) mbar_arrive_expect_tx(smem_u32(&ctl->full[st]), (uint32_t)S * 128u);
                __syncwarp();
                if (lane < S) tma_load_2d(dst + lane * 128, tr, smem_u32(&ctl->full[st]), c * 32, krow0 + jA);
                if (lane + 32 < S) tma_load_2d(dst + (lane + 32) * 128, tr, smem_u32(&ctl->full[st]), c * 32, krow0 + jB);
                last_use[st] = use;
                last_tma[st] = true;
            }
            if (!ok) break;
            // the item's key blocks, chunk by chunk
            for (int q = 0; ok && q < nch; ++q)
                for (int c = 0; c < KC; ++c, ++step) {
                    const int st = step % Cfg::NSTAGE, use = step / Cfg::NSTAGE;
                    if (use > 0 &&
                        !__all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl->empty[st]), (use - 1) & 1, abort, args.status))) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        mbar_arrive_expect_tx(smem_u32(&ctl->full[st]), Cfg::B_PART);
                        tma_load_2d(base_u32 + Cfg::OFF_B + st * Cfg::STAGE + part * Cfg::B_PART, tb,
                                    smem_u32(&ctl->full[st]), c * 32, krow0 + q * NB);
                    }
                    last_use[st] = use;
                    last_tma[st] = true;
                }
        }
        // Drain: only the last use of a stage (and of the q^ tile) can still be in flight.
        if (lane == 0) {
            if (a_last >= 0) mbar_wait_drain(smem_u32(&ctl->a_full), a_last & 1);
            for (int st = 0; st < Cfg::NSTAGE; ++st)
                if (last_use[st] >= 0 && last_tma[st]) mbar_wait_drain(smem_u32(&ctl->full[st]), last_use[st] & 1);
        }
    } else if (warp == 2) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int step = 0, chunk = 0, a_use = 0;
            bool ok = true;
            // Shared-memory descriptors: the 14-bit start address (16-byte units) is
            // the only field that changes, so a K step adds (32 bytes >> 4) = 2.
            const uint64_t d_a = smem_desc_sw128(base_u32, 16, 1024);
            const uint64_t d_b = smem_desc_sw128(base_u32 + Cfg::OFF_B, 16, 1024);
            for (int it = 0; ok && it < my_items; ++it) {
                const int64_t item = blockIdx.x + (int64_t)it * gridDim.x;
                const int m0 = (int)(item % mtiles) * 128;
                if (!needs_mma(m0)) continue;
                if (!mbar_wait(smem_u32(&ctl->a_full), a_use & 1, abort, args.status)) { ok = false; break; }
                ++a_use;
                tc_fence_after();
                for (int q = 0; ok && q <= nch; ++q, ++chunk) {
                    const int a = chunk & 1;
                    if (chunk >= 2 && !mbar_wait(smem_u32(&ctl->acc_empty[a]), ((chunk >> 1) - 1) & 1, abort, args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int N = (q == 0) ? ((S + 15) & ~15) : NB;        // q = 0: the sample
                    const uint32_t idesc = idesc_tf32_f32(128, N);
                    const uint32_t d_tmem = tmem + a * NB;
                    for (int c = 0; c < KC; ++c, ++step) {
                        const int st = step % Cfg::NSTAGE;
                        if (!mbar_wait(smem_u32(&ctl->full[st]), (step / Cfg::NSTAGE) & 1, abort, args.status)) { ok = false; break; }
                        tc_fence_after();
                        const uint64_t ah = d_a + ((2 * c * Cfg::A_PART) >> 4), al = ah + (Cfg::A_PART >> 4);
                        const uint64_t bhd = d_b + ((st * Cfg::STAGE) >> 4), bld = bhd + (Cfg::B_PART >> 4);
                        #pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {                   // 8 floats = 32 bytes per K step
                            const uint32_t first = (c == 0 && ks == 0) ? 0u : 1u;
                            mma_ss_tf32(d_tmem, ah + 2 * ks, bhd + 2 * ks, idesc, first);
                            mma_ss_tf32(d_tmem, ah + 2 * ks, bld + 2 * ks, idesc, 1u);
                            mma_ss_tf32(d_tmem, al + 2 * ks, bhd + 2 * ks, idesc, 1u);
                        }
                        mma_commit(smem_u32(&ctl->empty[st]));
                    }
                    if (ok) mma_commit(smem_u32(&ctl->acc_full[a]));
                }
                if (ok) mma_commit(smem_u32(&ctl->a_empty));
            }
            mma_commit(smem_u32(&ctl->drain));
            mbar_wait_drain(smem_u32(&ctl->drain), 0);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ row sets
        const int set = (warp >= 8) ? 1 : 0;
        const int wq = warp & 3;                               // TMEM lane quarter
        const int rl = wq * 32 + lane;                         // row within the item
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        int chunk = 0, nitem = 0;
        bool ok = true;
        for (int it = 0; ok && it < my_items; ++it) {
            const int64_t item = blockIdx.x + (int64_t)it * gridDim.x;
            const int m0 = (int)(item % mtiles) * 128;
            if (!needs_mma(m0)) continue;
            const int i = m0 + rl;
            const bool active = i < row_end;                   // a non-sink row that selects
            // ---- bracket from the sampled scores (the set holding the sample chunk
            // sorts them and hands the bracket to the other set: both sets reach row
            // r through TMEM lane r, so it passes through two TMEM columns)
            const int xs = nitem & 1;
            const uint32_t xpar = (uint32_t)(nitem >> 1) & 1u;
            const uint32_t xcol = tmem + lane_addr + Cfg::TM_XCH + 2 * xs;
            ++nitem;
            float2 br;
            if ((chunk & 1) == set) {
                const int a = chunk & 1;
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl->acc_full[a]), (chunk >> 1) & 1, abort, args.status));
                if (!ok) break;
                tc_fence_after();
                uint32_t r0[32], r1[32];
                tmem_ld32(tmem + lane_addr + a * NB, r0);
                tmem_ld32(tmem + lane_addr + a * NB + 32, r1);
                tmem_wait_ld();
                reg_fence(r0);
                reg_fence(r1);
                tc_fence_before();
                mbar_arrive(smem_u32(&ctl->acc_empty[a]));
                float v[64];
                #pragma unroll
                for (int k = 0; k < 32; ++k) {
                    v[k] = (k < S) ? __uint_as_float(r0[k]) : -INFINITY;
                    v[k + 32] = (k + 32 < S) ? __uint_as_float(r1[k]) : -INFINITY;
                }
                // bitonic sort, descending
                #pragma unroll
                for (int kk = 2; kk <= 64; kk <<= 1)
                    #pragma unroll
                    for (int jj = kk >> 1; jj > 0; jj >>= 1)
                        #pragma unroll
                        for (int x = 0; x < 64; ++x) {
                            const int y = x ^ jj;
                            if (y > x) {
                                const float p = v[x], q = v[y];
                                const bool desc = (x & kk) == 0;
                                v[x] = desc ? fmaxf(p, q) : fminf(p, q);
                                v[y] = desc ? fminf(p, q) : fmaxf(p, q);
                            }
                        }
                const int pos = (int)(((int64_t)n * S) / Tb);
                const int ih = pos - 10, il = pos + 10;
                const int ihc = max(ih, 0), ilc = min(il, S - 1);
                float hi = v[0], lo = v[0];
                #pragma unroll
                for (int k = 0; k < 64; ++k) {
                    hi = (k == ihc) ? v[k] : hi;
                    lo = (k == ilc) ? v[k] : lo;
                }
                const float wd = hi - lo;
                if (ih < 0) hi += 0.25f * wd;
                if (il > S - 1) lo -= 0.25f * wd;
                if (!(hi - lo >= args.min_width)) hi = lo + args.min_width;
                br = make_float2(lo, hi);
                uint32_t xv[2] = {__float_as_uint(lo), __float_as_uint(hi)};
                tmem_st2(xcol, xv);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(smem_u32(&ctl->xch_full[xs]));
            } else {
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl->xch_full[xs]), xpar, abort, args.status));
                if (!ok) break;
                tc_fence_after();
                uint32_t xv[2];
                tmem_ld2(xcol, xv);
                tmem_wait_ld();
                reg_fence(xv);
                br = make_float2(__uint_as_float(xv[0]), __uint_as_float(xv[1]));
            }
            ++chunk;
            // 16-bit code floor(256 x), x = 8 + 240 (s - lo) / (hi - lo); the
            // conversion to unsigned saturates below at 0 (and maps NaN to 0)
            const float sc = 61440.f / (br.y - br.x);
            const float off = 2048.f - br.x * sc;
            auto code_of = [&](float sv) -> uint32_t { return min(__float2uint_rd(fmaf(sv, sc, off)), 65535u); };
            if (set == 0 && active) args.width[item * 128 + rl] = (br.y - br.x) * (1.f / 240.f);

            // ---- codes, and a histogram of code >> 3 (32 bins, registers).  The
            // histogram is bit-sliced: for 32 keys at a time the five bits of
            // code >> 3 become five 32-bit planes (bit k = key k), and a bin's
            // count is the popcount of the AND of its planes (or their complements).
            uint32_t hist[32];
            #pragma unroll
            for (int b = 0; b < 32; ++b) hist[b] = 0u;
            uint32_t* crow = args.codes + (size_t)item * G * 8 * 128 + rl;           // word k at k * 128
            uint32_t* frow = args.fine + (size_t)item * G * 8 * 128 + rl;
            for (int q = 0; q < nch; ++q, ++chunk) {
                if ((chunk & 1) != set) continue;
                const int a2 = chunk & 1;
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl->acc_full[a2]), (chunk >> 1) & 1, abort, args.status));
                if (!ok) break;
                tc_fence_after();
                #pragma unroll 1
                for (int g = 0; g < NB / 32; ++g) {
                    const int j0 = q * NB + g * 32;
                    if (j0 >= Tb) break;                        // uniform
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_addr + a2 * NB + g * 32, r);
                    tmem_wait_ld();
                    reg_fence(r);
                    uint32_t wv[8], fv[8];
                    #pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t c0 = code_of(__uint_as_float(r[4 * k])), c1 = code_of(__uint_as_float(r[4 * k + 1]));
                        const uint32_t c2 = code_of(__uint_as_float(r[4 * k + 2])), c3 = code_of(__uint_as_float(r[4 * k + 3]));
                        const uint32_t p01 = __byte_perm(c0, c1, 0x5410), p23 = __byte_perm(c2, c3, 0x5410);
                        wv[k] = __byte_perm(p01, p23, 0x7531);          // high bytes: coarse codes
                        fv[k] = __byte_perm(p01, p23, 0x6420);          // low bytes: fine codes
                    }
                    if (active) {
                        uint32_t* dst = crow + (size_t)(j0 >> 2) * 128;
                        uint32_t* dsf = frow + (size_t)(j0 >> 2) * 128;
                        #pragma unroll
                        for (int k = 0; k < 8; ++k) { dst[k * 128] = wv[k]; dsf[k * 128] = fv[k]; }
                    }
                    const int nv = min(32, Tb - j0);
                    const uint32_t vm = (nv >= 32) ? 0xffffffffu : ((1u << nv) - 1u);
                    uint32_t pl[5];
                    #pragma unroll
                    for (int p = 0; p < 5; ++p) {
                        uint32_t x = 0;
                        #pragma unroll
                        for (int k = 0; k < 8; ++k) x |= byte_flags(wv[k] << (4 - p)) << (4 * k);
                        pl[p] = x;
                    }
                    uint32_t t1[2] = {vm & ~pl[4], vm & pl[4]};
                    uint32_t t2[4], t3[8], t4[16];
                    #pragma unroll
                    for (int b = 0; b < 2; ++b) { t2[2 * b] = t1[b] & ~pl[3]; t2[2 * b + 1] = t1[b] & pl[3]; }
                    #pragma unroll
                    for (int b = 0; b < 4; ++b) { t3[2 * b] = t2[b] & ~pl[2]; t3[2 * b + 1] = t2[b] & pl[2]; }
                    #pragma unroll
                    for (int b = 0; b < 8; ++b) { t4[2 * b] = t3[b] & ~pl[1]; t4[2 * b + 1] = t3[b] & pl[1]; }
                    #pragma unroll
                    for (int b = 0; b < 16; ++b) {
                        hist[2 * b] += __popc(t4[b] & ~pl[0]);
                        hist[2 * b + 1] += __popc(t4[b] & pl[0]);
                    }
                }
                tc_fence_before();
                mbar_arrive(smem_u32(&ctl->acc_empty[a2]));
            }
            if (!ok) break;
            if (active) {
                uint32_t* hd = args.hist + ((size_t)item * 2 + set) * 16 * 128 + rl;
                #pragma unroll
                for (int p = 0; p < 16; ++p) hd[p * 128] = hist[2 * p] | (hist[2 * p + 1] << 16);
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

// Selection for the rows topn_rows_kernel lists (eq. (8) and section 3.4):
// one CTA per row.  Every warp reads the row's coarse codes (lane l holds the
// l-th of 32 contiguous slices in registers) and finds, as topn_rows_kernel
// does, the bin b* of coarse >> 3 holding the n-th largest code (suffix sums
// of the two row sets' histograms, one bin per lane), then the code c* and
// need of its m keys.  If some keys of c* are dropped and the code is not
// narrower than the tie width (a tie: the lowest j are kept), the CTA scores
// the keys of c* again exactly in fp32 from the full means (q^ = hi + lo,
// k^ = hi + lo; a warp shares each dot product over d, the warps split the
// keys), and warp 0 keeps the need best by (score desc, j asc) (radix
// select).  Warp 0 then writes the row: the kept keys below the sink columns,
// ascending (a warp scan of the lanes' counts gives every lane its output
// positions), then the sink columns.  The listed rows are the few whose
// threshold code holds too many keys for topn_rows_kernel, most of them rows
// whose sampled bracket missed the threshold (their c* is a saturated code).
template <int D>
__global__ void __launch_bounds__(512) topn_overflow_kernel(const TopnArgs args)
{
    constexpr int E = D / 32;                              // q^ elements per lane in a dot product
    constexpr int WMAX = 16;                               // code words per lane (T_b <= 2048)
    constexpr int KB = 16;                                 // keys a warp scores at a time
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const MaskGeo mg = args.mg;
    const int Tb = mg.Tb, n = mg.n_keep;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int mtiles = (Tb + 127) / 128;
    const int G = (Tb + 31) / 32;
    const int W8 = 8 * G;                                  // code words per row
    const int WPL = (W8 + 31) / 32;                        // words per lane
    const int row_end = min(mg.sink_first, Tb);
    const int sf = mg.sink_first;                          // <= Tb
    int32_t* mem_j = reinterpret_cast<int32_t*>(smem_raw);             // [Tb]: keys of c*, then kept flags
    uint32_t* mem_k = reinterpret_cast<uint32_t*>(mem_j + Tb);         // [Tb]: their scores (order keys)
    uint32_t* hist = mem_k + Tb;                                       // [256]: radix bins
    const int64_t nrows = *reinterpret_cast<volatile const int32_t*>(args.overflow);
    const int w0 = lane * WPL;                             // first word of this lane
    for (int64_t idx = blockIdx.x; idx < nrows; idx += gridDim.x) {
        const int64_t row = args.overflow[1 + idx];
        const int64_t bh = row / Tb;
        const int i = (int)(row - bh * Tb);
        const int64_t rs = row_offset(mg, bh, i);
        int32_t* out = args.col_idx + rs;
        if (i >= row_end || n >= Tb) {                     // not listed by topn_rows_kernel; kept for safety
            if (warp == 0) {
                for (int j = lane; j < Tb; j += 32) csr_put(out, j, j, rs, mg.col_capacity);
                if (lane == 0) { args.row_start[row] = (int32_t)rs; args.row_count[row] = Tb; }
            }
            continue;
        }
        const int64_t item = bh * mtiles + i / 128;
        const int rl = i & 127;
        // 1. bin b*: lane b holds bin b
        const uint32_t* hs = args.hist + (size_t)item * 2 * 16 * 128 + rl;
        const int hb = (int)(((hs[(lane >> 1) * 128] >> (16 * (lane & 1))) & 0xFFFFu) +
                             ((hs[16 * 128 + (lane >> 1) * 128] >> (16 * (lane & 1))) & 0xFFFFu));
        int suf = hb;                                      // sum over bins >= lane
        #pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_down_sync(0xffffffffu, suf, o);
            if (lane + o < 32) suf += v;
        }
        const uint32_t reach = __ballot_sync(0xffffffffu, suf >= n);     // bins b with count(>= b) >= n
        const int bstar = 31 - __clz(reach);
        const int need_in = n - __shfl_sync(0xffffffffu, suf - hb, bstar);
        // the lane's code words and the bytes of each inside the row
        const uint32_t* cr = args.codes + ((size_t)item * W8 + w0) * 128 + rl;      // word k at k * 128
        uint32_t w[WMAX];
        uint32_t vn = 0;                                   // bit 4 k + b: byte b of word k is a key of the row
        #pragma unroll
        for (int k = 0; k < WMAX; ++k) {
            const int wi = w0 + k;
            w[k] = (k < WPL && wi < W8) ? cr[(size_t)k * 128] : 0u;
            const int nv = Tb - 4 * wi;
            const uint32_t v4 = (k >= WPL || nv <= 0) ? 0u : (nv >= 4 ? 0xFu : ((1u << nv) - 1u));
            if (k < 8) vn |= v4 << (4 * k);
        }
        uint32_t vn2 = 0;                                  // words 8..15
        #pragma unroll
        for (int k = 8; k < WMAX; ++k) {
            const int wi = w0 + k;
            const int nv = Tb - 4 * wi;
            const uint32_t v4 = (k >= WPL || nv <= 0) ? 0u : (nv >= 4 ? 0xFu : ((1u << nv) - 1u));
            vn2 |= v4 << (4 * (k - 8));
        }
        auto vnib = [&](int k) -> uint32_t { return (k < 8) ? ((vn >> (4 * k)) & 0xFu) : ((vn2 >> (4 * (k - 8))) & 0xFu); };
        // 2. counts of the eight codes of bin b*
        uint32_t cnt[8];
        #pragma unroll
        for (int k = 0; k < 8; ++k) cnt[k] = 0u;
        const uint32_t pat_bin = (uint32_t)bstar * 0x08080808u;
        #pragma unroll
        for (int k = 0; k < WMAX; ++k) {
            uint32_t M = bytes_eq(w[k] & 0xF8F8F8F8u, pat_bin) & vnib(k);
            while (M) {
                const int b = __ffs(M) - 1;
                M &= M - 1;
                const uint32_t sub = (w[k] >> (8 * b)) & 7u;
                #pragma unroll
                for (int x = 0; x < 8; ++x) cnt[x] += (sub == (uint32_t)x);
            }
        }
        int sub = 0, need = need_in, m = 0;
        {
            int cum = 0;
            bool found = false;
            #pragma unroll
            for (int x = 7; x >= 0; --x) {
                const int h = __reduce_add_sync(0xffffffffu, cnt[x]);
                if (!found && cum + h >= need_in) { found = true; sub = x; need = need_in - cum; m = h; }
                cum += h;
            }
        }
        const uint32_t cstar = (uint32_t)(bstar * 8 + sub);
        const bool partial = need < m;
        const bool tiny = cstar > 0 && cstar < 255 && args.width[item * 128 + rl] <= args.tiny_width;
        const bool rank_exact = partial && !tiny;
        const uint32_t pat_eq = cstar * 0x01010101u;
        uint32_t eqm = 0, eqm2 = 0;                        // keys of code c*, as for vn / vn2
        #pragma unroll
        for (int k = 0; k < WMAX; ++k) {
            const uint32_t e4 = bytes_eq(w[k], pat_eq) & vnib(k);
            if (k < 8) eqm |= e4 << (4 * k); else eqm2 |= e4 << (4 * (k - 8));
        }
        // index of this lane's first key of c* among the row's (ascending j)
        const int ceq = __popc(eqm) + __popc(eqm2);
        int e_first = ceq;
        #pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, e_first, o);
            if (lane >= o) e_first += v;
        }
        e_first -= ceq;
        // 3. exact scores of the keys of code c*, and the need best of them
        if (rank_exact) {
            if (warp == 0) {
                int at = e_first;
                uint32_t M = eqm;
                while (M) { const int b = __ffs(M) - 1; M &= M - 1; mem_j[at++] = 4 * w0 + b; }
                M = eqm2;
                while (M) { const int b = __ffs(M) - 1; M &= M - 1; mem_j[at++] = 4 * w0 + 32 + b; }
            }
            __syncthreads();
            const int64_t qr = bh * Tb + i, kr0 = args.BH * Tb + bh * Tb;
            float qv[E];
            #pragma unroll
            for (int u = 0; u < E; ++u) qv[u] = args.means_hi[qr * D + E * lane + u] + args.means_lo[qr * D + E * lane + u];
            for (int e0 = warp * KB; e0 < m; e0 += nwarps * KB) {
                float part[KB];
                #pragma unroll
                for (int u = 0; u < KB; ++u) {
                    const int j = mem_j[min(e0 + u, m - 1)];
                    const float* kh = args.means_hi + (kr0 + j) * D + E * lane;
                    const float* kl = args.means_lo + (kr0 + j) * D + E * lane;
                    float a = 0.f;
                    if (E == 4) {
                        const float4 h4 = __ldcg(reinterpret_cast<const float4*>(kh));
                        const float4 l4 = __ldcg(reinterpret_cast<const float4*>(kl));
                        a = fmaf(qv[0], h4.x + l4.x, a);
                        a = fmaf(qv[1 % E], h4.y + l4.y, a);
                        a = fmaf(qv[2 % E], h4.z + l4.z, a);
                        a = fmaf(qv[3 % E], h4.w + l4.w, a);
                    } else {
                        const float2 h2 = __ldcg(reinterpret_cast<const float2*>(kh));
                        const float2 l2 = __ldcg(reinterpret_cast<const float2*>(kl));
                        a = fmaf(qv[0], h2.x + l2.x, a);
                        a = fmaf(qv[1 % E], h2.y + l2.y, a);
                    }
                    part[u] = a;
                }
                #pragma unroll
                for (int u = 0; u < KB; ++u) {
                    #pragma unroll
                    for (int o = 16; o > 0; o >>= 1) part[u] += __shfl_xor_sync(0xffffffffu, part[u], o);
                }
                if (lane < KB && e0 + lane < m) {
                    float mine = part[0];
                    #pragma unroll
                    for (int u = 1; u < KB; ++u) mine = (lane == u) ? part[u] : mine;
                    mem_k[e0 + lane] = float_order_key(mine);
                }
            }
            __syncthreads();
            if (warp == 0) {
                uint32_t kmin = 0xffffffffu, kmax = 0u;
                for (int e = lane; e < m; e += 32) { kmin = min(kmin, mem_k[e]); kmax = max(kmax, mem_k[e]); }
                kmin = __reduce_min_sync(0xffffffffu, kmin);
                kmax = __reduce_max_sync(0xffffffffu, kmax);
                int eq_left;
                const uint32_t thr = radix_kth(mem_k, m, need, kmin, kmax, hist, lane, eq_left);
                for (int e0 = 0; e0 < m; e0 += 32) {
                    const int e = e0 + lane;
                    const uint32_t kk = (e < m) ? mem_k[e] : 0u;
                    const bool eq = (e < m) && kk == thr;
                    const uint32_t eb = __ballot_sync(0xffffffffu, eq);
                    const int er = __popc(eb & ((1u << lane) - 1u));
                    if (e < m) mem_j[e] = (kk > thr || (eq && er < eq_left)) ? 1 : 0;
                    eq_left -= __popc(eb);
                }
                __syncwarp();
            }
        }
        // 4. output by warp 0: kept keys below the sink columns, then the sink columns
        if (warp == 0) {
            const uint32_t y_gt = (cstar < 255u) ? (cstar + 1) * 0x01010101u : 0u;
            uint32_t keep = 0, keep2 = 0;
            int e = e_first;
            #pragma unroll
            for (int k = 0; k < WMAX; ++k) {
                uint32_t kp = ((cstar < 255u) ? bytes_ge(w[k], y_gt) : 0u) & vnib(k);
                uint32_t Eq = ((k < 8) ? (eqm >> (4 * k)) : (eqm2 >> (4 * (k - 8)))) & 0xFu;
                if (partial) {
                    while (Eq) {
                        const int b = __ffs(Eq) - 1;
                        Eq &= Eq - 1;
                        const bool take = rank_exact ? (mem_j[e] != 0) : (e < need);
                        kp |= (uint32_t)take << b;
                        ++e;
                    }
                } else {
                    kp |= Eq;
                }
                const int j0 = 4 * (w0 + k);
                if (j0 + 4 > sf) kp &= (j0 >= sf) ? 0u : ((1u << (sf - j0)) - 1u);
                if (k < 8) keep |= kp << (4 * k); else keep2 |= kp << (4 * (k - 8));
            }
            const int c = __popc(keep) + __popc(keep2);
            int at = c;
            #pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, at, o);
                if (lane >= o) at += v;
            }
            const int total = __shfl_sync(0xffffffffu, at, 31);
            at -= c;
            while (keep) { const int b = __ffs(keep) - 1; keep &= keep - 1; csr_put(out, at++, 4 * w0 + b, rs, mg.col_capacity); }
            while (keep2) { const int b = __ffs(keep2) - 1; keep2 &= keep2 - 1; csr_put(out, at++, 4 * w0 + 32 + b, rs, mg.col_capacity); }
            for (int j = sf + lane; j < Tb; j += 32) csr_put(out, total + (j - sf), j, rs, mg.col_capacity);
            if (lane == 0) { args.row_start[row] = (int32_t)rs; args.row_count[row] = total + (Tb - sf); }
        }
        __syncthreads();
    }
}

// Selection from the codes (eq. (8) and section 3.4), one thread per
// query-block row: a CTA of one warp takes 32 rows of an item.  Per row:
//   1. The bin b* of coarse >> 3 that holds the n-th largest code (suffix sums
//      of the two row sets' histograms).
//   2. One pass over the row's coarse codes (word-major layout: the warp's
//      loads are coalesced; four groups of 32 keys in flight): coarse codes
//      above bin b* set their bits in the row's bitmap at once; the keys of
//      bin b* (about a dozen) are kept aside with their coarse code.  The fine
//      bytes are read only for the keys of c* that step 3 ranks.
//   3. From those, the coarse code c* holding the n-th largest and how many
//      keys of c* are kept (need of m); keys of bin b* above c* are kept.  If
//      some keys of c* are dropped (need < m): where a coarse code is narrower
//      than the tie width the lowest j are kept; otherwise the keys of c* are
//      ranked by (fine code desc, j asc); where the need-th and the next share
//      a fine code wider than the tie width, the keys of that fine code (up to
//      4) are ranked again by exact fp32 scores, then j.  A row with more than
//      64 keys in bin b*, more than 16 keys of c* to rank, more than 4 keys
//      tied in the fine code, or its threshold in a saturated code (0 or 255:
//      the bracket missed) is listed for topn_overflow_kernel.
//   4. Each thread writes its own row's kept keys below the sink columns (the
//      kept bits of its bitmap in ascending order), the 32 rows in parallel;
//      the warp then writes the sink columns of each row, and all of a sink
//      row (or of every row at keep = 1), one row at a time, coalesced.
template <int D>
__global__ void __launch_bounds__(32, 12) topn_rows_kernel(const TopnArgs args)
{
    constexpr int BCAP = 64;                               // keys of bin b* kept aside per row
    constexpr int RCAP = 16;                               // keys of code c* ranked per row
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const MaskGeo mg = args.mg;
    const int Tb = mg.Tb, n = mg.n_keep;
    const int lane = threadIdx.x;
    const int mtiles = (Tb + 127) / 128;
    const int G = (Tb + 31) / 32;                          // bitmap words per row (<= 64)
    const int W8 = 8 * G;                                  // code words per row
    const int BS = G | 1;                                  // bitmap row stride (odd: conflict-free)
    const int row_end = min(mg.sink_first, Tb);
    const int sf = mg.sink_first;                          // <= Tb
    uint32_t* bm = reinterpret_cast<uint32_t*>(smem_raw);              // [32][BS]
    uint32_t* cand = bm + 32 * BS;                                       // [BCAP][32]: coarse << 24 | j
    const int64_t units = args.BH * mtiles * 4;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int64_t item = u >> 2;
        const int64_t bh = item / mtiles;
        const int m0 = (int)(item % mtiles) * 128;
        const int rl = (int)(u & 3) * 32 + lane;           // row within the item
        const int i = m0 + rl;
        // row kinds: 0 from the bitmap, 1 every block, 2 listed for the warp kernel, 3 no row
        int rk = (i >= Tb) ? 3 : ((i >= row_end || n >= Tb) ? 1 : 0);
        if (rk == 0) {
            uint32_t* brow = bm + lane * BS;
            // 1. bin b*
            const uint32_t* hs = args.hist + (size_t)item * 2 * 16 * 128 + rl;
            int bstar = 0, need_in = n;
            {
                int cum = 0;
                bool found = false;
                #pragma unroll
                for (int p = 15; p >= 0; --p) {
                    const uint32_t h2 = hs[p * 128] + hs[16 * 128 + p * 128];   // two 16-bit counts
                    const int hh = (int)(h2 >> 16), hl = (int)(h2 & 0xFFFFu);
                    if (!found && cum + hh >= n) { found = true; bstar = 2 * p + 1; need_in = n - cum; }
                    cum += hh;
                    if (!found && cum + hl >= n) { found = true; bstar = 2 * p; need_in = n - cum; }
                    cum += hl;
                }
            }
            // 2. one pass: codes above bin b* into the bitmap, the keys of bin b* aside
            const uint32_t y_def = (bstar < 31) ? (uint32_t)(8 * bstar + 8) * 0x01010101u : 0u;
            const uint32_t pat_bin = (uint32_t)bstar * 0x08080808u;
            const size_t wbase = (size_t)item * W8 * 128 + rl;
            const uint32_t* cw = args.codes + wbase;
            const uint32_t* fw = args.fine + wbase;
            const float width = args.width[item * 128 + rl];       // loaded early: used after the pass
            int nb = 0;
            // the coarse codes of groups g + 1 .. g + 4 in flight while group g is read
            // (the fine bytes are read later, for the few keys that are ranked)
            uint32_t ca[8], cb[8], cc[8], cd[8];
            #pragma unroll
            for (int k = 0; k < 8; ++k) {
                ca[k] = cw[(size_t)k * 128];
                cb[k] = (G > 1) ? cw[(size_t)(8 + k) * 128] : 0u;
                cc[k] = (G > 2) ? cw[(size_t)(16 + k) * 128] : 0u;
                cd[k] = (G > 3) ? cw[(size_t)(24 + k) * 128] : 0u;
            }
            #pragma unroll 1
            for (int g = 0; g < G; ++g) {
                uint32_t w[8];
                #pragma unroll
                for (int k = 0; k < 8; ++k) { w[k] = ca[k]; ca[k] = cb[k]; cb[k] = cc[k]; cc[k] = cd[k]; }
                if (g + 4 < G) {
                    #pragma unroll
                    for (int k = 0; k < 8; ++k) cd[k] = cw[(size_t)(8 * (g + 4) + k) * 128];
                }
                const int nv = Tb - 32 * g;
                const uint32_t vm = (nv >= 32) ? 0xffffffffu : ((1u << nv) - 1u);
                uint32_t bits = 0, inb = 0;
                #pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (bstar < 31) bits |= bytes_ge(w[k], y_def) << (4 * k);
                    inb |= bytes_eq(w[k] & 0xF8F8F8F8u, pat_bin) << (4 * k);
                }
                inb &= vm;
                while (inb) {
                    const int b = __ffs(inb) - 1;
                    inb &= inb - 1;
                    if (nb < BCAP) cand[nb * 32 + lane] = (byte_of8(w, b) << 24) | (uint32_t)(32 * g + b);
                    ++nb;
                }
                brow[g] = bits & vm;
            }
            if (nb > BCAP) {
                rk = 2;
            } else {
                // 3. the code c* and the keys of bin b* that are kept
                int cnt8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                for (int e = 0; e < nb; ++e) {
                    const int sub = (int)((cand[e * 32 + lane] >> 24) & 7u);
                    #pragma unroll
                    for (int x = 0; x < 8; ++x) cnt8[x] += (sub == x);
                }
                int sub = 0, need = need_in, m = 0;
                {
                    int cum = 0;
                    bool found = false;
                    #pragma unroll
                    for (int x = 7; x >= 0; --x) {
                        if (!found && cum + cnt8[x] >= need_in) { found = true; sub = x; need = need_in - cum; m = cnt8[x]; }
                        cum += cnt8[x];
                    }
                }
                const uint32_t cstar = (uint32_t)(bstar * 8 + sub);
                const bool partial = need < m;
                const bool tiny = cstar > 0 && cstar < 255 && width <= args.tiny_width;
                const bool ranked = partial && !tiny;
                uint32_t kept_mask = 0;                        // bit e: the e-th key of c* (j order) is kept
                if (ranked) {
                    if (cstar == 0 || cstar == 255 || m > RCAP) {
                        rk = 2;
                    } else {
                        // rank by (fine desc, j asc): key = fine << 16 | (0xFFFF - j); the
                        // fine bytes of the m keys of c* are read together (one round trip)
                        int jr[RCAP];
                        #pragma unroll
                        for (int y = 0; y < RCAP; ++y) jr[y] = 0;
                        int c = 0;
                        for (int e = 0; e < nb; ++e) {
                            const uint32_t x = cand[e * 32 + lane];
                            if ((x >> 24) == cstar) {
                                #pragma unroll
                                for (int y = 0; y < RCAP; ++y) jr[y] = (y == c) ? (int)(x & 0xFFFFu) : jr[y];
                                ++c;
                            }
                        }
                        uint32_t key[RCAP];
                        #pragma unroll
                        for (int y = 0; y < RCAP; ++y) key[y] = (y < m) ? fw[(size_t)(jr[y] >> 2) * 128] : 0u;
                        #pragma unroll
                        for (int y = 0; y < RCAP; ++y)
                            key[y] = (y < m) ? ((((key[y] >> (8 * (jr[y] & 3))) & 255u) << 16) | (0xFFFFu - (uint32_t)jr[y])) : 0u;
                        uint32_t f_last = 0, f_next = 256;
                        #pragma unroll
                        for (int y = 0; y < RCAP; ++y) {
                            int rank = 0;
                            #pragma unroll
                            for (int z = 0; z < RCAP; ++z) rank += (z < m) && (key[z] > key[y]);
                            if (y < m && rank < need) kept_mask |= 1u << y;
                            if (y < m && rank == need - 1) f_last = key[y] >> 16;
                            if (y < m && rank == need) f_next = key[y] >> 16;
                        }
                        if (f_last == f_next && width > args.tiny_width_fine) {
                            // the keys of c* with fine code f_last (up to TCAP of them)
                            // are ranked again by exact fp32 scores (q^ = hi + lo,
                            // k^ = hi + lo, over d in order), then j; `above` keys of
                            // c* have a larger fine code and are kept already
                            constexpr int TCAP = 4;
                            int jt[TCAP], yt[TCAP];
                            int nt = 0, above = 0;
                            #pragma unroll
                            for (int t = 0; t < TCAP; ++t) { jt[t] = 0; yt[t] = 0; }
                            #pragma unroll
                            for (int y = 0; y < RCAP; ++y) {
                                const uint32_t f = key[y] >> 16;
                                if (y < m && f > f_last) ++above;
                                if (y < m && f == f_last) {
                                    #pragma unroll
                                    for (int t = 0; t < TCAP; ++t) {
                                        jt[t] = (t == nt) ? (int)(0xFFFFu - (key[y] & 0xFFFFu)) : jt[t];
                                        yt[t] = (t == nt) ? y : yt[t];
                                    }
                                    ++nt;
                                }
                            }
                            if (nt > TCAP) {
                                rk = 2;
                            } else {
                                const int64_t qr = bh * Tb + i, kr0 = args.BH * Tb + bh * Tb;
                                const float4* qh = reinterpret_cast<const float4*>(args.means_hi + qr * D);
                                const float4* ql = reinterpret_cast<const float4*>(args.means_lo + qr * D);
                                float acc[TCAP];
                                #pragma unroll
                                for (int t = 0; t < TCAP; ++t) acc[t] = 0.f;
                                #pragma unroll 1
                                for (int c4 = 0; c4 < D / 4; c4 += 4) {
                                    float4 qa[4];
                                    #pragma unroll
                                    for (int u = 0; u < 4; ++u) {
                                        const float4 a4 = __ldcg(qh + c4 + u), b4 = __ldcg(ql + c4 + u);
                                        qa[u] = make_float4(a4.x + b4.x, a4.y + b4.y, a4.z + b4.z, a4.w + b4.w);
                                    }
                                    #pragma unroll
                                    for (int t = 0; t < TCAP; ++t) {
                                        if (t < nt) {
                                            const float4* kh = reinterpret_cast<const float4*>(args.means_hi + (kr0 + jt[t]) * D) + c4;
                                            const float4* kl = reinterpret_cast<const float4*>(args.means_lo + (kr0 + jt[t]) * D) + c4;
                                            float sacc = acc[t];
                                            #pragma unroll
                                            for (int u = 0; u < 4; ++u) {
                                                const float4 h4 = __ldcg(kh + u), l4 = __ldcg(kl + u);
                                                sacc = fmaf(qa[u].x, h4.x + l4.x, sacc);
                                                sacc = fmaf(qa[u].y, h4.y + l4.y, sacc);
                                                sacc = fmaf(qa[u].z, h4.z + l4.z, sacc);
                                                sacc = fmaf(qa[u].w, h4.w + l4.w, sacc);
                                            }
                                            acc[t] = sacc;
                                        }
                                    }
                                }
                                const int take = need - above;
                                #pragma unroll
                                for (int t = 0; t < TCAP; ++t) {
                                    int rank = 0;
                                    #pragma unroll
                                    for (int u = 0; u < TCAP; ++u)
                                        rank += (u < nt) && (acc[u] > acc[t] || (acc[u] == acc[t] && jt[u] < jt[t]));
                                    if (t < nt) {
                                        const uint32_t bit = 1u << yt[t];
                                        kept_mask = (rank < take) ? (kept_mask | bit) : (kept_mask & ~bit);
                                    }
                                }
                            }
                        }
                    }
                }
                if (rk == 0) {
                    // keys of bin b*: above c* kept; of c*, all, the ranked ones, or
                    // (a tie) the lowest-j `need`
                    int seen = 0;
                    for (int e = 0; e < nb; ++e) {
                        const uint32_t x = cand[e * 32 + lane];
                        const uint32_t code = x >> 24;
                        const int j = (int)(x & 0xFFFFu);
                        bool take = code > cstar;
                        if (code == cstar) {
                            take = !partial || (ranked ? ((kept_mask >> seen) & 1u) : (seen < need));
                            ++seen;
                        }
                        if (take) brow[j >> 5] |= 1u << (j & 31);
                    }
                }
            }
            if (rk == 2) {
                const int at = atomicAdd(args.overflow, 1);
                args.overflow[1 + at] = (int32_t)(bh * Tb + i);
            }
        }
        // 4. the CSR rows: thread r writes the kept keys below the sink columns
        // of row r from its own bitmap (rows stride BS, odd: the lanes' words
        // sit in distinct banks), in ascending order, the 32 rows in parallel;
        // then the whole warp writes, one row at a time and coalesced, the
        // sink columns of every row and all of a row that keeps every block.
        int nk = 0;
        if (rk == 0) {
            const uint32_t* brow = bm + lane * BS;
            const int64_t rs = row_offset(mg, bh, i);
            int32_t* out = args.col_idx + rs;
            const int wl = (sf + 31) >> 5;                 // bitmap words below the sink columns
            for (int wi = 0; wi < wl; ++wi) {
                uint32_t v = brow[wi];
                const int j0 = 32 * wi;
                if (j0 + 32 > sf) v &= (1u << (sf - j0)) - 1u;
                while (v) {
                    const int b = __ffs(v) - 1;
                    v &= v - 1;
                    csr_put(out, nk++, j0 + b, rs, mg.col_capacity);
                }
            }
        }
        uint32_t todo = __ballot_sync(0xffffffffu, rk < 2);
        while (todo) {
            const int r = __ffs(todo) - 1;
            todo &= todo - 1;
            const int rkr = __shfl_sync(0xffffffffu, rk, r);
            const int nkr = __shfl_sync(0xffffffffu, nk, r);
            const int ir = m0 + (rl - lane) + r;
            const int64_t row_id = bh * Tb + ir;
            const int64_t rs = row_offset(mg, bh, ir);
            int32_t* out = args.col_idx + rs;
            const int j_from = (rkr == 1) ? 0 : sf;        // every block, or the sink columns
            const int base = (rkr == 1) ? 0 : nkr;
            for (int j = j_from + lane; j < Tb; j += 32) csr_put(out, base + (j - j_from), j, rs, mg.col_capacity);
            if (lane == 0) {
                args.row_start[row_id] = (int32_t)rs;
                args.row_count[row_id] = base + (Tb - j_from);
            }
        }
    }
}

}  // namespace rf2
