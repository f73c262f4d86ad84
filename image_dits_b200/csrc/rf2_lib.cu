// C ABI of the RainFusion2.0 block-sparse attention library (include/rf2.h).
//
// Host code: argument validation, closed-form sizes, TMA tensor maps and
// kernel launches.  All kernels live in this one translation unit so they
// share the device status word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "rf2.h"
#include "attn.cuh"
#include "geometry.cuh"
#include "mask.cuh"
#include "permute.cuh"
#include "ptx.cuh"
#include "topn.cuh"

namespace rf2 {

// Top-n selection keeps rows of up to this many key blocks in registers
// (select_probe_kernel, 16 keys per lane); see launch_select_topn.
constexpr int32_t kSelectRegMaxBlocks = 32 * 16;

constexpr int32_t kMaxBlocks = 4096;     // T_b limit (N <= 262,144 tokens)

struct Checked {
    int status;
    PermGeo pg;
    int64_t BH;
    int32_t N, Tb, D;
};

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static Checked check_geometry(const rf2_geometry* g)
{
    Checked c;
    memset(&c, 0, sizeof c);
    c.status = RF2_ERR_INVALID_ARGUMENT;
    if (!g) return c;
    if (g->batch <= 0 || g->heads <= 0 || g->frames <= 0 || g->height <= 0 || g->width <= 0 ||
        g->win_t <= 0 || g->win_h <= 0 || g->win_w <= 0 || g->head_dim <= 0 || g->block <= 0 ||
        (g->first_frame_sink != 0 && g->first_frame_sink != 1) || g->text_tokens < 0)
        return c;
    const int64_t N = (int64_t)g->frames * g->height * g->width + g->text_tokens;
    if (N > INT32_MAX) return c;
    c.status = RF2_ERR_UNSUPPORTED;
    if (g->head_dim != 64 && g->head_dim != 128) return c;
    if (g->block != kBlock) return c;
    const int64_t Tb = (N + kBlock - 1) / kBlock;
    if (Tb > kMaxBlocks) return c;
    if ((int64_t)2 * g->batch * g->heads * Tb > INT32_MAX) return c;   // block-mean rows index a TMA map
    c.BH = (int64_t)g->batch * g->heads;
    if (c.BH > (int64_t)INT32_MAX / 2) return c;
    c.N = (int32_t)N;
    c.Tb = (int32_t)Tb;
    c.D = g->head_dim;
    c.pg = make_perm_geo(g->frames, g->height, g->width, g->win_t, g->win_h, g->win_w, g->first_frame_sink,
                         g->text_tokens);
    c.status = RF2_OK;
    return c;
}

static int keep_count(double keep, int32_t Tb, int32_t* n)
{
    if (!(keep > 0.0) || !(keep <= 1.0)) return RF2_ERR_INVALID_ARGUMENT;
    int64_t k = (int64_t)ceil(keep * (double)Tb - 1e-9);
    if (k < 1) k = 1;
    if (k > Tb) k = Tb;
    *n = (int32_t)k;
    return RF2_OK;
}

// Mask-prediction workspace: the block means as a tf32 hi/lo split, two
// fp32 arrays [2][BH][T_b][d], then the pooled-score buffer of one group of
// heads [G][T_b][ld] (ld = T_b rounded up to 4 floats); heads are scored and
// selected group by group so that the score buffer stays in L2 between the
// two kernels: the workspace holds as many heads' scores as fit in
// kScoreGroupBytes (at least one head).
constexpr size_t kScoreGroupBytes = (size_t)96 << 20;
static int32_t score_ld(int32_t Tb) { return (Tb + 3) & ~3; }
static size_t mask_means_bytes(const Checked& c) { return ((size_t)2 * c.BH * c.Tb * c.D * sizeof(float) + 255) & ~(size_t)255; }
static size_t score_head_bytes(const Checked& c) { return (size_t)c.Tb * score_ld(c.Tb) * sizeof(float); }
static int64_t score_group_heads(const Checked& c)
{
    int64_t g = (int64_t)(kScoreGroupBytes / score_head_bytes(c));
    if (g < 1) g = 1;
    return c.BH < g ? c.BH : g;
}
// Top-n selection from codes (topn_codes_kernel, topn_rows_kernel, topn_overflow_kernel): the
// codes, the per-row histograms and code widths.  They share the region after
// the means with the score buffer of the score-matrix path (never both in one
// call); the region is the larger of the two.
static int64_t topn_items(const Checked& c) { return c.BH * ((c.Tb + 127) / 128); }
static size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }
static size_t codes_bytes(const Checked& c) { return round256(4 * topn_codes_words(topn_items(c), c.Tb)); }
static size_t hist_bytes(const Checked& c) { return round256(4 * topn_hist_words(topn_items(c))); }
static size_t width_bytes(const Checked& c) { return round256((size_t)4 * topn_items(c) * 128); }
static size_t topn_overflow_bytes(const Checked& c) { return round256(4 * topn_overflow_words(c.BH * c.Tb)); }
static size_t topn_region_bytes(const Checked& c)
{
    return 2 * codes_bytes(c) + hist_bytes(c) + width_bytes(c) + topn_overflow_bytes(c);
}
static size_t after_means_bytes(const Checked& c, int64_t score_heads)
{
    const size_t sb = (size_t)score_heads * score_head_bytes(c), tb = topn_region_bytes(c);
    return sb > tb ? sb : tb;
}

static int sizes_for(const rf2_geometry* g, double keep, Checked& c, MaskGeo& mg, rf2_sizes* out)
{
    c = check_geometry(g);
    if (c.status != RF2_OK) return c.status;
    int32_t n = 0;
    const int st = keep_count(keep, c.Tb, &n);
    if (st != RF2_OK) return st;
    mg = make_mask_geo(c.N, n, sink_first_token(c.pg, g->first_frame_sink));
    const int64_t total = c.BH * mg.head_total;
    mg.col_capacity = total;
    if (total > INT32_MAX) return RF2_ERR_UNSUPPORTED;
    if (out) {
        out->num_tokens = c.N;
        out->num_blocks = c.Tb;
        out->n_keep = n;
        out->sink_first = (mg.sink_first < c.Tb) ? mg.sink_first : -1;
        out->row_capacity = mg.cap;
        out->num_rows = c.BH * c.Tb;
        out->col_idx_capacity = total;
        out->mask_workspace_bytes = 2 * mask_means_bytes(c) + after_means_bytes(c, score_group_heads(c));
    }
    return RF2_OK;
}

// Launch errors are reported per call: every launch helper drops a pending
// (non-sticky) error left by unrelated earlier work before it launches, and
// reads and clears its own launch's error after.  A sticky error (a context
// that has already faulted) persists and is reported by every later call.
static void clear_pending_error() { (void)cudaGetLastError(); }

static int launch_status()
{
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? RF2_OK : RF2_ERR_CUDA;
}

// ---------------------------------------------------------------- contexts
// Per-context caches (the dynamic shared-memory attribute of a kernel) are
// keyed by the unique id of the calling thread's current CUDA context, so a
// context created anew (after cudaDeviceReset, say) is set up again instead
// of trusting state that belonged to the old one.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

template <typename Fn>
static Fn driver_fn(const char* name)
{
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<Fn>(p);
    return nullptr;
}

// Unique id of the current context; false when there is none or it cannot be read.
static bool current_context_id(unsigned long long* id)
{
    static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    if (!get_current || !get_id) return false;
    CUcontext c = nullptr;
    if (get_current(&c) != CUDA_SUCCESS || !c) return false;
    return get_id(c, id) == CUDA_SUCCESS;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (kernel, context),
// raised when a later call needs more.
static int ensure_dynamic_smem(const void* func, size_t bytes)
{
    struct Entry { const void* func; unsigned long long ctx; size_t bytes; };
    static Entry cache[64];
    static int used = 0;
    static std::mutex mu;
    unsigned long long ctx = 0;
    const bool have_ctx = current_context_id(&ctx);
    std::lock_guard<std::mutex> lock(mu);
    Entry* e = nullptr;
    if (have_ctx)
        for (int i = 0; i < used; ++i)
            if (cache[i].func == func && cache[i].ctx == ctx) { e = &cache[i]; break; }
    if (e && e->bytes >= bytes) return RF2_OK;
    if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess) {
        clear_pending_error();
        return RF2_ERR_CUDA;
    }
    if (!have_ctx) return RF2_OK;
    if (!e) {
        e = &cache[used < 64 ? used++ : (int)(ctx % 64)];   // full: overwrite a slot (it is set again when needed)
        e->func = func;
        e->ctx = ctx;
        e->bytes = 0;
    }
    e->bytes = bytes;
    return RF2_OK;
}

static int grid_for_rows(int64_t rows)
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t warps = (rows + RF2_PERMUTE_ROWS - 1) / RF2_PERMUTE_ROWS;
    int64_t blocks = (warps + 7) / 8;
    const int64_t cap = (int64_t)sms * RF2_PERMUTE_MINB * 4;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return (int)blocks;
}

static int permute_impl(const rf2_geometry* geom, const void* in, void* out, void* stream, bool forward)
{
    Checked c = check_geometry(geom);
    if (c.status != RF2_OK) return c.status;
    if (!in || !out || !aligned16(in) || !aligned16(out) || in == out) return RF2_ERR_INVALID_ARGUMENT;
    const int64_t rows = c.BH * c.N;
    const int grid = grid_for_rows(rows);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const uint4* i4 = reinterpret_cast<const uint4*>(in);
    uint4* o4 = reinterpret_cast<uint4*>(out);
    clear_pending_error();
    if (c.D == 128) {
        if (forward) permute_rows_kernel<128, true><<<grid, 256, 0, s>>>(i4, o4, c.pg, rows);
        else         permute_rows_kernel<128, false><<<grid, 256, 0, s>>>(i4, o4, c.pg, rows);
    } else {
        if (forward) permute_rows_kernel<64, true><<<grid, 256, 0, s>>>(i4, o4, c.pg, rows);
        else         permute_rows_kernel<64, false><<<grid, 256, 0, s>>>(i4, o4, c.pg, rows);
    }
    return launch_status();
}

// ---------------------------------------------------------------- TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [BH, N, D] bf16 viewed as a 3D tensor (D, N, BH); box = 64 columns x rows,
// 128-byte swizzle (the canonical K-major / MN-major SW128 tcgen05 layouts).
static bool make_map(CUtensorMap* m, const void* ptr, int32_t D, int32_t N, int64_t BH, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)N * D * 2};
    const cuuint32_t box[3] = {64, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The same tensor viewed as 4D (64 columns, N rows, D/64 column chunks, BH):
// one box = `box_rows` rows x all of d, landing in shared memory chunk by
// chunk ([chunk][row][64 columns], 128-byte swizzle), i.e. one TMA load per
// tile instead of one per 64-column chunk.
static bool make_map_chunked(CUtensorMap* m, const void* ptr, int32_t D, int32_t N, int64_t BH, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {64, (cuuint64_t)N, (cuuint64_t)(D / 64), (cuuint64_t)BH};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, 128, (cuuint64_t)N * D * 2};
    const cuuint32_t box[4] = {64, box_rows, (cuuint32_t)(D / 64), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

static int* status_word_ptr()
{
    int* p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_status_word) != cudaSuccess) return nullptr;
    return p;
}

template <int D>
static int launch_attn(const Checked& c, const MaskGeo& mg, const void* qp, const void* kp, const void* vp,
                       const int32_t* row_start, const int32_t* row_count, const int32_t* col_idx, void* op,
                       float* lse, cudaStream_t s)
{
    using Cfg = AttnCfg<D>;
    CUtensorMap mq, mk, mv;
    if (!make_map_chunked(&mq, qp, D, c.N, c.BH, 128) || !make_map(&mk, kp, D, c.N, c.BH, 64) ||
        !make_map_chunked(&mv, vp, D, c.N, c.BH, 64))
        return RF2_ERR_CUDA;
    int* status = status_word_ptr();
    if (!status) return RF2_ERR_CUDA;
    AttnArgs a;
    a.row_start = row_start;
    a.row_count = row_count;
    a.col_idx = col_idx;
    a.op = reinterpret_cast<uint16_t*>(op);
    a.lse = lse;
    a.status = status;
    a.N = c.N;
    a.Tb = c.Tb;
    a.pairs = (c.Tb + 1) / 2;
    a.sink_pairs = (mg.sink_first < c.Tb) ? a.pairs - mg.sink_first / 2 : 0;
    a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    a.col_capacity = c.BH * (int64_t)c.Tb * c.Tb;      // the largest layout the library writes
    const size_t smem = Cfg::smem_bytes(c.Tb);
    if (ensure_dynamic_smem(reinterpret_cast<const void*>(block_sparse_attn_kernel<D>), smem) != RF2_OK)
        return RF2_ERR_CUDA;
    const int64_t grid = c.BH * a.pairs;
    clear_pending_error();
    block_sparse_attn_kernel<D><<<(unsigned)grid, Cfg::THREADS, smem, s>>>(mq, mk, mv, a);
    return launch_status();
}

// The [2*BH*T_b, d] fp32 block-mean array (hi or lo part) as a 2D tensor map:
// box = 32 floats (128 bytes) x `box_rows` rows, 128-byte swizzle (K-major
// tf32 tiles).
static bool make_means_map(CUtensorMap* m, const float* ptr, int32_t D, int64_t rows, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 4};
    const cuuint32_t box[2] = {32, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

static int num_sms()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <int D>
static int launch_scores(const Checked& c, const float* means_hi, const float* means_lo, float* S, int64_t h0,
                         int64_t g, cudaStream_t s)
{
    using Cfg = ScoreCfg<D>;
    int* status = status_word_ptr();
    if (!status) return RF2_ERR_CUDA;
    const int64_t rows = 2 * c.BH * c.Tb;
    CUtensorMap mh, ml, mhb, mlb;
    if (!make_means_map(&mh, means_hi, D, rows, 128) || !make_means_map(&ml, means_lo, D, rows, 128) ||
        !make_means_map(&mhb, means_hi, D, rows, Cfg::NCH) || !make_means_map(&mlb, means_lo, D, rows, Cfg::NCH))
        return RF2_ERR_CUDA;
    if (ensure_dynamic_smem(reinterpret_cast<const void*>(score_tc_kernel<D>), Cfg::SMEM) != RF2_OK)
        return RF2_ERR_CUDA;
    const int64_t items = g * ((c.Tb + 127) / 128);
    const int grid = (int)(items < num_sms() ? items : num_sms());
    clear_pending_error();
    score_tc_kernel<D><<<grid, Cfg::THREADS, Cfg::SMEM, s>>>(mh, ml, mhb, mlb, S, c.Tb, score_ld(c.Tb), c.BH, h0,
                                                             (int32_t)g, (float)(1.0 / sqrt((double)D)), status);
    return launch_status();
}

template <int R>
static int launch_select(const Checked& c, const MaskGeo& mg, const float* S, int64_t h0, int64_t g,
                         int32_t* row_start, int32_t* row_count, int32_t* col_idx, cudaStream_t s)
{
    const size_t smem = sizeof(uint32_t) * ((size_t)R * c.Tb + (256 + kSelCand) * (kSelThreads / 32));
    if (ensure_dynamic_smem(reinterpret_cast<const void*>(select_from_scores_kernel<R>), smem) != RF2_OK)
        return RF2_ERR_CUDA;
    dim3 grid((c.Tb + R - 1) / R, (unsigned)g);
    clear_pending_error();
    select_from_scores_kernel<R><<<grid, kSelThreads, smem, s>>>(S, score_ld(c.Tb), row_start, row_count,
                                                                 col_idx, mg, h0);
    return launch_status();
}

template <int KPL>
static int launch_select_probe(const Checked& c, const MaskGeo& mg, const float* S, int64_t h0, int64_t g,
                               int32_t* row_start, int32_t* row_count, int32_t* col_idx, cudaStream_t s)
{
    constexpr int rows_per_cta = kSelThreads / 32;
    dim3 grid((c.Tb + rows_per_cta - 1) / rows_per_cta, (unsigned)g);
    clear_pending_error();
    select_probe_kernel<KPL><<<grid, kSelThreads, 0, s>>>(S, score_ld(c.Tb), row_start, row_count, col_idx, mg, h0);
    return launch_status();
}

static int launch_select_topn(const Checked& c, const MaskGeo& mg, const float* S, int64_t h0, int64_t g,
                              int32_t* row_start, int32_t* row_count, int32_t* col_idx, cudaStream_t s)
{
    // Keys in registers pay off while a lane holds few of them (measured: the
    // image shape's mask 19% faster, 480p equal; at T_b = 1182, 40 keys per
    // lane, the register footprint halves occupancy and the shared-memory
    // radix select is faster).
    if (c.Tb <= kSelectRegMaxBlocks)
        return launch_select_probe<16>(c, mg, S, h0, g, row_start, row_count, col_idx, s);
    return launch_select<8>(c, mg, S, h0, g, row_start, row_count, col_idx, s);
}

// CDF-threshold selection for a group of heads: one warp per row, R rows per
// CTA, the rows' keys and weights in shared memory (R * T_b * 8 bytes).
template <int R>
static int launch_select_cdf(const Checked& c, const MaskGeo& mg, const float* S, int64_t h0, int64_t g,
                             int32_t* row_start, int32_t* row_count, int32_t* col_idx, float tau, cudaStream_t s)
{
    const size_t smem = (size_t)R * c.Tb * 8;
    if (ensure_dynamic_smem(reinterpret_cast<const void*>(select_cdf_kernel<R>), smem) != RF2_OK)
        return RF2_ERR_CUDA;
    dim3 grid((c.Tb + R - 1) / R, (unsigned)g);
    clear_pending_error();
    select_cdf_kernel<R><<<grid, 32 * R, smem, s>>>(S, score_ld(c.Tb), row_start, row_count, col_idx, mg, h0, tau);
    return launch_status();
}

// Block means, then per group of heads the tensor-core scores and the
// selection.  `ws` holds the means followed by a score buffer for as many
// heads as `ws_bytes` allows, at most kScoreGroupBytes of scores and at most
// as many heads as give the score kernel one item per SM.
// Workspace pointers of the mask path; G = heads scored per group.
struct MaskWs {
    float* means_hi;
    float* means_lo;
    float* S;
    int64_t G;
};

static int mask_ws(const Checked& c, void* ws, size_t ws_bytes, MaskWs* w, bool score_matrix = false)
{
    const size_t mb = mask_means_bytes(c);
    const size_t need = score_matrix ? score_head_bytes(c) : after_means_bytes(c, 1);
    if (ws_bytes < 2 * mb + need) return RF2_ERR_INSUFFICIENT_WORKSPACE;
    int64_t G = (int64_t)((ws_bytes - 2 * mb) / score_head_bytes(c));
    if (G > score_group_heads(c)) G = score_group_heads(c);
    // one round of the persistent score kernel: a group's (head, 128-row tile)
    // items at most one per SM (160 items on 148 SMs would take two rounds)
    const int64_t tiles = (c.Tb + 127) / 128;
    int64_t round_heads = num_sms() / tiles;
    if (round_heads < 1) round_heads = 1;
    if (G > round_heads) G = round_heads;
    w->means_hi = reinterpret_cast<float*>(ws);
    w->means_lo = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + mb);
    w->S = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + 2 * mb);
    w->G = G;
    return RF2_OK;
}

// Top-n selection without the score matrix: topn_codes_kernel (scores on
// the tensor cores, reduced to 16-bit codes and per-row histograms as they
// leave TMEM), topn_rows_kernel (one thread per row) and topn_overflow_kernel
// (one CTA for each row the former lists).
template <int D>
static int launch_topn(const Checked& c, const MaskGeo& mg, const MaskWs& w, int32_t* row_start,
                       int32_t* row_count, int32_t* col_idx, cudaStream_t s)
{
    using Cfg = TopnCfg<D>;
    int* status = status_word_ptr();
    if (!status) return RF2_ERR_CUDA;
    const int64_t rows = 2 * c.BH * c.Tb;
    CUtensorMap ah, al, bh, bl, rh, rlo;
    if (!make_means_map(&ah, w.means_hi, D, rows, 128) || !make_means_map(&al, w.means_lo, D, rows, 128) ||
        !make_means_map(&bh, w.means_hi, D, rows, Cfg::NB) || !make_means_map(&bl, w.means_lo, D, rows, Cfg::NB) ||
        !make_means_map(&rh, w.means_hi, D, rows, 1) || !make_means_map(&rlo, w.means_lo, D, rows, 1))
        return RF2_ERR_CUDA;
    if (ensure_dynamic_smem(reinterpret_cast<const void*>(topn_codes_kernel<D>), Cfg::SMEM) != RF2_OK)
        return RF2_ERR_CUDA;
    // topn_rows_kernel: bitmaps [32][G | 1], bin-b* keys [64][32];
    // topn_overflow_kernel: the keys of the threshold code, their scores, radix bins
    const int G = (c.Tb + 31) / 32;
    const size_t rows_smem = ((size_t)32 * (G | 1) + 64 * 32) * 4;
    const size_t ovf_smem = (size_t)(2 * c.Tb + 256) * 4;
    if (ensure_dynamic_smem(reinterpret_cast<const void*>(topn_rows_kernel<D>), rows_smem) != RF2_OK ||
        ensure_dynamic_smem(reinterpret_cast<const void*>(topn_overflow_kernel<D>), ovf_smem) != RF2_OK)
        return RF2_ERR_CUDA;
    uint8_t* region = reinterpret_cast<uint8_t*>(w.S);
    TopnArgs a;
    a.means_hi = w.means_hi;
    a.means_lo = w.means_lo;
    a.codes = reinterpret_cast<uint32_t*>(region);
    a.fine = reinterpret_cast<uint32_t*>(region + codes_bytes(c));
    a.hist = reinterpret_cast<uint32_t*>(region + 2 * codes_bytes(c));
    a.width = reinterpret_cast<float*>(region + 2 * codes_bytes(c) + hist_bytes(c));
    a.overflow = reinterpret_cast<int32_t*>(region + 2 * codes_bytes(c) + hist_bytes(c) + width_bytes(c));
    a.row_start = row_start;
    a.row_count = row_count;
    a.col_idx = col_idx;
    a.status = status;
    a.mg = mg;
    a.BH = c.BH;
    // Scores are compared unscaled (q^ . k^): 1e-6 after the 1/sqrt(d) scale
    // is the code width up to which a code's keys count as tied.
    a.tiny_width = (float)(1e-6 * sqrt((double)D));
    a.tiny_width_fine = 256.f * a.tiny_width;
    a.min_width = 120.f * a.tiny_width;
    const int64_t items = topn_items(c);
    const int sms = num_sms();
    const int grid = (int)(items < sms ? items : sms);
    clear_pending_error();
    if (cudaMemsetAsync(a.overflow, 0, sizeof(int32_t), s) != cudaSuccess) return RF2_ERR_CUDA;
    topn_codes_kernel<D><<<grid, Cfg::THREADS, Cfg::SMEM, s>>>(ah, al, bh, bl, rh, rlo, a);
    int r = launch_status();
    if (r != RF2_OK) return r;
    const int64_t rows_grid = 4 * items < (int64_t)sms * 12 ? 4 * items : (int64_t)sms * 12;
    topn_rows_kernel<D><<<(unsigned)rows_grid, 32, rows_smem, s>>>(a);
    r = launch_status();
    if (r != RF2_OK) return r;
    // rows with too many keys near their threshold for topn_rows_kernel (rare; the
    // launch returns at once when there are none)
    topn_overflow_kernel<D><<<sms, 512, ovf_smem, s>>>(a);
    return launch_status();
}

// Per group of heads: the tensor-core scores, then the selection (top-n, or
// the CDF threshold when tau > 0).
static int launch_score_select(const Checked& c, const MaskGeo& mg, const MaskWs& w, int32_t* row_start,
                               int32_t* row_count, int32_t* col_idx, cudaStream_t s, float tau = 0.f,
                               bool score_matrix = false)
{
    // The score-matrix path is the faster one while all heads' scores fit one
    // group (they then stay in L2); beyond that, selection from codes.  The
    // environment variable RF2_MASK_SELECT = "codes" or "scores" overrides
    // the choice (both give the same masks outside the tie band).
    bool from_codes = (uint64_t)c.BH * score_head_bytes(c) > kScoreGroupBytes;
    if (const char* e = getenv("RF2_MASK_SELECT")) {
        if (strcmp(e, "codes") == 0) from_codes = true;
        else if (strcmp(e, "scores") == 0) from_codes = false;
    }
    if (tau <= 0.f && !score_matrix && from_codes && c.Tb <= TopnCfg<128>::MAX_TB)
        return (c.D == 128) ? launch_topn<128>(c, mg, w, row_start, row_count, col_idx, s)
                            : launch_topn<64>(c, mg, w, row_start, row_count, col_idx, s);
    int r = RF2_OK;
    for (int64_t h0 = 0; r == RF2_OK && h0 < c.BH; h0 += w.G) {
        const int64_t g = (c.BH - h0 < w.G) ? c.BH - h0 : w.G;
        r = (c.D == 128) ? launch_scores<128>(c, w.means_hi, w.means_lo, w.S, h0, g, s)
                         : launch_scores<64>(c, w.means_hi, w.means_lo, w.S, h0, g, s);
        if (r != RF2_OK) break;
        if (tau > 0.f)
            r = (c.Tb <= 1600) ? launch_select_cdf<8>(c, mg, w.S, h0, g, row_start, row_count, col_idx, tau, s)
                               : launch_select_cdf<4>(c, mg, w.S, h0, g, row_start, row_count, col_idx, tau, s);
        else
            r = launch_select_topn(c, mg, w.S, h0, g, row_start, row_count, col_idx, s);
    }
    return r;
}

// Block means of the permuted Q and K, then scores and selection.
static int launch_mask(const Checked& c, const MaskGeo& mg, const void* qp, const void* kp, int32_t* row_start,
                       int32_t* row_count, int32_t* col_idx, void* ws, size_t ws_bytes, cudaStream_t s,
                       float tau = 0.f, bool score_matrix = false)
{
    MaskWs w;
    const int st = mask_ws(c, ws, ws_bytes, &w, score_matrix);
    if (st != RF2_OK) return st;
    const int64_t warps = 2 * c.BH * c.Tb;
    const unsigned grid = (unsigned)((warps + 7) / 8);
    clear_pending_error();
    if (c.D == 128)
        block_mean_kernel<128><<<grid, 256, 0, s>>>(reinterpret_cast<const uint4*>(qp),
                                                     reinterpret_cast<const uint4*>(kp), w.means_hi, w.means_lo,
                                                     c.N, c.Tb, c.BH);
    else
        block_mean_kernel<64><<<grid, 256, 0, s>>>(reinterpret_cast<const uint4*>(qp),
                                                    reinterpret_cast<const uint4*>(kp), w.means_hi, w.means_lo,
                                                    c.N, c.Tb, c.BH);
    const int r = launch_status();
    if (r != RF2_OK) return r;
    return launch_score_select(c, mg, w, row_start, row_count, col_idx, s, tau, score_matrix);
}

// ------------------------------------------------------------------------
// Fixed device scratch for rf2_predict_mask_static (callers that cannot
// allocate).  Every device that loads this library holds these 64 MiB until
// the process exits.  In host code `g_static_scratch` only names a host-side
// stand-in, so every call looks up its device address on the current device
// (no cached pointer can outlive the context it was read in).
constexpr size_t kStaticScratchBytes = (size_t)64 << 20;
static __device__ __align__(256) float g_static_scratch[kStaticScratchBytes / sizeof(float)];

// Device address of the scratch on the calling thread's current device.
static int static_scratch(float** out)
{
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
        clear_pending_error();
        return RF2_ERR_CUDA;
    }
    *out = static_cast<float*>(p);
    return RF2_OK;
}

}  // namespace rf2

using namespace rf2;

extern "C" {

const char* rf2_status_string(int status)
{
    switch (status) {
    case RF2_OK: return "ok";
    case RF2_ERR_INVALID_ARGUMENT: return "invalid argument";
    case RF2_ERR_UNSUPPORTED: return "unsupported geometry";
    case RF2_ERR_INSUFFICIENT_WORKSPACE: return "workspace too small";
    case RF2_ERR_CUDA: return "CUDA error";
    case RF2_ERR_TIMEOUT: return "device wait timed out";
    case RF2_ERR_RANGE: return "index out of range (checked build)";
    default: return "unknown status";
    }
}

int rf2_query(const rf2_geometry* geom, double keep_ratio, rf2_sizes* out)
{
    if (!out) return RF2_ERR_INVALID_ARGUMENT;
    Checked c;
    MaskGeo mg;
    return sizes_for(geom, keep_ratio, c, mg, out);
}

int rf2_permutation_index(const rf2_geometry* geom, int32_t* perm)
{
    Checked c = check_geometry(geom);
    if (c.status != RF2_OK) return c.status;
    if (!perm) return RF2_ERR_INVALID_ARGUMENT;
    for (int32_t p = 0; p < c.N; ++p) perm[p] = perm_src(c.pg, p);
    return RF2_OK;
}

int rf2_permute(const rf2_geometry* geom, const void* x, void* xp, void* stream)
{
    return permute_impl(geom, x, xp, stream, true);
}

int rf2_unpermute(const rf2_geometry* geom, const void* xp, void* x, void* stream)
{
    return permute_impl(geom, xp, x, stream, false);
}

int rf2_predict_mask(const rf2_geometry* geom, const void* qp, const void* kp, double keep_ratio,
                     int32_t* row_start, int32_t* row_count, int32_t* col_idx, void* workspace,
                     size_t workspace_bytes, void* stream)
{
    Checked c;
    MaskGeo mg;
    rf2_sizes sz;
    const int st = sizes_for(geom, keep_ratio, c, mg, &sz);
    if (st != RF2_OK) return st;
    if (!qp || !kp || !row_start || !row_count || !col_idx || !workspace) return RF2_ERR_INVALID_ARGUMENT;
    if (!aligned16(qp) || !aligned16(kp) || !aligned16(workspace) || !aligned16(row_start) ||
        !aligned16(row_count) || !aligned16(col_idx))
        return RF2_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < sz.mask_workspace_bytes) return RF2_ERR_INSUFFICIENT_WORKSPACE;
    return launch_mask(c, mg, qp, kp, row_start, row_count, col_idx, workspace, workspace_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

int rf2_block_sparse_attn(const rf2_geometry* geom, const void* qp, const void* kp, const void* vp,
                          const int32_t* row_start, const int32_t* row_count, const int32_t* col_idx,
                          void* op, float* lse, void* stream)
{
    const Checked c = check_geometry(geom);
    if (c.status != RF2_OK) return c.status;
    const MaskGeo mg = make_mask_geo(c.N, 1, sink_first_token(c.pg, geom->first_frame_sink));
    if (!qp || !kp || !vp || !row_start || !row_count || !col_idx || !op) return RF2_ERR_INVALID_ARGUMENT;
    if (!aligned16(qp) || !aligned16(kp) || !aligned16(vp) || !aligned16(op) || !aligned16(row_start) ||
        !aligned16(row_count) || !aligned16(col_idx) || (lse && !aligned16(lse)))
        return RF2_ERR_INVALID_ARGUMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return (c.D == 128) ? launch_attn<128>(c, mg, qp, kp, vp, row_start, row_count, col_idx, op, lse, s)
                        : launch_attn<64>(c, mg, qp, kp, vp, row_start, row_count, col_idx, op, lse, s);
}

int rf2_predict_mask_static(const rf2_geometry* geom, const void* qp, const void* kp, double keep_ratio,
                            int32_t* row_start, int32_t* row_count, int32_t* col_idx, void* stream)
{
    Checked c;
    MaskGeo mg;
    rf2_sizes sz;
    const int st = sizes_for(geom, keep_ratio, c, mg, &sz);
    if (st != RF2_OK) return st;
    if (!qp || !kp || !row_start || !row_count || !col_idx) return RF2_ERR_INVALID_ARGUMENT;
    if (!aligned16(qp) || !aligned16(kp) || !aligned16(row_start) || !aligned16(row_count) || !aligned16(col_idx))
        return RF2_ERR_INVALID_ARGUMENT;
    // Needs room for the block means and the scores of at least one head (the
    // fixed array serves the score-matrix path: scores and selection head
    // group by head group, as many heads per group as fit).
    if (2 * mask_means_bytes(c) + score_head_bytes(c) > kStaticScratchBytes) return RF2_ERR_INSUFFICIENT_WORKSPACE;
    float* scratch = nullptr;
    const int ss = static_scratch(&scratch);
    if (ss != RF2_OK) return ss;
    // Every scratch element the kernels read is written earlier in the same
    // call, so nothing left from an earlier call needs clearing.
    return launch_mask(c, mg, qp, kp, row_start, row_count, col_idx, scratch, kStaticScratchBytes,
                       reinterpret_cast<cudaStream_t>(stream), 0.f, true);
}

int rf2_permute_qk_pool(const rf2_geometry* geom, const void* q, const void* k, void* qp, void* kp,
                        void* workspace, size_t workspace_bytes, void* stream)
{
    Checked c;
    MaskGeo mg;
    rf2_sizes sz;
    const int st = sizes_for(geom, 1.0, c, mg, &sz);
    if (st != RF2_OK) return st;
    if (!q || !k || !qp || !kp || !workspace) return RF2_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(qp) || !aligned16(kp) || !aligned16(workspace))
        return RF2_ERR_INVALID_ARGUMENT;
    if (q == qp || k == kp || q == kp || k == qp) return RF2_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < sz.mask_workspace_bytes) return RF2_ERR_INSUFFICIENT_WORKSPACE;
    MaskWs w;
    const int ws_st = mask_ws(c, workspace, workspace_bytes, &w);
    if (ws_st != RF2_OK) return ws_st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t blocks = 2 * c.BH * c.Tb;
    int64_t grid = (blocks + 7) / 8;
    const int64_t cap = (int64_t)num_sms() * 16;
    if (grid > cap) grid = cap;
    clear_pending_error();
    if (c.D == 128)
        permute_pool_kernel<128><<<(unsigned)grid, 256, 0, s>>>(
            reinterpret_cast<const uint4*>(q), reinterpret_cast<const uint4*>(k), reinterpret_cast<uint4*>(qp),
            reinterpret_cast<uint4*>(kp), c.pg, c.Tb, c.BH, w.means_hi, w.means_lo);
    else
        permute_pool_kernel<64><<<(unsigned)grid, 256, 0, s>>>(
            reinterpret_cast<const uint4*>(q), reinterpret_cast<const uint4*>(k), reinterpret_cast<uint4*>(qp),
            reinterpret_cast<uint4*>(kp), c.pg, c.Tb, c.BH, w.means_hi, w.means_lo);
    return launch_status();
}

int rf2_predict_mask_pooled(const rf2_geometry* geom, double keep_ratio, int32_t* row_start, int32_t* row_count,
                            int32_t* col_idx, void* workspace, size_t workspace_bytes, void* stream)
{
    Checked c;
    MaskGeo mg;
    rf2_sizes sz;
    const int st = sizes_for(geom, keep_ratio, c, mg, &sz);
    if (st != RF2_OK) return st;
    if (!row_start || !row_count || !col_idx || !workspace) return RF2_ERR_INVALID_ARGUMENT;
    if (!aligned16(workspace) || !aligned16(row_start) || !aligned16(row_count) || !aligned16(col_idx))
        return RF2_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < sz.mask_workspace_bytes) return RF2_ERR_INSUFFICIENT_WORKSPACE;
    MaskWs w;
    const int ws_st = mask_ws(c, workspace, workspace_bytes, &w);
    if (ws_st != RF2_OK) return ws_st;
    return launch_score_select(c, mg, w, row_start, row_count, col_idx, reinterpret_cast<cudaStream_t>(stream));
}

static bool tau_ok(double tau) { return tau > 0.0 && tau <= 1.0; }

int rf2_predict_mask_cdf(const rf2_geometry* geom, const void* qp, const void* kp, double tau, int32_t* row_start,
                         int32_t* row_count, int32_t* col_idx, void* workspace, size_t workspace_bytes, void* stream)
{
    Checked c;
    MaskGeo mg;
    rf2_sizes sz;
    const int st = sizes_for(geom, 1.0, c, mg, &sz);      // rows at full capacity T_b
    if (st != RF2_OK) return st;
    if (!tau_ok(tau)) return RF2_ERR_INVALID_ARGUMENT;
    if (!qp || !kp || !row_start || !row_count || !col_idx || !workspace) return RF2_ERR_INVALID_ARGUMENT;
    if (!aligned16(qp) || !aligned16(kp) || !aligned16(workspace) || !aligned16(row_start) || !aligned16(row_count) ||
        !aligned16(col_idx))
        return RF2_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < sz.mask_workspace_bytes) return RF2_ERR_INSUFFICIENT_WORKSPACE;
    return launch_mask(c, mg, qp, kp, row_start, row_count, col_idx, workspace, workspace_bytes,
                       reinterpret_cast<cudaStream_t>(stream), (float)tau);
}

int rf2_predict_mask_cdf_pooled(const rf2_geometry* geom, double tau, int32_t* row_start, int32_t* row_count,
                                int32_t* col_idx, void* workspace, size_t workspace_bytes, void* stream)
{
    Checked c;
    MaskGeo mg;
    rf2_sizes sz;
    const int st = sizes_for(geom, 1.0, c, mg, &sz);
    if (st != RF2_OK) return st;
    if (!tau_ok(tau)) return RF2_ERR_INVALID_ARGUMENT;
    if (!row_start || !row_count || !col_idx || !workspace) return RF2_ERR_INVALID_ARGUMENT;
    if (!aligned16(workspace) || !aligned16(row_start) || !aligned16(row_count) || !aligned16(col_idx))
        return RF2_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < sz.mask_workspace_bytes) return RF2_ERR_INSUFFICIENT_WORKSPACE;
    MaskWs w;
    const int ws_st = mask_ws(c, workspace, workspace_bytes, &w);
    if (ws_st != RF2_OK) return ws_st;
    return launch_score_select(c, mg, w, row_start, row_count, col_idx, reinterpret_cast<cudaStream_t>(stream),
                               (float)tau);
}

// Self-test of the timeout path: one CTA of two warps, each waiting (lane 0)
// on its own mbarrier that nothing ever completes.  Warp 0 gives up after
// `limit_ns`, records the timeout in the status word and raises the CTA's
// abort flag; warp 1 (no time limit of its own beyond the usual one) must
// leave through that flag.  Nothing faults; both waits end.
static __global__ void selftest_timeout_kernel(uint64_t limit_ns, int* status, int* left)
{
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (lane == 0) {
        const bool ok = mbar_wait(smem_u32(&bars[warp]), 0, &abort_flag, status,
                                  warp == 0 ? limit_ns : kWaitLimitNs);
        if (!ok) atomicAdd(left, 1);
    }
}

__device__ int g_selftest_given_up;

static int* selftest_counter()
{
    int* p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_selftest_given_up) != cudaSuccess) return nullptr;
    return p;
}

int rf2_selftest_wait_timeout(uint32_t limit_us, int32_t* waits_given_up, void* stream)
{
    if (!waits_given_up || limit_us == 0 || limit_us > 1000000) return RF2_ERR_INVALID_ARGUMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int* status = status_word_ptr();
    int* left = selftest_counter();
    if (!status || !left) return RF2_ERR_CUDA;
    clear_pending_error();
    if (cudaMemsetAsync(left, 0, sizeof(int), s) != cudaSuccess) return RF2_ERR_CUDA;
    selftest_timeout_kernel<<<1, 64, 0, s>>>((uint64_t)limit_us * 1000u, status, left);
    const int r = launch_status();
    if (r != RF2_OK) return r;
    if (cudaMemcpyAsync(waits_given_up, left, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return RF2_ERR_CUDA;
    return cudaStreamSynchronize(s) == cudaSuccess ? RF2_OK : RF2_ERR_CUDA;
}

// ---------------------------------------------------------------- host-memory call
// Heads per chunk: `chunks` near-equal chunks (cuts at round-half-even of
// c * heads / chunks), the last split into halves (rounded up) down to one head.
static int host_chunk_sizes(int32_t heads, int32_t chunks, int32_t* sizes, int cap)
{
    const int n = (int)(chunks < 1 ? 1 : (chunks > heads ? heads : chunks));
    int m = 0;
    int prev = 0;
    for (int c = 1; c <= n; ++c) {
        const int cut = (int)nearbyint((double)c * heads / n);
        if (m >= cap) return -1;
        sizes[m++] = cut - prev;
        prev = cut;
    }
    int r = sizes[--m];
    while (r > 1) {
        const int h = (r + 1) / 2;
        if (m >= cap) return -1;
        sizes[m++] = h;
        r -= h;
    }
    if (r) {
        if (m >= cap) return -1;
        sizes[m++] = r;
    }
    return m;
}

struct HostPlan {
    Checked c;
    int32_t sizes[256];
    int n;
    int32_t hmax;
    rf2_geometry gmax;       // geometry of the largest chunk
    rf2_sizes sz;            // its mask sizes
    size_t tensor_bytes, chunk_bytes, work_bytes;
    size_t off_q, off_k, off_v, off_o, off_qp, off_kp, off_vp, off_op, off_rs, off_rc, off_ci, off_ws;
};

static rf2_geometry chunk_geometry(const rf2_geometry* g, int32_t heads)
{
    rf2_geometry h = *g;
    h.batch = 1;
    h.heads = heads;
    return h;
}

static int host_plan(const rf2_geometry* geom, double keep, double tau, int32_t chunks, HostPlan& p)
{
    p.c = check_geometry(geom);
    if (p.c.status != RF2_OK) return p.c.status;
    if ((keep > 0.0) == (tau > 0.0)) return RF2_ERR_INVALID_ARGUMENT;          // exactly one selection
    if (tau > 0.0 && !(tau <= 1.0)) return RF2_ERR_INVALID_ARGUMENT;
    if (p.c.BH > INT32_MAX) return RF2_ERR_UNSUPPORTED;
    p.n = host_chunk_sizes((int32_t)p.c.BH, chunks, p.sizes, 256);
    if (p.n <= 0) return RF2_ERR_INVALID_ARGUMENT;
    p.hmax = 0;
    for (int i = 0; i < p.n; ++i) p.hmax = p.sizes[i] > p.hmax ? p.sizes[i] : p.hmax;
    p.gmax = chunk_geometry(geom, p.hmax);
    Checked cm;
    MaskGeo mg;
    const int st = sizes_for(&p.gmax, tau > 0.0 ? 1.0 : keep, cm, mg, &p.sz);
    if (st != RF2_OK) return st;
    const size_t row_bytes = (size_t)p.c.N * p.c.D * 2;
    p.tensor_bytes = (size_t)p.c.BH * row_bytes;
    p.chunk_bytes = (size_t)p.hmax * row_bytes;
    size_t at = 0;
    auto take = [&](size_t bytes) { const size_t o = at; at += round256(bytes); return o; };
    p.off_q = take(p.tensor_bytes);
    p.off_k = take(p.tensor_bytes);
    p.off_v = take(p.tensor_bytes);
    p.off_o = take(p.tensor_bytes);
    p.off_qp = take(p.chunk_bytes);
    p.off_kp = take(p.chunk_bytes);
    p.off_vp = take(p.chunk_bytes);
    p.off_op = take(p.chunk_bytes);
    p.off_rs = take((size_t)p.sz.num_rows * 4);
    p.off_rc = take((size_t)p.sz.num_rows * 4);
    p.off_ci = take((size_t)p.sz.col_idx_capacity * 4);
    p.off_ws = take(p.sz.mask_workspace_bytes);
    p.work_bytes = at;
    return RF2_OK;
}

int rf2_attention_host_query(const rf2_geometry* geom, double keep_ratio, double tau, int32_t chunks,
                             rf2_host_sizes* out)
{
    if (!out) return RF2_ERR_INVALID_ARGUMENT;
    HostPlan p;
    const int st = host_plan(geom, keep_ratio, tau, chunks, p);
    if (st != RF2_OK) return st;
    out->num_chunks = p.n;
    out->max_chunk_heads = p.hmax;
    out->work_bytes = p.work_bytes;
    return RF2_OK;
}

int rf2_attention_host(const rf2_geometry* geom, double keep_ratio, double tau, int32_t chunks,
                       const void* q_host, const void* k_host, const void* v_host, void* o_host, void* work,
                       size_t work_bytes, void* stream_h2d, void* stream_compute, void* stream_d2h,
                       void** events, int32_t num_events)
{
    HostPlan p;
    int st = host_plan(geom, keep_ratio, tau, chunks, p);
    if (st != RF2_OK) return st;
    if (!q_host || !k_host || !v_host || !o_host || !work) return RF2_ERR_INVALID_ARGUMENT;
    if (!aligned16(q_host) || !aligned16(k_host) || !aligned16(v_host) || !aligned16(o_host) ||
        (reinterpret_cast<uintptr_t>(work) & 255u))
        return RF2_ERR_INVALID_ARGUMENT;
    if (work_bytes < p.work_bytes) return RF2_ERR_INSUFFICIENT_WORKSPACE;
    cudaStream_t sh = reinterpret_cast<cudaStream_t>(stream_h2d);
    cudaStream_t sc = reinterpret_cast<cudaStream_t>(stream_compute);
    cudaStream_t sd = reinterpret_cast<cudaStream_t>(stream_d2h);
    if (sh == sc || sh == sd || sc == sd) return RF2_ERR_INVALID_ARGUMENT;
    const bool per_chunk = events != nullptr && num_events > 0;
    if (per_chunk && num_events < 2 * p.n) return RF2_ERR_INVALID_ARGUMENT;
    cudaEvent_t* chunk_ev = reinterpret_cast<cudaEvent_t*>(events);   // [2c]: computed, [2c+1]: copied back
    uint8_t* w = reinterpret_cast<uint8_t*>(work);
    const size_t row_bytes = (size_t)p.c.N * p.c.D * 2;
    // events: 0 compute idle, 1 copy-back idle, then per chunk: inputs in, chunk computed
    const int nev = 2 + 2 * p.n;
    cudaEvent_t ev[2 + 2 * 256];
    int made = 0;
    auto cleanup = [&](int r) {
        for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
        return r;
    };
    clear_pending_error();
    for (; made < nev; ++made)
        if (cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming) != cudaSuccess) return cleanup(RF2_ERR_CUDA);
    // the previous calls on these streams: computation done before `work` is overwritten by
    // copies, copy-back done before it is overwritten by computation (whole calls, or chunk
    // by chunk through the caller's events; an event never recorded is no wait)
    if (!per_chunk &&
        (cudaEventRecord(ev[0], sc) != cudaSuccess || cudaStreamWaitEvent(sh, ev[0], 0) != cudaSuccess ||
         cudaEventRecord(ev[1], sd) != cudaSuccess || cudaStreamWaitEvent(sc, ev[1], 0) != cudaSuccess))
        return cleanup(RF2_ERR_CUDA);
    // inputs, chunk by chunk
    int64_t h0 = 0;
    for (int c = 0; c < p.n; ++c) {
        const size_t off = (size_t)h0 * row_bytes, bytes = (size_t)p.sizes[c] * row_bytes;
        if (per_chunk && cudaStreamWaitEvent(sh, chunk_ev[2 * c], 0) != cudaSuccess) return cleanup(RF2_ERR_CUDA);
        if (cudaMemcpyAsync(w + p.off_q + off, static_cast<const uint8_t*>(q_host) + off, bytes,
                            cudaMemcpyHostToDevice, sh) != cudaSuccess ||
            cudaMemcpyAsync(w + p.off_k + off, static_cast<const uint8_t*>(k_host) + off, bytes,
                            cudaMemcpyHostToDevice, sh) != cudaSuccess ||
            cudaMemcpyAsync(w + p.off_v + off, static_cast<const uint8_t*>(v_host) + off, bytes,
                            cudaMemcpyHostToDevice, sh) != cudaSuccess ||
            cudaEventRecord(ev[2 + 2 * c], sh) != cudaSuccess)
            return cleanup(RF2_ERR_CUDA);
        h0 += p.sizes[c];
    }
    // computation on one stream (the chunk buffers are reused), each chunk's copy-back after it
    int32_t* rs = reinterpret_cast<int32_t*>(w + p.off_rs);
    int32_t* rc = reinterpret_cast<int32_t*>(w + p.off_rc);
    int32_t* ci = reinterpret_cast<int32_t*>(w + p.off_ci);
    void* ws = w + p.off_ws;
    h0 = 0;
    for (int c = 0; c < p.n; ++c) {
        const rf2_geometry g = chunk_geometry(geom, p.sizes[c]);
        const size_t off = (size_t)h0 * row_bytes, bytes = (size_t)p.sizes[c] * row_bytes;
        if (cudaStreamWaitEvent(sc, ev[2 + 2 * c], 0) != cudaSuccess ||
            (per_chunk && cudaStreamWaitEvent(sc, chunk_ev[2 * c + 1], 0) != cudaSuccess))
            return cleanup(RF2_ERR_CUDA);
        st = rf2_permute_qk_pool(&g, w + p.off_q + off, w + p.off_k + off, w + p.off_qp, w + p.off_kp, ws,
                                 p.sz.mask_workspace_bytes, sc);
        if (st == RF2_OK) st = rf2_permute(&g, w + p.off_v + off, w + p.off_vp, sc);
        if (st == RF2_OK)
            st = (tau > 0.0) ? rf2_predict_mask_cdf_pooled(&g, tau, rs, rc, ci, ws, p.sz.mask_workspace_bytes, sc)
                             : rf2_predict_mask_pooled(&g, keep_ratio, rs, rc, ci, ws, p.sz.mask_workspace_bytes, sc);
        if (st == RF2_OK)
            st = rf2_block_sparse_attn(&g, w + p.off_qp, w + p.off_kp, w + p.off_vp, rs, rc, ci, w + p.off_op,
                                       nullptr, sc);
        if (st == RF2_OK) st = rf2_unpermute(&g, w + p.off_op, w + p.off_o + off, sc);
        if (st != RF2_OK) return cleanup(st);
        if (cudaEventRecord(ev[3 + 2 * c], sc) != cudaSuccess || cudaStreamWaitEvent(sd, ev[3 + 2 * c], 0) != cudaSuccess ||
            (per_chunk && cudaEventRecord(chunk_ev[2 * c], sc) != cudaSuccess) ||
            cudaMemcpyAsync(static_cast<uint8_t*>(o_host) + off, w + p.off_o + off, bytes, cudaMemcpyDeviceToHost,
                            sd) != cudaSuccess ||
            (per_chunk && cudaEventRecord(chunk_ev[2 * c + 1], sd) != cudaSuccess))
            return cleanup(RF2_ERR_CUDA);
        h0 += p.sizes[c];
    }
    return cleanup(RF2_OK);
}

int rf2_host_events_create(int32_t count, void** events)
{
    if (count < 0 || (count > 0 && !events)) return RF2_ERR_INVALID_ARGUMENT;
    for (int32_t i = 0; i < count; ++i) {
        cudaEvent_t e;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
            for (int32_t k = 0; k < i; ++k) cudaEventDestroy(reinterpret_cast<cudaEvent_t>(events[k]));
            return RF2_ERR_CUDA;
        }
        events[i] = e;
    }
    return RF2_OK;
}

int rf2_host_events_destroy(int32_t count, void** events)
{
    if (count < 0 || (count > 0 && !events)) return RF2_ERR_INVALID_ARGUMENT;
    int st = RF2_OK;
    for (int32_t i = 0; i < count; ++i)
        if (events[i] && cudaEventDestroy(reinterpret_cast<cudaEvent_t>(events[i])) != cudaSuccess) st = RF2_ERR_CUDA;
    return st;
}

int rf2_device_status(void* stream)
{
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return RF2_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status_word, sizeof v) != cudaSuccess) return RF2_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof zero) != cudaSuccess) return RF2_ERR_CUDA;
    if (v & kDevErrRange) return RF2_ERR_RANGE;
    return (v & kDevErrTimeout) ? RF2_ERR_TIMEOUT : RF2_OK;
}

}  // extern "C"
