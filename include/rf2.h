/*
 * rf2.h — C ABI of a B200 (sm_100a) implementation of the block-wise sparse
 * attention of
 *
 *   "RainFusion2.0: Temporal-Spatial Awareness and Hardware-Efficient
 *    Block-wise Sparse Attention" (arXiv 2512.24086).
 *
 * One attention call of a DiT layer is four library calls on one stream:
 *
 *   rf2_permute(Q), rf2_permute(K), rf2_permute(V)       section 3.3 + 3.4
 *   rf2_predict_mask(Qp, Kp) -> block mask as CSR         section 3.2, eqs. (5)-(8) + 3.4
 *   rf2_block_sparse_attn(Qp, Kp, Vp, mask) -> Op         section 3.1, eqs. (1)-(4)
 *   rf2_unpermute(Op) -> O                                inverse of section 3.3
 *
 * Conventions shared by every call
 * --------------------------------
 * - Tensors are dense, row-major [batch, heads, N, head_dim] bf16 (d fastest),
 *   N = frames * height * width in the model's [F, H, W] raster order, or the
 *   permuted order for the "p" tensors.  Device pointers must be 16-byte
 *   aligned.  The caller owns every buffer; the library never allocates
 *   device memory, never synchronizes (except rf2_device_status) and keeps no
 *   state between calls (rf2_predict_mask_static's fixed scratch aside).
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   Every call is asynchronous on it and launches 1-2 kernels.
 * - Arguments are validated on the host before anything is launched; an
 *   invalid call returns an error status and launches nothing.  A failed
 *   launch returns RF2_ERR_CUDA (a pending error left by unrelated earlier
 *   work is cleared before the call launches, so it is not reported as this
 *   call's; an error that has made the context unusable is).  Kernels never trap: a bounded wait that
 *   runs out records RF2_ERR_TIMEOUT in a device status word that
 *   rf2_device_status reads back.
 * - Blocks are 64 consecutive tokens of the permuted sequence; T_b =
 *   ceil(N/64) and the last block may be short.
 * - The geometry must be identical across the four calls of one invocation.
 */
#ifndef RF2_H
#define RF2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RF2_OK = 0,
    RF2_ERR_INVALID_ARGUMENT = 1,     /* null/misaligned pointer, bad size or ratio */
    RF2_ERR_UNSUPPORTED = 2,          /* head_dim not 64/128, block not 64, too many blocks */
    RF2_ERR_INSUFFICIENT_WORKSPACE = 3,
    RF2_ERR_CUDA = 4,                 /* a CUDA runtime call or launch failed */
    RF2_ERR_TIMEOUT = 5,              /* a kernel's bounded wait ran out (device status) */
    RF2_ERR_RANGE = 6                 /* librf2_checked.so only: an index out of range was
                                         skipped (device status) */
} rf2_status;

/* Problem geometry.  The window (win_t, win_h, win_w) is the 3D (video) or 2D
 * (image, frames = 1) tile of section 3.3; the paper leaves its shape open, so
 * it is a parameter.  Windows tile each segment from its origin and are cut
 * short at the grid edge.  With first_frame_sink = 1 (section 3.4) frame 0 is
 * moved behind frames 1..F-1, every query block holding a first-frame token
 * keeps every key block, and every query block keeps every key block holding
 * a first-frame token.  Text tokens (text_tokens > 0; sequence length
 * N = frames*height*width + text_tokens) join that full-attention region
 * (section 3.4 groups the first frame with the text tokens of multimodal
 * models): with the sink on, the region starts at frame 0; with it off, at
 * the first text token. */
typedef struct {
    int32_t batch, heads, head_dim;     /* head_dim in {64, 128} */
    int32_t frames, height, width;      /* latent grid; frames = 1 for images */
    int32_t win_t, win_h, win_w;        /* permutation window, each >= 1 */
    int32_t block;                      /* query/key block size; 64 */
    int32_t first_frame_sink;           /* 0 or 1 */
    int32_t text_tokens;                /* >= 0: text tokens of a joint video-text attention, stored
                                           after the frames*height*width video tokens; they stay
                                           after the permuted video (behind frame 0) and take part
                                           in full attention as sink rows and columns (section 3.4) */
} rf2_geometry;

/* Derived sizes (rf2_query). */
typedef struct {
    int64_t num_tokens;          /* N */
    int32_t num_blocks;          /* T_b = ceil(N / 64) */
    int32_t n_keep;              /* top-n per query block: ceil(keep * T_b), in [1, T_b] */
    int32_t sink_first;          /* first sink block, -1 when the sink is off */
    int32_t row_capacity;        /* col_idx slots of a non-sink row: min(T_b, n_keep + sink blocks) */
    int64_t num_rows;            /* batch * heads * T_b: length of row_start / row_count */
    int64_t col_idx_capacity;    /* length of col_idx */
    size_t  mask_workspace_bytes;/* scratch for rf2_predict_mask: the block means as a
                                    tf32 hi/lo pair of fp32 arrays, then the larger of
                                    (a) the pooled scores of as many heads as fit in
                                    96 MiB (at least one head; all of them when they
                                    fit) and (b) two bytes of score code per score,
                                    per-row code histograms and widths and a row list
                                    (the top-n path for T_b <= 2048) */
} rf2_sizes;

/* Human-readable name of a status code (static string, never NULL). */
const char* rf2_status_string(int status);

/* Sizes for a geometry and keep ratio (the fraction of key blocks each query
 * block keeps before the sink is added: 0.2 = "80% sparsity").  Host only.
 * Returns RF2_ERR_INVALID_ARGUMENT / RF2_ERR_UNSUPPORTED for bad input. */
int rf2_query(const rf2_geometry* geom, double keep_ratio, rf2_sizes* out);

/* The window permutation of sections 3.3-3.4 as a host table:
 * perm[p] = [F,H,W] raster index of the token placed at permuted position p.
 * perm must hold N int32.  Host only; no device work. */
int rf2_permutation_index(const rf2_geometry* geom, int32_t* perm);

/* Xp[b,h,p,:] = X[b,h,perm[p],:] — gathers every (b, h) slice into window
 * order (sections 3.3-3.4).  X and Xp must not overlap.  Pure copy: bit exact. */
int rf2_permute(const rf2_geometry* geom, const void* x_bf16, void* xp_bf16, void* stream);

/* X[b,h,perm[p],:] = Xp[b,h,p,:] — the inverse of rf2_permute, returning the
 * attention output to the model's [F,H,W] order.  Bit exact. */
int rf2_unpermute(const rf2_geometry* geom, const void* xp_bf16, void* x_bf16, void* stream);

/* Online block-mask prediction (section 3.2, eqs. (5)-(8), and section 3.4).
 *   q^_i = mean of the valid rows of query block i (fp32), likewise k^_j;
 *   S^_ij = q^_i . k^_j / sqrt(d) (tensor cores, tf32 hi/lo split: about
 *           2^-21 relative error, i.e. fp32 accuracy);
 *   a non-sink row keeps its n_keep largest S^_ij (equal scores: lower j
 *   first) plus every sink column; a sink row keeps every column.
 * Output is one CSR row per (b, h, i), r = (b*heads + h)*T_b + i:
 *   row_start[r]  closed-form offset into col_idx (rows are laid out at
 *                 their capacity, so col_idx may have gaps),
 *   row_count[r]  number of kept key blocks,
 *   col_idx[row_start[r] .. + row_count[r]) kept key blocks, ascending.
 * row_start/row_count hold num_rows int32, col_idx col_idx_capacity int32,
 * workspace at least mask_workspace_bytes (device, 16-byte aligned); its
 * contents on entry do not matter.  qp/kp are the permuted Q and K.
 * Two selections give the same masks outside a 1e-5 band around each row's
 * threshold: from the score matrix (chosen while the scores of all heads
 * fit in 96 MiB) and, for larger calls with T_b <= 2048, from 16-bit codes
 * of the scores that never leave the SM as floats.  The environment
 * variable RF2_MASK_SELECT = "scores" or "codes" forces one of them (read
 * on every call; "codes" still needs T_b <= 2048). */
int rf2_predict_mask(const rf2_geometry* geom, const void* qp_bf16, const void* kp_bf16,
                     double keep_ratio, int32_t* row_start, int32_t* row_count, int32_t* col_idx,
                     void* workspace, size_t workspace_bytes, void* stream);

/* rf2_predict_mask without a caller-supplied workspace: the same arguments
 * and outputs, with the block-mean scratch taken from a fixed 64 MiB array
 * inside the library instead.  For callers that cannot allocate device
 * memory themselves — for example code embedded in a host framework that
 * owns the device allocator and hands out no workspace, or a latency-critical
 * loop where cudaMalloc's implicit device synchronization is not acceptable.
 * (The paper has no counterpart to this call; it exists only for such callers.)
 * - Limit: the block means as a hi/lo pair (2 x 2*batch*heads*T_b*head_dim*4
 *   bytes) plus the pooled scores of one head (T_b*ceil4(T_b)*4 bytes) must
 *   fit in 64 MiB (67,108,864), i.e. batch*heads <= 25 at 720p (75,600
 *   tokens, d = 128);
 *   larger problems return RF2_ERR_INSUFFICIENT_WORKSPACE and launch nothing
 *   (split the heads over several calls, or use rf2_predict_mask).
 * - It always selects from the score matrix (rf2_predict_mask with
 *   RF2_MASK_SELECT=scores gives the identical mask; without it, large calls
 *   of rf2_predict_mask select from codes and may differ inside the 1e-5 tie
 *   band of a row's threshold).
 * - Every GPU that loads the library holds the 64 MiB until the process exits.
 * - Every call looks up the array's device address on the calling thread's
 *   current device (cudaGetSymbolAddress; nothing is cached, so a context
 *   created anew after cudaDeviceReset is served correctly).  The first call
 *   on a device also loads the library's device code there: make it before
 *   any stream capture.  No call allocates, or calls an allocating routine.
 * - All calls share the one array and it keeps the last call's contents;
 *   nothing in it needs to start at zero, but calls that overlap on the GPU
 *   (different streams, or different host threads on one device) race on it.
 * Arguments, outputs and errors are otherwise those of rf2_predict_mask. */
int rf2_predict_mask_static(const rf2_geometry* geom, const void* qp_bf16, const void* kp_bf16,
                            double keep_ratio, int32_t* row_start, int32_t* row_count, int32_t* col_idx,
                            void* stream);

/* The permutation of Q and K fused with the block means of mask prediction
 * (sections 3.3-3.4 and eqs. (5)-(6)): writes Qp and Kp exactly as
 * rf2_permute does, and the block means of Qp and Kp into `workspace`
 * (a buffer of at least mask_workspace_bytes) while the rows pass through, so
 * the mask step need not read Qp and Kp again.  Follow it with
 * rf2_predict_mask_pooled on the same workspace; the masks equal those of
 * rf2_permute + rf2_predict_mask bit for bit.  Inputs and outputs must not
 * overlap. */
int rf2_permute_qk_pool(const rf2_geometry* geom, const void* q_bf16, const void* k_bf16, void* qp_bf16,
                        void* kp_bf16, void* workspace, size_t workspace_bytes, void* stream);

/* Mask prediction (section 3.2 eqs. (7)-(8), section 3.4) from the block
 * means that rf2_permute_qk_pool left in `workspace`; outputs and errors as
 * rf2_predict_mask. */
int rf2_predict_mask_pooled(const rf2_geometry* geom, double keep_ratio, int32_t* row_start, int32_t* row_count,
                            int32_t* col_idx, void* workspace, size_t workspace_bytes, void* stream);

/* Mask prediction with CDF-threshold selection instead of a fixed top-n: the
 * alternative the pages name among the online adaptive patterns (section 2,
 * "Related Work" (2): block means -> scores -> the top blocks whose
 * cumulative distribution meets a threshold).  Per non-sink query-block row,
 * the pooled scores (eqs. (5)-(7)) are turned into p_j = softmax_j(S_ij); the
 * key blocks are ordered by (score desc, j asc) and the shortest prefix whose
 * cumulative p reaches tau (0 < tau <= 1) is kept; the first-frame sink is
 * added as in rf2_predict_mask (section 3.4).  Rows are adaptive: every row
 * has capacity T_b, so size the outputs with rf2_query(geom, 1.0, ...)
 * (col_idx_capacity = B*H*T_b^2, row_start[r] = r*T_b); the workspace is
 * mask_workspace_bytes of the same query.  Arithmetic is fp32 (weights
 * 2^((S - max) log2 e), sums in a fixed order, so the result is
 * deterministic).  tau outside (0, 1] -> RF2_ERR_INVALID_ARGUMENT; other
 * errors as rf2_predict_mask. */
int rf2_predict_mask_cdf(const rf2_geometry* geom, const void* qp_bf16, const void* kp_bf16, double tau,
                         int32_t* row_start, int32_t* row_count, int32_t* col_idx, void* workspace,
                         size_t workspace_bytes, void* stream);

/* The same from the block means rf2_permute_qk_pool left in `workspace`. */
int rf2_predict_mask_cdf_pooled(const rf2_geometry* geom, double tau, int32_t* row_start, int32_t* row_count,
                                int32_t* col_idx, void* workspace, size_t workspace_bytes, void* stream);

/* Block-sparse FlashAttention forward (section 3.1): for every query block i,
 * O_i = softmax(Q_i K_J^T / sqrt(d)) V_J over the key blocks J kept in row i
 * of the CSR mask (eqs. (1)-(4); Q_i K_j^T and P_ij V_j are skipped when
 * M_ij = 0).  bf16 operands, fp32 accumulation and fp32 softmax, P rounded to
 * bf16 as the operand of the PV product.  op receives bf16 [B,H,N,d]; lse,
 * when not NULL, receives the natural-log row sums fp32 [B,H,N].  Every row
 * must keep at least one key block; col_idx entries must lie in [0, T_b) and
 * ascend within a row (as rf2_predict_mask writes them). */
int rf2_block_sparse_attn(const rf2_geometry* geom, const void* qp_bf16, const void* kp_bf16,
                          const void* vp_bf16, const int32_t* row_start, const int32_t* row_count,
                          const int32_t* col_idx, void* op_bf16, float* lse, void* stream);

/* One attention call on HOST memory, end to end: the host-to-device copy of
 * Q, K, V, the whole path (rf2_permute_qk_pool, rf2_permute of V,
 * rf2_predict_mask_pooled or rf2_predict_mask_cdf_pooled, rf2_block_sparse_attn,
 * rf2_unpermute) and the device-to-host copy of O.  The (batch, head) problems
 * are independent (sections 3.1-3.4 are all per head), so the B*H heads go in
 * chunks: `chunks` near-equal ones, the last split further into shrinking
 * parts down to one head (what follows the last input copy is then small).
 * Chunk c's input copies run on stream_h2d, its computation on
 * stream_compute, its output copy on stream_d2h; the copies of one chunk
 * overlap the computation of another.  Each chunk is computed by the same
 * calls on a geometry of its heads, so O is bit-identical to the calls on the
 * whole tensors.
 *   keep_ratio, tau   exactly one > 0: top-n selection with keep_ratio, or
 *                     the CDF threshold with tau (both in (0, 1])
 *   q/k/v/o_host      bf16 [B, H, N, d] in page-locked host memory (16-byte
 *                     aligned); o_host is written
 *   work              device scratch of at least rf2_attention_host_query's
 *                     work_bytes (256-byte aligned); the library allocates
 *                     no memory (it creates and destroys a few CUDA events)
 *   stream_*          three streams (may not be the same stream twice)
 *   events, num_events  NULL / 0, or 2 * num_chunks events from
 *                     rf2_host_events_create, the same array on every call
 *                     with this `work` (see below)
 * Returns after enqueueing: the host buffers and `work` must stay untouched
 * until stream_d2h has completed.  Calls one after another on the same
 * `work` are ordered: without events, a call's copies wait for everything
 * already on stream_compute and its computation for everything already on
 * stream_d2h; with events, chunk c of a call waits only for chunk c of the
 * previous call (its computation before the copy into the chunk's inputs,
 * its copy-back before the computation into the chunk's output), so the
 * input copies of the next call start while the previous one computes.
 * Errors as the calls it makes; after an error part of the work may be
 * enqueued. */
typedef struct {
    int32_t num_chunks;      /* chunks after the tail split */
    int32_t max_chunk_heads; /* heads of the largest chunk */
    size_t  work_bytes;      /* device scratch rf2_attention_host needs */
} rf2_host_sizes;

int rf2_attention_host_query(const rf2_geometry* geom, double keep_ratio, double tau, int32_t chunks,
                             rf2_host_sizes* out);
int rf2_attention_host(const rf2_geometry* geom, double keep_ratio, double tau, int32_t chunks,
                       const void* q_host, const void* k_host, const void* v_host, void* o_host, void* work,
                       size_t work_bytes, void* stream_h2d, void* stream_compute, void* stream_d2h,
                       void** events, int32_t num_events);

/* `count` CUDA events (timing disabled) for rf2_attention_host, created on
 * the current device into events[0 .. count); destroy them with
 * rf2_host_events_destroy once no enqueued call uses them. */
int rf2_host_events_create(int32_t count, void** events);
int rf2_host_events_destroy(int32_t count, void** events);

/* Synchronizes `stream`, then returns and clears the device status word of
 * the calling thread's current device: RF2_OK, RF2_ERR_TIMEOUT if a kernel's
 * bounded wait ran out since the last call, or (checked library only, ahead
 * of a timeout) RF2_ERR_RANGE if a range check failed.
 *
 * The checked library, librf2_checked.so, is this library compiled with
 * RF2_CHECKED=1: the same entry points and results, plus range checks in the
 * kernels, each of which, when it fails, records RF2_ERR_RANGE here and skips
 * the access: the CSR rows the attention reads (row_count in [0, T_b],
 * row_start >= 0 and row_start + row_count within B*H*T_b^2, the largest
 * layout the library writes; col_idx values in [0, T_b)), every col_idx
 * store of the mask kernels against the mask's col_idx_capacity, and every
 * computed permutation source row against [0, N). */
int rf2_device_status(void* stream);

/* Self-test of failure detection (tests only).  Launches, on `stream`, one
 * CTA of two warps that wait on mbarriers nothing completes: the first gives
 * up after `limit_us` microseconds (1 .. 1,000,000), records RF2_ERR_TIMEOUT in
 * the device status word (read it with rf2_device_status) and raises the
 * CTA's abort flag, through which the second leaves too -- the same bounded
 * waits and abort path every kernel of the library uses.  Nothing faults and
 * the context stays usable.  Synchronizes `stream`; *waits_given_up (host)
 * receives the number of waits that ended without their barrier (2 when the
 * path works).  Returns RF2_ERR_INVALID_ARGUMENT for a null pointer or a limit
 * out of range. */
int rf2_selftest_wait_timeout(uint32_t limit_us, int32_t* waits_given_up, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RF2_H */
