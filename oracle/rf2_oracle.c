/*
 * Plain CPU oracle for RainFusion2.0 block-wise sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link or call
 * this file; only tests/, the smoke check and the bench's CPU-baseline leg do.
 * It shares no code, header or constant with the CUDA library.
 *
 * Every step is written as the plain definition the paper gives, in fp64, on
 * bf16 inputs converted exactly:
 *
 *   "RainFusion2.0: Temporal-Spatial Awareness and Hardware-Efficient
 *    Block-wise Sparse Attention", arXiv 2512.24086
 *   - section 3.1 "Blockwise Sparse": S = QK^T/sqrt(d), P = Softmax(S), O = PV;
 *     blocks of b rows, ceil(N/b) of them; block mask M skips Q_i K_j^T and
 *     P_ij V_j when M_ij = 0.
 *   - section 3.2 "Representative Token for Blocks", eqs. (5)-(8): block means
 *     q^_i, k^_j, pooled scores S^_ij = q^_i k^_j^T, top-n key blocks per
 *     query block.
 *   - section 3.3 "3D Window Permutation" and Key Idea 2 of section 1: tokens
 *     regrouped window by window, raster order inside and across windows.
 *   - section 3.4 "First Frame Sink": first-frame queries see every key, every
 *     query sees the first-frame keys, and the first frame is moved to the end
 *     of the sequence.
 *
 * Readings where the paper is silent (window shape, ragged edges, block-level
 * sink, 1/sqrt(d) on S^, tie order) are fixed by the caller-visible arguments
 * below and are the same ones the library documents.
 *
 * Attention is the definition itself (max-shifted softmax over the kept keys
 * of each query row), not the online recurrence of eqs. (1)-(4): the two are
 * algebraically identical, and the definition is the one a reader can check.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_BLOCK 64

static double bf16_bits_to_double(uint16_t u)
{
    uint32_t bits = ((uint32_t)u) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------- */
/* Permutation (section 3.3, section 3.4 last paragraph).                    */
/* ------------------------------------------------------------------------- */

typedef struct {
    int64_t k[7];   /* segment, window t, window h, window w, t, h, w */
    int64_t src;    /* original [F,H,W] raster index */
} perm_entry;

static int perm_entry_cmp(const void* a, const void* b)
{
    const perm_entry* x = (const perm_entry*)a;
    const perm_entry* y = (const perm_entry*)b;
    for (int i = 0; i < 7; ++i) {
        if (x->k[i] < y->k[i]) return -1;
        if (x->k[i] > y->k[i]) return 1;
    }
    /* ties cannot happen (t,h,w is unique) but keep the sort total */
    return (x->src < y->src) ? -1 : (x->src > y->src);
}

/*
 * perm[p] = original token index placed at permuted position p.
 *
 * Sort key of token (t,h,w): (segment, t'/wt, h/wh, w/ww, t', h, w) where,
 * when the first-frame sink is on and there is more than one frame, frame 0
 * forms segment 1 (placed last, section 3.4) and frames 1..F-1 form segment 0
 * with t' = t-1; otherwise everything is segment 0 with t' = t.  Windows tile
 * each segment from its origin and are cut short at the grid edge; windows and
 * the tokens inside a window are both taken in raster order (t, then h, then w).
 */
int orc_permutation(int T, int H, int W, int wt, int wh, int ww, int sink, int64_t* perm)
{
    if (T <= 0 || H <= 0 || W <= 0 || wt <= 0 || wh <= 0 || ww <= 0 || !perm) return 1;
    const int64_t N = (int64_t)T * H * W;
    perm_entry* e = (perm_entry*)malloc(sizeof(perm_entry) * (size_t)N);
    if (!e) return 2;
    const int move_first = (sink && T > 1);
    int64_t q = 0;
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h)
            for (int w = 0; w < W; ++w, ++q) {
                int64_t seg = (move_first && t == 0) ? 1 : 0;
                int64_t tl = move_first ? (t == 0 ? 0 : t - 1) : t;
                e[q].k[0] = seg;
                e[q].k[1] = tl / wt;
                e[q].k[2] = h / wh;
                e[q].k[3] = w / ww;
                e[q].k[4] = tl;
                e[q].k[5] = h;
                e[q].k[6] = w;
                e[q].src = ((int64_t)t * H + h) * W + w;
            }
    qsort(e, (size_t)N, sizeof(perm_entry), perm_entry_cmp);
    for (int64_t p = 0; p < N; ++p) perm[p] = e[p].src;
    free(e);
    return 0;
}

/* xp[bh, p, :] = x[bh, perm[p], :] on raw bf16 bit patterns (a pure copy). */
void orc_permute_rows(const uint16_t* x, uint16_t* xp, int64_t BH, int64_t N, int64_t d,
                      const int64_t* perm)
{
    #pragma omp parallel for schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t p = 0; p < N; ++p)
            memcpy(xp + (bh * N + p) * d, x + (bh * N + perm[p]) * d, sizeof(uint16_t) * (size_t)d);
}

/* x[bh, perm[p], :] = xp[bh, p, :]: the inverse reordering. */
void orc_unpermute_rows(const uint16_t* xp, uint16_t* x, int64_t BH, int64_t N, int64_t d,
                        const int64_t* perm)
{
    #pragma omp parallel for schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t p = 0; p < N; ++p)
            memcpy(x + (bh * N + perm[p]) * d, xp + (bh * N + p) * d, sizeof(uint16_t) * (size_t)d);
}

/* ------------------------------------------------------------------------- */
/* Representative tokens, eqs. (5)-(6): mean of each 64-row block.           */
/* The last block may be short; its mean is over the rows it has.           */
/* ------------------------------------------------------------------------- */
void orc_block_means(const uint16_t* xp, int64_t BH, int64_t N, int64_t d, double* means)
{
    const int64_t Tb = (N + ORC_BLOCK - 1) / ORC_BLOCK;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t i = 0; i < Tb; ++i) {
            const int64_t r0 = i * ORC_BLOCK;
            const int64_t r1 = (r0 + ORC_BLOCK < N) ? r0 + ORC_BLOCK : N;
            double* m = means + (bh * Tb + i) * d;
            for (int64_t c = 0; c < d; ++c) m[c] = 0.0;
            for (int64_t r = r0; r < r1; ++r) {
                const uint16_t* row = xp + (bh * N + r) * d;
                for (int64_t c = 0; c < d; ++c) m[c] += bf16_bits_to_double(row[c]);
            }
            for (int64_t c = 0; c < d; ++c) m[c] /= (double)(r1 - r0);
        }
}

/* Pooled scores, eq. (7) with the 1/sqrt(d) of section 3.1: S^ = q^ k^T / sqrt(d). */
void orc_pooled_scores(const double* qm, const double* km, int64_t BH, int64_t Tb, int64_t d,
                       double* S)
{
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t i = 0; i < Tb; ++i) {
            const double* q = qm + (bh * Tb + i) * d;
            for (int64_t j = 0; j < Tb; ++j) {
                const double* k = km + (bh * Tb + j) * d;
                double acc = 0.0;
                for (int64_t c = 0; c < d; ++c) acc += q[c] * k[c];
                S[(bh * Tb + i) * Tb + j] = acc * inv_sqrt_d;
            }
        }
}

/* ------------------------------------------------------------------------- */
/* Block mask, eq. (8) plus the first-frame sink of section 3.4.             */
/* ------------------------------------------------------------------------- */
typedef struct { double v; int64_t j; } scored;

static int scored_cmp(const void* a, const void* b)
{
    const scored* x = (const scored*)a;
    const scored* y = (const scored*)b;
    if (x->v > y->v) return -1;   /* larger score first */
    if (x->v < y->v) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);  /* equal scores: lower block first */
}

/*
 * mask[bh, i, j] = 1 iff key block j is kept for query block i.
 * Non-sink rows keep their n best-scoring key blocks (equal scores: lower j
 * first), then every sink column is added.  Rows in the sink (sink_start <= i)
 * keep every column.  sink_start < 0 means "no sink".
 * thr[bh, i] receives the n-th best score of the row (NaN for sink rows).
 */
void orc_select_blocks(const double* S, int64_t BH, int64_t Tb, int64_t n, int64_t sink_start,
                       uint8_t* mask, double* thr)
{
    #pragma omp parallel
    {
        scored* buf = (scored*)malloc(sizeof(scored) * (size_t)Tb);
        #pragma omp for collapse(2) schedule(static)
        for (int64_t bh = 0; bh < BH; ++bh)
            for (int64_t i = 0; i < Tb; ++i) {
                uint8_t* m = mask + (bh * Tb + i) * Tb;
                const double* s = S + (bh * Tb + i) * Tb;
                if (sink_start >= 0 && i >= sink_start) {
                    for (int64_t j = 0; j < Tb; ++j) m[j] = 1;
                    thr[bh * Tb + i] = NAN;
                    continue;
                }
                for (int64_t j = 0; j < Tb; ++j) { buf[j].v = s[j]; buf[j].j = j; m[j] = 0; }
                qsort(buf, (size_t)Tb, sizeof(scored), scored_cmp);
                for (int64_t r = 0; r < n; ++r) m[buf[r].j] = 1;
                thr[bh * Tb + i] = buf[n - 1].v;
                if (sink_start >= 0)
                    for (int64_t j = sink_start; j < Tb; ++j) m[j] = 1;
            }
        free(buf);
    }
}

/*
 * CDF-threshold selection ("RainFusion2.0" section 2, online adaptive
 * patterns: the top blocks of the pooled-score attention are kept until
 * their cumulative distribution reaches a threshold), with the sink of
 * section 3.4 added as for top-n.
 * Per non-sink row: p_j = exp(S_ij - max_j S_ij) / sum_j exp(...), the key
 * blocks in the order (score desc, j asc), and the first m of them kept,
 * m = the smallest count whose cumulative p reaches tau (tau in (0, 1]).
 * Sink rows keep every column.
 * cum[bh, i, 0] / cum[bh, i, 1] receive the cumulative p of the first m-1 and
 * of the first m blocks (NaN for sink rows); bnd[bh, i] the score of the
 * m-th block.
 */
void orc_select_cdf(const double* S, int64_t BH, int64_t Tb, double tau, int64_t sink_start,
                    uint8_t* mask, double* cum, double* bnd)
{
    #pragma omp parallel
    {
        scored* buf = (scored*)malloc(sizeof(scored) * (size_t)Tb);
        #pragma omp for collapse(2) schedule(static)
        for (int64_t bh = 0; bh < BH; ++bh)
            for (int64_t i = 0; i < Tb; ++i) {
                const int64_t row = bh * Tb + i;
                uint8_t* m = mask + row * Tb;
                const double* s = S + row * Tb;
                if (sink_start >= 0 && i >= sink_start) {
                    for (int64_t j = 0; j < Tb; ++j) m[j] = 1;
                    cum[2 * row] = NAN;
                    cum[2 * row + 1] = NAN;
                    bnd[row] = NAN;
                    continue;
                }
                double mx = s[0];
                for (int64_t j = 1; j < Tb; ++j) mx = s[j] > mx ? s[j] : mx;
                double z = 0.0;
                for (int64_t j = 0; j < Tb; ++j) z += exp(s[j] - mx);
                for (int64_t j = 0; j < Tb; ++j) { buf[j].v = s[j]; buf[j].j = j; m[j] = 0; }
                qsort(buf, (size_t)Tb, sizeof(scored), scored_cmp);
                double c = 0.0, before = 0.0;
                int64_t r = 0;
                for (; r < Tb; ++r) {
                    before = c;
                    c += exp(buf[r].v - mx) / z;
                    m[buf[r].j] = 1;
                    if (c >= tau) break;
                }
                if (r == Tb) r = Tb - 1;               /* rounding kept the sum below tau */
                cum[2 * row] = before;
                cum[2 * row + 1] = c;
                bnd[row] = buf[r].v;
                if (sink_start >= 0)
                    for (int64_t j = sink_start; j < Tb; ++j) m[j] = 1;
            }
        free(buf);
    }
}

/* ------------------------------------------------------------------------- */
/* Attention under a block mask (section 3.1): for every valid query row x of */
/* block i, softmax(q_x K_J^T / sqrt(d)) V_J over the valid key rows of the   */
/* kept blocks J.  Computed only for the listed (bh, i) items.                */
/* out: [n_items, 64, d] (rows past the end of the sequence stay 0)           */
/* lse: [n_items, 64] natural-log sum of exp of the scaled scores             */
/* ------------------------------------------------------------------------- */
void orc_masked_attention(const uint16_t* qp, const uint16_t* kp, const uint16_t* vp,
                          int64_t BH, int64_t N, int64_t d, const uint8_t* mask,
                          const int64_t* items, int64_t n_items, double* out, double* lse)
{
    const int64_t Tb = (N + ORC_BLOCK - 1) / ORC_BLOCK;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    #pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)N);
        int64_t* y_of = (int64_t*)malloc(sizeof(int64_t) * (size_t)N);
        double* q = (double*)malloc(sizeof(double) * (size_t)d);
        #pragma omp for collapse(2) schedule(dynamic, 4)
        for (int64_t it = 0; it < n_items; ++it)
            for (int64_t rr = 0; rr < ORC_BLOCK; ++rr) {
                const int64_t bh = items[2 * it];
                const int64_t i = items[2 * it + 1];
                const int64_t x = i * ORC_BLOCK + rr;
                double* o = out + (it * ORC_BLOCK + rr) * d;
                for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
                lse[it * ORC_BLOCK + rr] = 0.0;
                if (x >= N) continue;
                for (int64_t c = 0; c < d; ++c) q[c] = bf16_bits_to_double(qp[(bh * N + x) * d + c]);
                const uint8_t* m = mask + (bh * Tb + i) * Tb;
                int64_t cnt = 0;
                double mx = -INFINITY;
                for (int64_t j = 0; j < Tb; ++j) {
                    if (!m[j]) continue;
                    const int64_t y1 = ((j + 1) * ORC_BLOCK < N) ? (j + 1) * ORC_BLOCK : N;
                    for (int64_t y = j * ORC_BLOCK; y < y1; ++y) {
                        const uint16_t* k = kp + (bh * N + y) * d;
                        double acc = 0.0;
                        for (int64_t c = 0; c < d; ++c) acc += q[c] * bf16_bits_to_double(k[c]);
                        acc *= inv_sqrt_d;
                        s[cnt] = acc;
                        y_of[cnt] = y;
                        ++cnt;
                        if (acc > mx) mx = acc;
                    }
                }
                double den = 0.0;
                for (int64_t u = 0; u < cnt; ++u) {
                    const double p = exp(s[u] - mx);
                    den += p;
                    const uint16_t* v = vp + (bh * N + y_of[u]) * d;
                    for (int64_t c = 0; c < d; ++c) o[c] += p * bf16_bits_to_double(v[c]);
                }
                for (int64_t c = 0; c < d; ++c) o[c] /= den;
                lse[it * ORC_BLOCK + rr] = mx + log(den);
            }
        free(s);
        free(y_of);
        free(q);
    }
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
