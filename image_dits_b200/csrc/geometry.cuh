// Closed-form geometry of the window permutation, the block grid and the CSR
// row layout.  Used by host validation, rf2_permutation_index and the kernels.
//
// Window permutation ("RainFusion2.0", section 3.3 and section 1 Key Idea 2;
// first frame moved to the end, section 3.4).  The video part is one segment
// (frames 0..F-1), or, with the first-frame sink on and F > 1, two: frames
// 1..F-1 followed by frame 0.  Text tokens of a joint video-text attention
// (section 3.4: the first frame is moved next to them) follow the video
// tokens in the input and keep their place after the permuted video.  Each segment is tiled from its origin by
// windows of (wt, wh, ww) frames/rows/columns, cut short at the grid edge.
// Windows go in raster order and so do the tokens inside each window.
// Because every window before the last one along an axis is full-sized, the
// position p of a token decomposes with plain divisions:
//   p = seg_base + a*wt'*H*W + b*tsz*wh*W + c*tsz*hsz*ww + lt*hsz*wsz + lh*wsz + lw
// where (a, b, c) is the window, (lt, lh, lw) the offset inside it and
// (tsz, hsz, wsz) the window's (possibly cut) size.
#pragma once
#include <stdint.h>

#ifdef __CUDACC__
#define RF2_HD __host__ __device__ __forceinline__
#else
#define RF2_HD inline
#endif

namespace rf2 {

constexpr int kBlock = 64;

struct PermGeo {
    int32_t T, H, W;       // grid
    int32_t wt, wh, ww;    // window
    int32_t move_first;    // frame 0 moved behind frames 1..T-1
    int32_t HW;
    int32_t Nv;            // video tokens T*H*W
    int32_t N;             // Nv + text tokens
};

RF2_HD int32_t imin(int32_t a, int32_t b) { return a < b ? a : b; }

RF2_HD PermGeo make_perm_geo(int32_t T, int32_t H, int32_t W, int32_t wt, int32_t wh, int32_t ww,
                             int32_t sink, int32_t text)
{
    PermGeo g;
    g.T = T; g.H = H; g.W = W; g.wt = wt; g.wh = wh; g.ww = ww;
    g.move_first = (sink && T > 1) ? 1 : 0;
    g.HW = H * W;
    g.Nv = T * H * W;
    g.N = g.Nv + text;
    return g;
}

// Permuted position -> original raster index.
RF2_HD int32_t perm_src(const PermGeo& g, int32_t p)
{
    if (p >= g.Nv) return p;                               // text tokens
    const int32_t seg0 = g.move_first ? (g.T - 1) * g.HW : g.Nv;
    int32_t t0, F, q;
    if (p < seg0) { t0 = g.move_first; F = g.move_first ? g.T - 1 : g.T; q = p; }
    else          { t0 = 0;            F = 1;                          q = p - seg0; }
    const int32_t wts = imin(g.wt, F);
    const int32_t a = q / (wts * g.HW);
    q -= a * wts * g.HW;
    const int32_t tsz = imin(wts, F - a * wts);
    const int32_t b = q / (tsz * g.wh * g.W);
    q -= b * tsz * g.wh * g.W;
    const int32_t hsz = imin(g.wh, g.H - b * g.wh);
    const int32_t c = q / (tsz * hsz * g.ww);
    q -= c * tsz * hsz * g.ww;
    const int32_t wsz = imin(g.ww, g.W - c * g.ww);
    const int32_t lt = q / (hsz * wsz);
    q -= lt * hsz * wsz;
    const int32_t lh = q / wsz;
    const int32_t lw = q - lh * wsz;
    const int32_t t = t0 + a * wts + lt;
    return (t * g.H + b * g.wh + lh) * g.W + c * g.ww + lw;
}

// Original raster index -> permuted position (inverse of perm_src).
RF2_HD int32_t perm_dst(const PermGeo& g, int32_t s)
{
    if (s >= g.Nv) return s;                               // text tokens
    const int32_t t = s / g.HW;
    const int32_t hw = s - t * g.HW;
    const int32_t h = hw / g.W;
    const int32_t w = hw - h * g.W;
    int32_t base, F, tl;
    if (g.move_first) {
        if (t == 0) { base = (g.T - 1) * g.HW; F = 1; tl = 0; }
        else        { base = 0; F = g.T - 1; tl = t - 1; }
    } else {
        base = 0; F = g.T; tl = t;
    }
    const int32_t wts = imin(g.wt, F);
    const int32_t a = tl / wts, lt = tl - a * wts, tsz = imin(wts, F - a * wts);
    const int32_t b = h / g.wh, lh = h - b * g.wh, hsz = imin(g.wh, g.H - b * g.wh);
    const int32_t c = w / g.ww, lw = w - c * g.ww, wsz = imin(g.ww, g.W - c * g.ww);
    return base + a * wts * g.HW + b * tsz * g.wh * g.W + c * tsz * hsz * g.ww
         + lt * hsz * wsz + lh * wsz + lw;
}

// Block grid and CSR row layout of the mask (section 3.2, eq. (8), plus the
// sink of section 3.4).  Rows are stored at their capacity so that the offset
// of every row is a closed form and no scan is needed:
//   non-sink rows i < sink_first:  cap = min(Tb, n_keep + Tb - sink_first)
//   sink rows:                     Tb
struct MaskGeo {
    int32_t Tb;          // blocks per head
    int32_t n_keep;      // top-n
    int32_t sink_first;  // first sink block, Tb when there is no sink
    int32_t cap;         // capacity of a non-sink row
    int64_t head_total;  // col_idx slots per (b, h)
    int64_t col_capacity;  // col_idx slots in all (set by the host; checked build only)
};

// First token of the full-attention region of the permuted sequence: frame 0
// (at the end of the video part) when the first-frame sink is on, else the
// first text token; -1 when there is neither.
RF2_HD int32_t sink_first_token(const PermGeo& g, int32_t sink_on)
{
    if (sink_on) return (g.T - 1) * g.HW;
    return (g.N > g.Nv) ? g.Nv : -1;
}

RF2_HD MaskGeo make_mask_geo(int32_t N, int32_t n_keep, int32_t first_sink_token)
{
    MaskGeo m;
    m.Tb = (N + kBlock - 1) / kBlock;
    m.n_keep = n_keep;
    m.sink_first = (first_sink_token >= 0) ? first_sink_token / kBlock : m.Tb;
    const int32_t n_sink = m.Tb - m.sink_first;
    m.cap = imin(m.Tb, n_keep + n_sink);
    m.head_total = (int64_t)m.sink_first * m.cap + (int64_t)n_sink * m.Tb;
    m.col_capacity = INT64_MAX;
    return m;
}

RF2_HD int64_t row_offset(const MaskGeo& m, int64_t bh, int32_t i)
{
    const int64_t in_head = (i < m.sink_first)
        ? (int64_t)i * m.cap
        : (int64_t)m.sink_first * m.cap + (int64_t)(i - m.sink_first) * m.Tb;
    return bh * m.head_total + in_head;
}

}  // namespace rf2
