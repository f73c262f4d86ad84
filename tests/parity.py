"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare what it produced with the oracle, element by element."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from image_dits_b200 import rf2

# Tolerances for bf16 inputs: attention output against the fp64 oracle under
# the GPU's own mask; masks exact outside a 1e-5 band around the threshold.
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
TIE_BAND = 1e-5


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> uint16 numpy array of its bit patterns."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def run_path(geom, q, k, v, keep, lse=False, fused=True):
    """All calls of one attention invocation; returns a dict of outputs.
    fused: Q/K permutation fused with the block means (rf2_permute_qk_pool +
    rf2_predict_mask_pooled), else three rf2_permute calls + rf2_predict_mask."""
    if fused:
        mask, ws = rf2.alloc_mask(geom, keep, q.device)
        qp, kp = rf2.permute_qk_pool(geom, q, k, ws)
        vp = rf2.permute(geom, v)
        rf2.predict_mask_pooled(geom, keep, mask, ws)
    else:
        qp = rf2.permute(geom, q)
        kp = rf2.permute(geom, k)
        vp = rf2.permute(geom, v)
        mask = rf2.predict_mask(geom, qp, kp, keep)
    lse_t = None
    if lse:
        lse_t = torch.full((geom.batch * geom.heads * qp.shape[2],), float("nan"), device=q.device)
    op = rf2.block_sparse_attn(geom, qp, kp, vp, mask, lse=lse_t)
    o = rf2.unpermute(geom, op)
    torch.cuda.synchronize()
    assert rf2.device_status() == rf2.RF2_OK
    return dict(qp=qp, kp=kp, vp=vp, mask=mask, op=op, o=o, lse=lse_t)


def check_csr(mask: rf2.BlockMask, sink_first: int):
    """Rows ascending, unique, in range, within capacity, and sink columns present."""
    sz = mask.sizes
    Tb = sz.num_blocks
    rs = mask.row_start.cpu().numpy().astype(np.int64)
    rc = mask.row_count.cpu().numpy().astype(np.int64)
    ci = mask.col_idx.cpu().numpy()
    for r in range(rs.size):
        i = r % Tb
        cap = Tb if (sink_first >= 0 and i >= sink_first) else sz.row_capacity
        assert 1 <= rc[r] <= cap
        row = ci[rs[r]:rs[r] + rc[r]]
        assert np.all(np.diff(row) > 0) and row[0] >= 0 and row[-1] < Tb
        if sink_first >= 0:
            assert set(range(sink_first, Tb)) <= set(row.tolist())
            if i >= sink_first:
                assert rc[r] == Tb
    # closed-form offsets
    s0 = Tb if sink_first < 0 else sink_first
    head_total = s0 * sz.row_capacity + (Tb - s0) * Tb
    for r in range(rs.size):
        bh, i = divmod(r, Tb)
        exp = bh * head_total + (i * sz.row_capacity if i < s0 else s0 * sz.row_capacity + (i - s0) * Tb)
        assert rs[r] == exp


def compare_masks(gpu_dense: np.ndarray, qp_bits, kp_bits, keep, T, H, W, sink, text=0):
    """Bit-exact mask parity outside the tie band.  Returns (excluded, compared)."""
    omask, thr, S = oracle.predict_mask(qp_bits, kp_bits, keep, T, H, W, sink, text)
    omask = omask.reshape(gpu_dense.shape)
    S = S.reshape(gpu_dense.shape)
    thr = thr.reshape(gpu_dense.shape[:2])
    s0 = oracle.sink_start(T, H, W, sink, text)
    Tb = gpu_dense.shape[-1]
    band = np.abs(S - thr[..., None]) <= TIE_BAND
    if s0 >= 0:
        band[:, s0:, :] = False      # sink rows: no selection
        band[:, :, s0:] = False      # sink columns: always kept
    diff = (gpu_dense != omask) & ~band
    if diff.any():
        idx = np.argwhere(diff)[:5]
        raise AssertionError(f"{int(diff.sum())} mask entries differ outside the tie band, e.g. {idx.tolist()}: "
                             f"S={[S[tuple(i)] for i in idx]} thr={[thr[tuple(i[:2])] for i in idx]}")
    return int(band.sum()), int((~band).sum())


def attention_errors(op: torch.Tensor, qp_bits, kp_bits, vp_bits, gpu_dense, items=None, lse=None):
    """Errors of the GPU output (permuted order) against the oracle under the GPU's mask."""
    BH = gpu_dense.shape[0]
    N, d = qp_bits.shape[-2:]
    q = qp_bits.reshape(BH, N, d)
    k = kp_bits.reshape(BH, N, d)
    v = vp_bits.reshape(BH, N, d)
    ref, ref_lse = oracle.masked_attention(q, k, v, gpu_dense, items)
    got = bf16_to_f64(bits(op)).reshape(BH, N, d)
    if items is None:
        Tb = gpu_dense.shape[-1]
        items = np.stack(np.meshgrid(np.arange(BH), np.arange(Tb), indexing="ij"), -1).reshape(-1, 2)
    errs, lerrs = [], []
    lse_np = None if lse is None else lse.cpu().numpy().reshape(BH, N)
    for it, (bh, i) in enumerate(np.asarray(items)):
        r0, r1 = 64 * i, min(64 * i + 64, N)
        errs.append(np.abs(got[bh, r0:r1] - ref[it, :r1 - r0]))
        if lse_np is not None:
            lerrs.append(np.abs(lse_np[bh, r0:r1] - ref_lse[it, :r1 - r0]))
    e = np.concatenate([x.ravel() for x in errs])
    out = dict(max_abs=float(e.max()), mean_abs=float(e.mean()), n=int(e.size))
    if lerrs:
        out["lse_max_abs"] = float(np.concatenate(lerrs).max())
    return out


def full_size_items(BH, Tb, sink_first, n_random=64, seed=1):
    """Query blocks compared at full size: every sink row of the first and the
    last head (the longest rows: every key block, the most rescales), 64
    random non-sink blocks in each of four heads spread over the heads, and
    the ragged last block of the first and last head."""
    rng = np.random.default_rng(seed)
    heads = sorted({0, BH // 3, (2 * BH) // 3, BH - 1})
    upper = sink_first if 0 <= sink_first < Tb else Tb
    items = []
    if 0 <= sink_first < Tb:
        items += [(h, i) for h in (0, BH - 1) for i in range(sink_first, Tb)]
    for h in heads:
        picks = rng.choice(upper, size=min(n_random, upper), replace=False)
        items += [(h, int(i)) for i in picks]
    items += [(0, Tb - 1), (BH - 1, Tb - 1)]
    return sorted(set(items))
