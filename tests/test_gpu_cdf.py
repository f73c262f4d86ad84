"""GPU parity of CDF-threshold block selection (rf2_predict_mask_cdf and
rf2_predict_mask_cdf_pooled) against the oracle, on the same seeded inputs.

Masks are compared exactly except, per non-sink row, at the selection
boundary: blocks whose oracle score lies within 1e-5 of the last kept block's
score, and, where the oracle's cumulative mass before or after the last kept
block lies within 1e-5 of tau, the last kept block and the next one in the
(score desc, j asc) order.  Attention under the GPU's CDF mask (adaptive row
lengths) is checked like the top-n path.
"""
import numpy as np
import pytest
import torch

import oracle
from image_dits_b200 import build as rf2_build
from image_dits_b200 import rf2
from image_dits_b200.workload import WORKLOADS, Workload, make_qkv
from parity import ATTN_MAX_ABS, ATTN_MEAN_ABS, attention_errors, bits, check_csr, full_size_items

pytestmark = pytest.mark.gpu
BAND = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    rf2_build.build()
    rf2.lib()
    yield
    torch.cuda.synchronize()


def compare_cdf_masks(gpu_dense, qp_b, kp_b, tau, T, H, W, sink, text=0):
    """Exact comparison outside the boundary band.  Returns (excluded, compared)."""
    omask, cum, bnd, S = oracle.predict_mask_cdf(qp_b, kp_b, tau, T, H, W, sink, text)
    Tb = gpu_dense.shape[-1]
    omask = omask.reshape(gpu_dense.shape)
    S = S.reshape(gpu_dense.shape)
    cum = cum.reshape(gpu_dense.shape[:2] + (2,))
    bnd = bnd.reshape(gpu_dense.shape[:2])
    s0 = oracle.sink_start(T, H, W, sink, text)
    excl = np.abs(S - bnd[..., None]) <= BAND
    near = (np.abs(cum[..., 0] - tau) <= BAND) | (np.abs(cum[..., 1] - tau) <= BAND)
    for bh, i in zip(*np.nonzero(near)):
        # the prefix length m in the (score desc, j asc) order, located in fp64
        order = np.lexsort((np.arange(Tb), -S[bh, i]))
        p = np.exp(S[bh, i] - S[bh, i].max())
        c = np.cumsum(p[order] / p.sum())
        m = int(np.argmax(c >= tau)) + 1 if (c >= tau).any() else Tb
        for pos in (m - 1, m):
            if 0 <= pos < Tb:
                excl[bh, i, order[pos]] = True
    if s0 >= 0:
        excl[:, s0:, :] = False
        excl[:, :, s0:] = False
    diff = (gpu_dense != omask) & ~excl
    assert not diff.any(), f"{int(diff.sum())} mask mismatches outside the boundary band"
    return int(excl.sum()), int((~excl).sum())


def _run(wl, tau, fused):
    q, k, v = make_qkv(wl, "cuda", seed=3)
    g = rf2.geometry_of(wl)
    mask, ws = rf2.alloc_mask(g, 1.0, q.device)
    if fused:
        qp, kp = rf2.permute_qk_pool(g, q, k, ws)
        rf2.predict_mask_cdf_pooled(g, tau, mask, ws)
    else:
        qp, kp = rf2.permute(g, q), rf2.permute(g, k)
        rf2.predict_mask_cdf(g, qp, kp, tau, mask, ws)
    vp = rf2.permute(g, v)
    op = rf2.block_sparse_attn(g, qp, kp, vp, mask)
    torch.cuda.synchronize()
    assert rf2.device_status() == rf2.RF2_OK
    return dict(qp=qp, kp=kp, vp=vp, mask=mask, op=op)


def _cases():
    W = Workload
    return [
        ("tiny", WORKLOADS["tiny"], 0.5),
        ("ragged_d128", W("c1", 1, 3, 128, 3, 7, 9, 2, 4, 4, 0.3, True, (44, 42, 42)), 0.3),
        ("ragged_d64_nosink", W("c2", 2, 1, 64, 2, 13, 11, 2, 3, 5, 0.5, False, (24, 20, 20)), 0.7),
        ("single_frame_sink", W("c3", 1, 2, 128, 1, 16, 20, 1, 8, 8, 0.25, True, (0, 64, 64)), 0.5),
        ("qwen_image", WORKLOADS["qwen_image"], 0.4),
        ("tau_one", W("c4", 1, 2, 64, 2, 12, 16, 2, 4, 4, 1.0, True, (24, 20, 20)), 1.0),
        ("tau_tiny", W("c5", 1, 2, 128, 3, 16, 16, 1, 8, 8, 0.01, True, (44, 42, 42)), 1e-4),
        ("text_nosink", W("c6", 1, 2, 64, 2, 8, 8, 2, 4, 4, 0.4, False, (24, 20, 20), 70), 0.4),
    ]


@pytest.mark.parametrize("name,wl,tau", _cases())
def test_cdf_small_parity(name, wl, tau):
    out = _run(wl, tau, fused=(name != "tiny"))
    sz = out["mask"].sizes
    check_csr(out["mask"], sz.sink_first)
    dense = out["mask"].dense()
    excluded, compared = compare_cdf_masks(dense, bits(out["qp"]), bits(out["kp"]), tau, wl.frames, wl.height,
                                           wl.width, wl.sink, wl.text_tokens)
    # at most the two boundary blocks of each row, plus score ties
    assert excluded <= 2 * dense.shape[0] * dense.shape[1] + 0.01 * compared
    e = attention_errors(out["op"], bits(out["qp"]), bits(out["kp"]), bits(out["vp"]), dense)
    assert e["max_abs"] <= ATTN_MAX_ABS and e["mean_abs"] <= ATTN_MEAN_ABS, e


def test_cdf_video480p_full_size():
    wl = WORKLOADS["video480p"]
    out = _run(wl, 0.2, fused=True)
    dense = out["mask"].dense()
    check_csr(out["mask"], out["mask"].sizes.sink_first)
    excluded, compared = compare_cdf_masks(dense, bits(out["qp"]), bits(out["kp"]), 0.2, wl.frames, wl.height,
                                           wl.width, wl.sink, wl.text_tokens)
    print(f"video480p cdf: mask compared exactly on {compared} blocks, {excluded} in the boundary band")
    assert excluded <= 0.01 * compared
    rc = out["mask"].row_count.cpu().numpy()
    assert rc.min() < rc.max()                       # adaptive row lengths
    Tb, s0 = wl.num_blocks, out["mask"].sizes.sink_first
    items = full_size_items(wl.heads, Tb, s0, seed=2)
    e = attention_errors(out["op"], bits(out["qp"]), bits(out["kp"]), bits(out["vp"]), dense, items=items)
    print(f"video480p cdf: attention compared on {len(items)} query blocks, max-abs {e['max_abs']:.3g}, "
          f"mean-abs {e['mean_abs']:.3g}")
    assert e["max_abs"] <= ATTN_MAX_ABS and e["mean_abs"] <= ATTN_MEAN_ABS, e


def test_cdf_fused_equals_unfused_and_deterministic():
    wl = WORKLOADS["video720p"]
    a = _run(wl, 0.2, fused=True)
    b = _run(wl, 0.2, fused=False)
    assert torch.equal(a["mask"].row_count, b["mask"].row_count)
    assert np.array_equal(a["mask"].dense(), b["mask"].dense())
    c = _run(wl, 0.2, fused=True)
    assert torch.equal(a["mask"].row_count, c["mask"].row_count)
    assert torch.equal(a["op"].view(torch.int16), c["op"].view(torch.int16))
