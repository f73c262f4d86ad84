"""GPU parity: the CUDA path, called through the C ABI, against the oracle on
the same seeded inputs.

- permutation and unpermutation: bit exact;
- block mask: bit exact outside the 1e-5 tie band around each row's threshold;
- attention output under the GPU's mask: max-abs <= 2e-2, mean-abs <= 2e-3.
Sizes span several tiles with ragged tails; the video workloads at full size
are compared in full for the permutation and the mask, and on sampled query
blocks for the attention output.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from image_dits_b200 import build as rf2_build
from image_dits_b200 import rf2
from image_dits_b200.workload import WORKLOADS, Workload, make_qkv
from parity import (ATTN_MAX_ABS, ATTN_MEAN_ABS, attention_errors, bits, check_csr, compare_masks,
                    full_size_items, run_path)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    rf2_build.build()
    rf2.lib()
    yield
    torch.cuda.synchronize()


def _perm_of(wl):
    return oracle.permutation(wl.frames, wl.height, wl.width, wl.win_t, wl.win_h, wl.win_w, wl.sink, wl.text_tokens)


def _small_cases():
    """(name, Workload) small geometries: ragged tails, odd block counts, N < 64,
    single frame with sink, windows larger than the grid, d = 64 and 128."""
    W = Workload
    return [
        ("tiny", WORKLOADS["tiny"]),
        ("ragged_d128", W("r1", 1, 3, 128, 3, 7, 9, 2, 4, 4, 0.3, True, (44, 42, 42))),
        ("ragged_d64_nosink", W("r2", 2, 1, 64, 2, 13, 11, 2, 3, 5, 0.5, False, (24, 20, 20))),
        ("one_block", W("r3", 1, 2, 64, 1, 5, 7, 1, 2, 2, 0.5, True, (0, 32, 32))),
        ("single_frame_sink", W("r4", 1, 2, 128, 1, 16, 20, 1, 8, 8, 0.25, True, (0, 64, 64))),
        ("big_window", W("r5", 1, 1, 128, 5, 9, 10, 8, 16, 16, 0.2, True, (44, 42, 42))),
        ("keep_one", W("r6", 1, 2, 128, 3, 16, 16, 1, 8, 8, 0.01, True, (44, 42, 42))),
        ("keep_all", W("r7", 1, 2, 64, 2, 12, 16, 2, 4, 4, 1.0, True, (24, 20, 20))),
        ("odd_blocks", W("r8", 1, 2, 128, 1, 24, 40, 1, 8, 8, 0.4, False, (0, 64, 64))),
        # text tokens of a joint video-text attention (section 3.4)
        ("text_sink", W("t1", 1, 2, 128, 3, 8, 8, 1, 8, 8, 0.3, True, (44, 42, 42), 77)),
        ("text_nosink", W("t2", 1, 2, 64, 2, 8, 8, 2, 4, 4, 0.4, False, (24, 20, 20), 70)),
        ("image_text", W("t3", 1, 2, 128, 1, 16, 16, 1, 8, 8, 0.3, False, (0, 64, 64), 100)),
    ]


@pytest.mark.parametrize("name,wl", _small_cases())
def test_small_case_parity(name, wl):
    q, k, v = make_qkv(wl, "cuda", seed=7)
    g = rf2.geometry_of(wl)
    out = run_path(g, q, k, v, wl.keep, lse=True)
    perm = _perm_of(wl)
    # permutation: bit exact, and unpermute(permute(x)) == x
    assert np.array_equal(bits(out["qp"]), oracle.permute(bits(q), perm))
    assert np.array_equal(bits(out["vp"]), oracle.permute(bits(v), perm))
    assert torch.equal(rf2.unpermute(g, out["qp"]).view(torch.int16), q.view(torch.int16))
    # mask
    sz = out["mask"].sizes
    check_csr(out["mask"], sz.sink_first)
    dense = out["mask"].dense()
    compare_masks(dense, bits(out["qp"]), bits(out["kp"]), wl.keep, wl.frames, wl.height, wl.width, wl.sink,
                  wl.text_tokens)
    # attention under the GPU's mask, and the unpermuted output
    e = attention_errors(out["op"], bits(out["qp"]), bits(out["kp"]), bits(out["vp"]), dense, lse=out["lse"])
    assert e["max_abs"] <= ATTN_MAX_ABS and e["mean_abs"] <= ATTN_MEAN_ABS, e
    assert e["lse_max_abs"] <= 1e-3, e
    assert np.array_equal(bits(out["o"]), oracle.unpermute(bits(out["op"]), perm))


@pytest.mark.parametrize("name", ["image", "qwen_image"])
def test_image_parity(name):
    wl = WORKLOADS[name]
    q, k, v = make_qkv(wl, "cuda", seed=0)
    g = rf2.geometry_of(wl)
    out = run_path(g, q, k, v, wl.keep)
    perm = _perm_of(wl)
    assert np.array_equal(bits(out["kp"]), oracle.permute(bits(k), perm))
    check_csr(out["mask"], -1)
    dense = out["mask"].dense()
    compare_masks(dense, bits(out["qp"]), bits(out["kp"]), wl.keep, 1, wl.height, wl.width, False,
                  wl.text_tokens)
    Tb = wl.num_blocks
    items = [(bh, i) for bh in (0, 11, 23) for i in range(Tb)]
    e = attention_errors(out["op"], bits(out["qp"]), bits(out["kp"]), bits(out["vp"]), dense, items=items)
    assert e["max_abs"] <= ATTN_MAX_ABS and e["mean_abs"] <= ATTN_MEAN_ABS, e


@pytest.mark.parametrize("d,T,H,W", [(128, 3, 16, 24), (64, 2, 20, 21), (128, 1, 64, 64)])
def test_pooled_scores_precision(d, T, H, W):
    """The tensor-core pooled scores (tf32 hi/lo products) agree with the fp64
    oracle's S^ to well inside the 1e-5 band.  The CDF-threshold path leaves
    them in the mask workspace (the top-n path never writes them out; it
    uses the same three products)."""
    rope = (0, d // 2, d // 2) if T == 1 else ((24, 20, 20) if d == 64 else (44, 42, 42))
    wl = Workload("scores", 1, 3, d, T, H, W, 1, 8, 8, 0.3, T > 1, rope)
    q, k, _ = make_qkv(wl, "cuda", seed=17)
    g = rf2.geometry_of(wl)
    qp, kp = rf2.permute(g, q), rf2.permute(g, k)
    mask, ws = rf2.alloc_mask(g, 1.0, qp.device)
    rf2.predict_mask_cdf(g, qp, kp, 0.5, mask, ws)
    torch.cuda.synchronize()
    Tb = wl.num_blocks
    means_bytes = (2 * wl.heads * Tb * d * 4 + 255) // 256 * 256
    ld = (Tb + 3) // 4 * 4
    S_gpu = ws[2 * means_bytes:2 * means_bytes + wl.heads * Tb * ld * 4].view(torch.float32).view(wl.heads, Tb, ld)[..., :Tb]
    S_ref = oracle.pooled_scores(oracle.block_means(bits(qp)), oracle.block_means(bits(kp)))[0]
    err = np.abs(S_gpu.double().cpu().numpy() - S_ref)
    assert err.max() <= 2e-6 * max(1.0, np.abs(S_ref).max()), (err.max(), np.abs(S_ref).max())


def test_keep_all_equals_dense_attention():
    """keep = 1 selects every block: the output is dense softmax attention, and
    unpermuting it gives dense attention in the model's order."""
    wl = Workload("dense", 1, 2, 128, 2, 10, 13, 2, 4, 4, 1.0, False, (44, 42, 42))
    q, k, v = make_qkv(wl, "cuda", seed=3)
    g = rf2.geometry_of(wl)
    out = run_path(g, q, k, v, 1.0)
    assert out["mask"].kept_pairs() == wl.heads * wl.num_blocks ** 2
    ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double())
    err = (out["o"].double() - ref).abs()
    assert err.max().item() <= ATTN_MAX_ABS and err.mean().item() <= ATTN_MEAN_ABS


def test_constant_value_rows():
    """With V constant along the sequence every output row equals that row."""
    wl = Workload("const", 1, 2, 128, 3, 9, 11, 2, 4, 4, 0.3, True, (44, 42, 42))
    q, k, v = make_qkv(wl, "cuda", seed=5)
    v = v[:, :, :1, :].expand_as(v).contiguous()
    out = run_path(rf2.geometry_of(wl), q, k, v, wl.keep)
    err = (out["o"].float() - v.float()).abs().max().item()
    assert err <= 2 ** -7 * v.float().abs().max().item() + 1e-6


@pytest.mark.parametrize("d,keep,step", [(128, 1.0, 30.0), (128, 0.5, 30.0), (64, 0.4, 30.0), (128, 0.5, 9.0)])
def test_running_max_rescale(d, keep, step):
    """Key blocks in four groups whose scores step up by `step` (log2 units)
    from one group to the next, and query rows alternating in sign.  With
    steps of 30 an entry's probabilities under the old running max sum past
    2^24 at a group boundary: those rows take the entry's max, raise their
    running max and rescale O, while the other rows of the same warp keep
    their first max; with steps of 9 the probabilities are used under the
    stale max (up to 2^9 each).  Under a sparse mask (chosen on the
    unmodified scores) the steps fall at different entries for the two query
    blocks of a tile."""
    rope = (44, 42, 42) if d == 128 else (24, 20, 20)
    wl = Workload("rescale", 1, 2, d, 4, 16, 16, 2, 4, 4, keep, False, rope)
    g = rf2.geometry_of(wl)
    q, k, v = make_qkv(wl, "cuda", seed=11)
    qp, kp, vp = rf2.permute(g, q), rf2.permute(g, k), rf2.permute(g, v)
    mask = rf2.predict_mask(g, qp, kp, keep)
    N, Tb = wl.num_tokens, wl.num_blocks
    sl2 = math.log2(math.e) / math.sqrt(d)
    A = 16.0
    sign = torch.where(torch.arange(N, device="cuda") % 2 == 0, 1.0, -1.0)
    qp[..., 0] = (A * sign).to(qp.dtype)
    group = (torch.arange(N, device="cuda") // 64) * 4 // Tb
    kp[..., 0] = (step * group / (sl2 * A)).to(kp.dtype)
    lse = torch.full((wl.heads * N,), float("nan"), device="cuda")
    op = rf2.block_sparse_attn(g, qp, kp, vp, mask, lse=lse)
    torch.cuda.synchronize()
    assert rf2.device_status() == rf2.RF2_OK
    e = attention_errors(op, bits(qp), bits(kp), bits(vp), mask.dense(), lse=lse)
    assert e["max_abs"] <= ATTN_MAX_ABS and e["mean_abs"] <= ATTN_MEAN_ABS, e
    assert e["lse_max_abs"] <= 1e-3, e


@pytest.mark.parametrize("name", ["tiny", "ragged_d128", "ragged_d64_nosink", "one_block", "single_frame_sink",
                                  "odd_blocks", "text_nosink", "video720p"])
def test_fused_permute_pool_matches_unfused(name):
    """rf2_permute_qk_pool writes the same Qp/Kp as rf2_permute and the same
    block means as the mask path's own pooling, bit for bit, so the predicted
    masks are identical."""
    wl = WORKLOADS[name] if name in WORKLOADS else dict(_small_cases())[name]
    q, k, _ = make_qkv(wl, "cuda", seed=9)
    g = rf2.geometry_of(wl)
    mask_a, ws_a = rf2.alloc_mask(g, wl.keep, q.device)
    qp_a, kp_a = rf2.permute_qk_pool(g, q, k, ws_a)
    rf2.predict_mask_pooled(g, wl.keep, mask_a, ws_a)
    qp_b, kp_b = rf2.permute(g, q), rf2.permute(g, k)
    mask_b, ws_b = rf2.alloc_mask(g, wl.keep, q.device)
    rf2.predict_mask(g, qp_b, kp_b, wl.keep, mask_b, ws_b)
    torch.cuda.synchronize()
    assert rf2.device_status() == rf2.RF2_OK
    assert torch.equal(qp_a.view(torch.int16), qp_b.view(torch.int16))
    assert torch.equal(kp_a.view(torch.int16), kp_b.view(torch.int16))
    Tb = wl.num_blocks
    means_bytes = (2 * wl.batch * wl.heads * Tb * wl.head_dim * 4 + 255) // 256 * 256
    assert torch.equal(ws_a[:2 * means_bytes], ws_b[:2 * means_bytes])
    assert torch.equal(mask_a.row_count, mask_b.row_count)
    assert torch.equal(mask_a.row_start, mask_b.row_start)
    assert np.array_equal(mask_a.dense(), mask_b.dense())
    if name != "video720p":
        perm = _perm_of(wl)
        assert np.array_equal(bits(kp_a), oracle.permute(bits(k), perm))
        hi = ws_a[:means_bytes].view(torch.float32)[:2 * wl.batch * wl.heads * Tb * wl.head_dim]
        lo = ws_a[means_bytes:2 * means_bytes].view(torch.float32)[:hi.numel()]
        m = (hi.double() + lo.double()).view(2, wl.batch * wl.heads, Tb, wl.head_dim).cpu().numpy()
        m_ref = oracle.block_means(bits(kp_a).reshape(wl.batch * wl.heads, -1, wl.head_dim))
        # fp32 sums of bf16 rows over at most 64 rows: relative 64 * 2^-24.
        assert np.abs(m[1] - m_ref).max() <= 4e-6 * max(1.0, np.abs(m_ref).max())


def test_deterministic():
    wl = WORKLOADS["tiny"]
    q, k, v = make_qkv(wl, "cuda", seed=11)
    g = rf2.geometry_of(wl)
    a = run_path(g, q, k, v, wl.keep)
    b = run_path(g, q, k, v, wl.keep)
    assert torch.equal(a["mask"].row_count, b["mask"].row_count)
    assert np.array_equal(a["mask"].dense(), b["mask"].dense())
    assert torch.equal(a["o"].view(torch.int16), b["o"].view(torch.int16))


def test_random_geometries():
    rng = np.random.default_rng(21)
    for it in range(12):
        T, H, W = int(rng.integers(1, 4)), int(rng.integers(2, 20)), int(rng.integers(2, 20))
        d = int(rng.choice([64, 128]))
        rope = (0, d // 2, d // 2) if T == 1 else ((24, 20, 20) if d == 64 else (44, 42, 42))
        wl = Workload(f"rand{it}", 1, int(rng.integers(1, 3)), d, T, H, W, int(rng.integers(1, 4)),
                      int(rng.integers(1, 9)), int(rng.integers(1, 9)), float(rng.choice([0.1, 0.3, 0.5, 0.8])),
                      bool(rng.integers(0, 2)), rope)
        q, k, v = make_qkv(wl, "cuda", seed=it)
        g = rf2.geometry_of(wl)
        out = run_path(g, q, k, v, wl.keep)
        assert np.array_equal(bits(out["qp"]), oracle.permute(bits(q), _perm_of(wl))), wl
        dense = out["mask"].dense()
        check_csr(out["mask"], out["mask"].sizes.sink_first)
        compare_masks(dense, bits(out["qp"]), bits(out["kp"]), wl.keep, T, H, W, wl.sink, wl.text_tokens)
        e = attention_errors(out["op"], bits(out["qp"]), bits(out["kp"]), bits(out["vp"]), dense)
        assert e["max_abs"] <= ATTN_MAX_ABS and e["mean_abs"] <= ATTN_MEAN_ABS, (wl, e)


@pytest.mark.parametrize("keep,sink", [(0.02, True), (0.2, False), (0.6, True), (0.97, False)])
def test_long_rows_selection(keep, sink):
    """Rows of more than 512 key blocks take the shared-memory selection (a
    stratified sample brackets the n-th largest score, a radix select ranks
    the bracketed keys, the whole row where the bracket misses): masks match
    the oracle at small and large keep ratios (the bracket clamped at either
    end of the sample), with and without the first-frame sink."""
    wl = Workload("long", 1, 2, 64, 4, 64, 144, 2, 8, 8, keep, sink, (24, 20, 20))
    assert wl.num_blocks > 512
    q, k, v = make_qkv(wl, "cuda", seed=31)
    g = rf2.geometry_of(wl)
    qp, kp = rf2.permute(g, q), rf2.permute(g, k)
    mask = rf2.predict_mask(g, qp, kp, keep)
    torch.cuda.synchronize()
    assert rf2.device_status() == rf2.RF2_OK
    check_csr(mask, mask.sizes.sink_first)
    compare_masks(mask.dense(), bits(qp), bits(kp), keep, wl.frames, wl.height, wl.width, sink)


@pytest.mark.parametrize("name,wl", _small_cases() + [("image", WORKLOADS["image"]),
                                                      ("long_rows", Workload("long", 1, 2, 128, 4, 64, 144, 2, 8, 8,
                                                                             0.2, True, (44, 42, 42))),
                                                      ("long_rows_keep_all", Workload("long", 1, 2, 128, 4, 64, 144, 2,
                                                                                      8, 8, 1.0, False, (44, 42, 42)))])
def test_mask_from_codes(name, wl, monkeypatch):
    """The selection from 16-bit score codes (the path of large calls), forced
    on small ones: the masks match the oracle outside the tie band, and the
    score-matrix selection on the same inputs (equal outside the band too)."""
    q, k, v = make_qkv(wl, "cuda", seed=11)
    g = rf2.geometry_of(wl)
    qp, kp = rf2.permute(g, q), rf2.permute(g, k)
    monkeypatch.setenv("RF2_MASK_SELECT", "codes")
    mask = rf2.predict_mask(g, qp, kp, wl.keep)
    torch.cuda.synchronize()
    assert rf2.device_status() == rf2.RF2_OK
    check_csr(mask, mask.sizes.sink_first)
    dense = mask.dense()
    compare_masks(dense, bits(qp), bits(kp), wl.keep, wl.frames, wl.height, wl.width, wl.sink, wl.text_tokens)
    monkeypatch.setenv("RF2_MASK_SELECT", "scores")
    ref = rf2.predict_mask(g, qp, kp, wl.keep).dense()
    differ = int((dense != ref).sum())
    assert differ <= max(4, 1e-4 * dense.size), differ


def _full_size(name):
    wl = WORKLOADS[name]
    q, k, v = make_qkv(wl, "cuda", seed=0)
    g = rf2.geometry_of(wl)
    out = run_path(g, q, k, v, wl.keep)
    perm = _perm_of(wl)
    qp_b, kp_b, vp_b = bits(out["qp"]), bits(out["kp"]), bits(out["vp"])
    assert np.array_equal(qp_b, oracle.permute(bits(q), perm))
    assert np.array_equal(vp_b, oracle.permute(bits(v), perm))
    del q, k, v
    sz = out["mask"].sizes
    dense = out["mask"].dense()
    excluded, compared = compare_masks(dense, qp_b, kp_b, wl.keep, wl.frames, wl.height, wl.width, wl.sink,
                                       wl.text_tokens)
    # Blocks inside the tie band are excluded from the exact comparison; on
    # these inputs they are a fraction of a percent (pooled scores cluster).
    print(f"{name}: mask compared exactly on {compared} blocks, {excluded} in the 1e-5 tie band")
    assert excluded <= 1e-2 * compared
    Tb = sz.num_blocks
    items = full_size_items(wl.heads, Tb, sz.sink_first)
    n_sink = sum(1 for _, i in items if sz.sink_first >= 0 and i >= sz.sink_first)
    e = attention_errors(out["op"], qp_b, kp_b, vp_b, dense, items=items)
    print(f"{name}: attention compared on {len(items)} query blocks ({n_sink} sink rows), "
          f"{e['n']} values: max-abs {e['max_abs']:.3g}, mean-abs {e['mean_abs']:.3g}")
    assert e["max_abs"] <= ATTN_MAX_ABS and e["mean_abs"] <= ATTN_MEAN_ABS, e
    assert np.array_equal(bits(out["o"][:, :2]), oracle.unpermute(bits(out["op"][:, :2]), perm))


def test_video480p_full_size():
    _full_size("video480p")


def test_video480p_text_full_size():
    _full_size("video480p_text")


def test_video720p_full_size():
    _full_size("video720p")


def test_device_status_clean():
    assert rf2.device_status() == rf2.RF2_OK


@pytest.mark.parametrize("chunk_events", [True, False])
def test_host_call_back_to_back(chunk_events):
    """rf2_attention_host called twice in a row on different inputs without a
    synchronization between: the second call's copies wait for the first
    call's computation (chunk by chunk with the caller's events, else as a
    whole), so both outputs equal their device-path results."""
    wl = WORKLOADS["video480p"]
    g = rf2.geometry_of(wl)
    refs, hosts = [], []
    for seed in (8, 9):
        q, k, v = make_qkv(wl, "cuda", seed=seed)
        ref, _ = rf2.rainfusion_attention(g, q, k, v, wl.keep)
        refs.append(ref.cpu())
        hosts.append(tuple(x.cpu().pin_memory() for x in (q, k, v)) + (torch.empty_like(q, device="cpu").pin_memory(),))
    torch.cuda.synchronize()
    pipe = rf2.HostPipeline(g, keep=wl.keep, chunks=4, chunk_events=chunk_events)
    for hq, hk, hv, ho in hosts:
        pipe.run(hq, hk, hv, ho)
    pipe.synchronize()
    for (hq, hk, hv, ho), ref in zip(hosts, refs):
        assert torch.equal(ho.view(torch.int16), ref.view(torch.int16))
    assert rf2.device_status() == rf2.RF2_OK


@pytest.mark.parametrize("name,chunks,tau", [("tiny", 2, None), ("image", 5, None), ("video480p_text", 4, None),
                                             ("video480p", 3, 0.2)])
def test_host_pipeline_matches_device_path(name, chunks, tau):
    """rf2_attention_host through HostPipeline (head chunks, copies overlapped
    with compute) gives the same output bits as the single device call, over
    two runs."""
    wl = WORKLOADS[name]
    q, k, v = make_qkv(wl, "cuda", seed=4)
    g = rf2.geometry_of(wl)
    if tau is None:
        ref, _ = rf2.rainfusion_attention(g, q, k, v, wl.keep)
    else:
        mask, ws = rf2.alloc_mask(g, 1.0, q.device)
        qp, kp = rf2.permute_qk_pool(g, q, k, ws)
        rf2.predict_mask_cdf_pooled(g, tau, mask, ws)
        ref = rf2.unpermute(g, rf2.block_sparse_attn(g, qp, kp, rf2.permute(g, v), mask))
    torch.cuda.synchronize()
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    ho = torch.empty_like(hq).pin_memory()
    pipe = rf2.HostPipeline(g, keep=None if tau is not None else wl.keep, tau=tau, chunks=chunks)
    for _ in range(2):
        ho.zero_()
        pipe.run(hq, hk, hv, ho)
        pipe.synchronize()
        assert torch.equal(ho.view(torch.int16), ref.cpu().view(torch.int16))
    assert rf2.device_status() == rf2.RF2_OK
