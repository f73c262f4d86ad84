"""C-ABI checks that need no GPU: the library loads, exports every entry point
that include/rf2.h declares, computes the documented sizes, rejects invalid
calls on the host before any launch, and its host permutation table (the same
closed form the kernels use) equals the oracle's sort-based definition."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from image_dits_b200 import build as rf2_build
from image_dits_b200 import rf2
from image_dits_b200.workload import WORKLOADS, random_grid_case

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    rf2_build.build()
    return rf2.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "rf2.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rf2_[a-z_]+)\s*\(", src)))


def test_exports_match_header(L):
    declared = _declared()
    assert declared == sorted(rf2.EXPORTED)
    for name in declared:
        assert hasattr(L, name), name


def test_status_strings(L):
    for s in range(6):
        assert rf2.status_string(s)
    assert rf2.status_string(99) == "unknown status"


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_query_matches_oracle_readings(L, name):
    wl = WORKLOADS[name]
    sz = rf2.query(rf2.geometry_of(wl), wl.keep)
    N = wl.num_tokens
    assert sz.num_tokens == N
    assert sz.num_blocks == oracle.num_blocks(N)
    assert sz.n_keep == oracle.keep_count(wl.keep, sz.num_blocks)
    assert sz.sink_first == oracle.sink_start(wl.frames, wl.height, wl.width, wl.sink, wl.text_tokens)
    Tb = sz.num_blocks
    n_sink = 0 if sz.sink_first < 0 else Tb - sz.sink_first
    assert sz.row_capacity == min(Tb, sz.n_keep + n_sink)
    BH = wl.batch * wl.heads
    assert sz.num_rows == BH * Tb
    s0 = Tb if sz.sink_first < 0 else sz.sink_first
    assert sz.col_idx_capacity == BH * (s0 * sz.row_capacity + (Tb - s0) * Tb)
    r256 = lambda b: (b + 255) // 256 * 256
    means = r256(2 * BH * Tb * wl.head_dim * 4)
    scores_per_head = Tb * ((Tb + 3) // 4 * 4) * 4
    score_group = min(BH, max(1, (96 << 20) // scores_per_head)) * scores_per_head
    items = BH * ((Tb + 127) // 128)          # (head, 128 query blocks)
    # coarse and fine code bytes, histograms, code widths, overflow list
    codes = (2 * r256(items * ((Tb + 31) // 32) * 128 * 8 * 4) + r256(items * 2 * 16 * 128 * 4)
             + r256(items * 128 * 4) + r256(4 * (BH * Tb + 1)))
    assert sz.mask_workspace_bytes == 2 * means + max(score_group, codes)


def test_keep_ratio_matches_oracle(L):
    g = rf2.make_geometry(1, 1, 128, 21, 45, 80, 4, 4, 4, True)
    for keep in (1.0, 0.5, 0.2, 0.1, 0.05, 0.3333, 1e-6, 0.9999):
        assert rf2.query(g, keep).n_keep == oracle.keep_count(keep, 1182)


def test_permutation_index_matches_oracle(L):
    rng = np.random.default_rng(0)
    cases = [random_grid_case(rng) for _ in range(250)]
    cases += [(21, 45, 80, 4, 4, 4, True), (21, 30, 52, 4, 4, 4, True), (1, 64, 64, 1, 8, 8, False),
              (4, 16, 16, 1, 8, 8, True), (5, 7, 9, 8, 9, 10, True)]
    for (T, H, W, wt, wh, ww, sink) in cases:
        g = rf2.make_geometry(1, 1, 64, T, H, W, wt, wh, ww, sink)
        assert np.array_equal(rf2.permutation_index(g), oracle.permutation(T, H, W, wt, wh, ww, sink)), \
            (T, H, W, wt, wh, ww, sink)


def test_permutation_index_with_text_matches_oracle(L):
    rng = np.random.default_rng(3)
    cases = [(21, 30, 52, 4, 4, 4, True, 256), (1, 64, 64, 1, 8, 8, False, 512), (4, 16, 16, 1, 8, 8, True, 77)]
    for _ in range(60):
        T, H, W, wt, wh, ww, sink = random_grid_case(rng)
        cases.append((T, H, W, wt, wh, ww, sink, int(rng.integers(0, 200))))
    for (T, H, W, wt, wh, ww, sink, text) in cases:
        g = rf2.make_geometry(1, 1, 64, T, H, W, wt, wh, ww, sink, text=text)
        assert np.array_equal(rf2.permutation_index(g), oracle.permutation(T, H, W, wt, wh, ww, sink, text)), \
            (T, H, W, wt, wh, ww, sink, text)
        sz = rf2.query(g, 0.3)
        assert sz.num_tokens == T * H * W + text
        assert sz.sink_first == oracle.sink_start(T, H, W, sink, text)


def _status(fn, *args):
    return fn(*args)


def test_host_validation(L):
    good = rf2.make_geometry(1, 2, 64, 4, 16, 16, 1, 8, 8, True)
    fake = ctypes.c_void_p(0x10000)            # aligned, never dereferenced: validation fails first
    G = ctypes.byref
    bad_dim = rf2.make_geometry(1, 2, 96, 4, 16, 16, 1, 8, 8, True)
    bad_blk = rf2.make_geometry(1, 2, 64, 4, 16, 16, 1, 8, 8, True, block=32)
    bad_win = rf2.make_geometry(1, 2, 64, 4, 16, 16, 0, 8, 8, True)
    bad_sink = rf2.make_geometry(1, 2, 64, 4, 16, 16, 1, 8, 8, True)
    bad_sink.first_frame_sink = 2
    bad_text = rf2.make_geometry(1, 2, 64, 4, 16, 16, 1, 8, 8, True, text=-1)
    huge = rf2.make_geometry(1, 1, 64, 100, 64, 64, 1, 8, 8, False)    # T_b > 4096
    sz = rf2.Sizes()
    assert L.rf2_query(G(good), 0.5, G(sz)) == rf2.RF2_OK
    assert L.rf2_query(G(good), 0.0, G(sz)) == rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_query(G(good), 1.5, G(sz)) == rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_query(G(good), float("nan"), G(sz)) == rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_query(None, 0.5, G(sz)) == rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_query(G(good), 0.5, None) == rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_query(G(bad_dim), 0.5, G(sz)) == rf2.RF2_ERR_UNSUPPORTED
    assert L.rf2_query(G(bad_blk), 0.5, G(sz)) == rf2.RF2_ERR_UNSUPPORTED
    assert L.rf2_query(G(huge), 0.5, G(sz)) == rf2.RF2_ERR_UNSUPPORTED
    assert L.rf2_query(G(bad_win), 0.5, G(sz)) == rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_query(G(bad_sink), 0.5, G(sz)) == rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_query(G(bad_text), 0.5, G(sz)) == rf2.RF2_ERR_INVALID_ARGUMENT
    # permute / unpermute
    for fn in (L.rf2_permute, L.rf2_unpermute):
        assert fn(G(good), None, fake, None) == rf2.RF2_ERR_INVALID_ARGUMENT
        assert fn(G(good), fake, None, None) == rf2.RF2_ERR_INVALID_ARGUMENT
        assert fn(G(good), ctypes.c_void_p(0x10008), ctypes.c_void_p(0x20000), None) == rf2.RF2_ERR_INVALID_ARGUMENT
        assert fn(G(good), fake, fake, None) == rf2.RF2_ERR_INVALID_ARGUMENT      # in place
        assert fn(G(bad_dim), fake, ctypes.c_void_p(0x20000), None) == rf2.RF2_ERR_UNSUPPORTED
    # predict_mask
    L.rf2_query(G(good), 0.5, G(sz))
    ws_small = sz.mask_workspace_bytes - 1
    assert L.rf2_predict_mask(G(good), fake, fake, 0.5, fake, fake, fake, fake, ws_small, None) == \
        rf2.RF2_ERR_INSUFFICIENT_WORKSPACE
    assert L.rf2_predict_mask(G(good), fake, fake, 0.0, fake, fake, fake, fake, 1 << 30, None) == \
        rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_predict_mask(G(good), None, fake, 0.5, fake, fake, fake, fake, 1 << 30, None) == \
        rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_predict_mask(G(good), fake, fake, 0.5, fake, fake, fake, ctypes.c_void_p(0x10004), 1 << 30,
                              None) == rf2.RF2_ERR_INVALID_ARGUMENT
    # permute_qk_pool / predict_mask_pooled
    f2, f3 = ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000)
    f4 = ctypes.c_void_p(0x40000)
    big = 1 << 30
    assert L.rf2_permute_qk_pool(G(good), fake, f2, f3, f4, ctypes.c_void_p(0x50000), ws_small, None) == \
        rf2.RF2_ERR_INSUFFICIENT_WORKSPACE
    assert L.rf2_permute_qk_pool(G(good), None, f2, f3, f4, fake, big, None) == rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_permute_qk_pool(G(good), fake, f2, fake, f4, ctypes.c_void_p(0x50000), big, None) == \
        rf2.RF2_ERR_INVALID_ARGUMENT                                                  # in place
    assert L.rf2_permute_qk_pool(G(good), fake, f2, f3, ctypes.c_void_p(0x40008), ctypes.c_void_p(0x50000), big,
                                 None) == rf2.RF2_ERR_INVALID_ARGUMENT                # misaligned
    assert L.rf2_permute_qk_pool(G(bad_dim), fake, f2, f3, f4, ctypes.c_void_p(0x50000), big, None) == \
        rf2.RF2_ERR_UNSUPPORTED
    assert L.rf2_predict_mask_pooled(G(good), 0.5, fake, fake, fake, fake, ws_small, None) == \
        rf2.RF2_ERR_INSUFFICIENT_WORKSPACE
    assert L.rf2_predict_mask_pooled(G(good), 0.0, fake, fake, fake, fake, big, None) == \
        rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_predict_mask_pooled(G(good), 0.5, fake, None, fake, fake, big, None) == \
        rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_predict_mask_pooled(G(good), 0.5, fake, fake, fake, None, big, None) == \
        rf2.RF2_ERR_INVALID_ARGUMENT
    # predict_mask_cdf / predict_mask_cdf_pooled: tau in (0, 1], workspace of rf2_query(geom, 1.0)
    for tau in (0.0, -0.5, 1.5, float("nan")):
        assert L.rf2_predict_mask_cdf(G(good), fake, fake, tau, fake, fake, fake, fake, big, None) == \
            rf2.RF2_ERR_INVALID_ARGUMENT
        assert L.rf2_predict_mask_cdf_pooled(G(good), tau, fake, fake, fake, fake, big, None) == \
            rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_predict_mask_cdf(G(good), fake, fake, 0.5, fake, fake, fake, fake, ws_small, None) == \
        rf2.RF2_ERR_INSUFFICIENT_WORKSPACE
    assert L.rf2_predict_mask_cdf(G(good), None, fake, 0.5, fake, fake, fake, fake, big, None) == \
        rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_predict_mask_cdf_pooled(G(good), 0.5, fake, fake, None, fake, big, None) == \
        rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_predict_mask_cdf_pooled(G(bad_dim), 0.5, fake, fake, fake, fake, big, None) == \
        rf2.RF2_ERR_UNSUPPORTED
    # block_sparse_attn
    assert L.rf2_block_sparse_attn(G(good), fake, fake, None, fake, fake, fake, fake, None, None) == \
        rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_block_sparse_attn(G(good), fake, fake, fake, fake, fake, fake, fake, ctypes.c_void_p(0x10002),
                                   None) == rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_block_sparse_attn(G(bad_dim), fake, fake, fake, fake, fake, fake, fake, None, None) == \
        rf2.RF2_ERR_UNSUPPORTED
    assert L.rf2_permutation_index(G(good), None) == rf2.RF2_ERR_INVALID_ARGUMENT


def test_selftest_timeout_argument_validation(L):
    """The timeout self-test rejects a limit outside 1 us .. 1 s before any launch."""
    import ctypes
    n = ctypes.c_int32(0)
    for bad in (0, 1_000_001):
        assert L.rf2_selftest_wait_timeout(ctypes.c_uint32(bad), ctypes.byref(n), None) == rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_selftest_wait_timeout(ctypes.c_uint32(1000), None, None) == rf2.RF2_ERR_INVALID_ARGUMENT


def test_host_pipeline_chunk_sizes():
    """Head chunks of rf2.HostPipeline: every head exactly once, in order; equal
    chunks (within one head) without the tail split; with it the last equal
    chunk is split in shrinking parts that end with a single head."""
    for heads in (1, 2, 3, 7, 12, 24, 40, 97):
        for chunks in (1, 2, 3, 5, 8, 10, 200):
            even = rf2.chunk_sizes(heads, chunks, tail_split=False)
            assert sum(even) == heads and all(s >= 1 for s in even)
            assert max(even) - min(even) <= 1
            assert len(even) == min(chunks, heads)
            split = rf2.chunk_sizes(heads, chunks, tail_split=True)
            assert sum(split) == heads and all(s >= 1 for s in split)
            assert split[:len(even) - 1] == even[:-1]
            tail = split[len(even) - 1:]
            assert sum(tail) == even[-1] and tail[-1] == 1
            assert all(a >= b for a, b in zip(tail, tail[1:]))
    assert rf2.chunk_sizes(40, 8) == [5, 5, 5, 5, 5, 5, 5, 3, 1, 1]


def test_host_call_plan(L):
    """rf2_attention_host_query (host only): the C chunking equals
    rf2.chunk_sizes (cuts at round-half-even of c*heads/chunks, the last chunk
    halved down to one head), and the device scratch is the four whole
    tensors, four chunk tensors of the largest chunk and its mask and mask
    workspace, each rounded up to 256 bytes; bad selections are refused."""
    import dataclasses
    r256 = lambda b: (b + 255) // 256 * 256
    for name, heads, chunks, keep, tau in [("video720p", 40, 8, 0.2, None), ("image", 24, 5, 0.5, None),
                                          ("video480p", 12, 3, None, 0.2), ("tiny", 2, 7, 0.5, None),
                                          ("video480p", 5, 2, 0.2, None)]:
        wl = dataclasses.replace(WORKLOADS[name], heads=heads)
        g = rf2.geometry_of(wl)
        hs = rf2.host_query(g, keep, tau, chunks)
        parts = rf2.chunk_sizes(heads, chunks)
        assert hs.num_chunks == len(parts) and hs.max_chunk_heads == max(parts)
        gm = rf2.geometry_of(dataclasses.replace(wl, heads=max(parts)))
        sz = rf2.query(gm, 1.0 if tau else keep)
        row = wl.num_tokens * wl.head_dim * 2
        want = (4 * r256(heads * row) + 4 * r256(max(parts) * row) + 2 * r256(4 * sz.num_rows)
                + r256(4 * sz.col_idx_capacity) + r256(sz.mask_workspace_bytes))
        assert hs.work_bytes == want, (name, hs.work_bytes, want)
    g = rf2.geometry_of(WORKLOADS["tiny"])
    out = rf2.HostSizes()
    for keep, tau in [(0.0, 0.0), (0.5, 0.5), (0.0, 1.5), (-1.0, 0.0)]:
        assert L.rf2_attention_host_query(ctypes.byref(g), keep, tau, 4, ctypes.byref(out)) == rf2.RF2_ERR_INVALID_ARGUMENT
    assert L.rf2_attention_host_query(ctypes.byref(g), 0.5, 0.0, 4, None) == rf2.RF2_ERR_INVALID_ARGUMENT


def test_static_scratch_size_limit_on_host(L):
    """rf2_predict_mask_static refuses, on the host and before any device call,
    a problem whose block means (hi/lo pair) plus one head's pooled scores
    exceed its 64 MiB array: at 720p that is 26 heads and more (25 fit)."""
    import dataclasses
    fake = ctypes.c_void_p(0x10000)
    for heads, fits in ((25, True), (26, False), (40, False)):
        g = rf2.geometry_of(dataclasses.replace(WORKLOADS["video720p"], heads=heads))
        Tb = 1182
        means = (2 * heads * Tb * 128 * 4 + 255) // 256 * 256
        need = 2 * means + Tb * ((Tb + 3) // 4 * 4) * 4
        assert (need <= 64 << 20) == fits
        if not fits:
            st = L.rf2_predict_mask_static(ctypes.byref(g), fake, fake, 0.2, fake, fake, fake, None)
            assert st == rf2.RF2_ERR_INSUFFICIENT_WORKSPACE


def test_no_fallback_without_the_library_or_a_gpu_tensor(L, tmp_path):
    """The binding has no CPU path: a missing library raises, and host tensors
    given to a device call are refused before anything reaches the library."""
    import torch
    with pytest.raises(RuntimeError):
        rf2.load(str(tmp_path / "librf2.so"))
    g = rf2.geometry_of(WORKLOADS["tiny"])
    wl = WORKLOADS["tiny"]
    x = torch.zeros(wl.batch, wl.heads, wl.num_tokens, wl.head_dim, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        rf2.permute(g, x)
    with pytest.raises(ValueError):
        rf2.unpermute(g, x)
