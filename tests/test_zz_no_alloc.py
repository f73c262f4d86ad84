"""rf2_predict_mask_static: the allocation-free variant of rf2_predict_mask.

Some callers cannot allocate device memory themselves (a host framework that
owns the allocator and offers no workspace, or a latency-critical loop where
cudaMalloc's implicit synchronization is not acceptable).  For them the
library keeps a fixed 64 MiB scratch array of its own.  These tests call the
variant through the C ABI and check that, on two calls in a row with
different problems, its block mask is identical to the one rf2_predict_mask
writes with a caller-supplied workspace and the same selection (the static
variant always selects from the score matrix, so the reference call is made
with RF2_MASK_SELECT=scores; masks are compared exactly), and that a problem
needing more scratch than the array holds is refused before anything is
launched.

Kept in a file of its own that pytest collects last.
"""
import ctypes

import pytest
import torch

from image_dits_b200 import build as rf2_build
from image_dits_b200 import rf2
from image_dits_b200.workload import WORKLOADS, Workload, make_qkv

pytestmark = pytest.mark.gpu


def _static_mask(g, qp, kp, keep):
    sz = rf2.query(g, keep)
    dev = qp.device
    m = rf2.BlockMask(torch.full((sz.num_rows,), -1, dtype=torch.int32, device=dev),
                      torch.full((sz.num_rows,), -1, dtype=torch.int32, device=dev),
                      torch.full((max(1, sz.col_idx_capacity),), -1, dtype=torch.int32, device=dev), sz)
    st = rf2.lib().rf2_predict_mask_static(ctypes.byref(g), qp.data_ptr(), kp.data_ptr(), float(keep),
                                           m.row_start.data_ptr(), m.row_count.data_ptr(), m.col_idx.data_ptr(),
                                           torch.cuda.current_stream().cuda_stream)
    assert st == rf2.RF2_OK, rf2.status_string(st)
    return m


def _same(a: rf2.BlockMask, b: rf2.BlockMask):
    assert torch.equal(a.row_start, b.row_start)
    assert torch.equal(a.row_count, b.row_count)
    ra, rb = a.dense(), b.dense()
    assert (ra == rb).all()


@pytest.fixture(autouse=True)
def _score_matrix_selection(monkeypatch):
    monkeypatch.setenv("RF2_MASK_SELECT", "scores")


def test_static_scratch_matches_workspace_variant():
    rf2_build.build()
    cases = [WORKLOADS["video480p"], WORKLOADS["tiny"],
             Workload("ragged", 2, 3, 128, 3, 7, 9, 2, 4, 4, 0.3, True, (44, 42, 42))]
    for call, wl in enumerate(cases):        # several calls in a row, different sizes
        q, k, _ = make_qkv(wl, "cuda", seed=call)
        g = rf2.geometry_of(wl)
        qp, kp = rf2.permute(g, q), rf2.permute(g, k)
        ref = rf2.predict_mask(g, qp, kp, wl.keep)
        got = _static_mask(g, qp, kp, wl.keep)
        torch.cuda.synchronize()
        assert rf2.device_status() == rf2.RF2_OK
        _same(got, ref)


def test_static_scratch_largest_720p_problem():
    """At 720p (75,600 tokens, d = 128) the scratch holds the block means of
    25 heads (2 x 30.3 MB as a hi/lo pair) plus one head's pooled scores
    (5.6 MB): 25 heads, the documented limit, run and match rf2_predict_mask
    exactly."""
    rf2_build.build()
    import dataclasses
    wl = dataclasses.replace(WORKLOADS["video720p"], heads=25)
    q, k, _ = make_qkv(wl, "cuda", seed=3)
    g = rf2.geometry_of(wl)
    qp, kp = rf2.permute(g, q), rf2.permute(g, k)
    del q, k
    ref = rf2.predict_mask(g, qp, kp, wl.keep)
    for _ in range(2):
        got = _static_mask(g, qp, kp, wl.keep)
        torch.cuda.synchronize()
        assert rf2.device_status() == rf2.RF2_OK
        _same(got, ref)


def test_static_scratch_refuses_oversize():
    """Problems whose block means and one head's scores exceed the 64 MiB
    array are refused before anything is launched: 26 heads at 720p (2 x
    31.5 MB of means + 5.6 MB of scores) and 2 x 40 heads (2 x 96.8 MB of
    means)."""
    rf2_build.build()
    import dataclasses
    fake = ctypes.c_void_p(0x10000)            # never touched: the size check comes first
    for g in (rf2.geometry_of(dataclasses.replace(WORKLOADS["video720p"], heads=26)),
              rf2.geometry_of(WORKLOADS["video720p"], batch=2)):
        st = rf2.lib().rf2_predict_mask_static(ctypes.byref(g), fake, fake, 0.2, fake, fake, fake, None)
        assert st == rf2.RF2_ERR_INSUFFICIENT_WORKSPACE
