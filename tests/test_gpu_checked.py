"""The range-checked library, librf2_checked.so (RF2_CHECKED=1): the whole
path through it gives output bit-identical to librf2.so with a clean device
status, and a malformed CSR mask is reported (RF2_ERR_RANGE) and skipped.

The malformed inputs are chosen so that even an unchecked build would stay
inside the buffers: a row_count above T_b on a middle row (clamped to T_b by
the attention kernel) and a col_idx value past T_b (skipped by it); only the
report differs."""
import pytest
import torch

from image_dits_b200 import build as rf2_build
from image_dits_b200 import rf2
from image_dits_b200.workload import WORKLOADS, Workload, make_qkv

pytestmark = pytest.mark.gpu

CASES = [("tiny", WORKLOADS["tiny"]),
         ("ragged_d128", Workload("r1", 1, 3, 128, 3, 7, 9, 2, 4, 4, 0.3, True, (44, 42, 42))),
         ("video480p", WORKLOADS["video480p"])]


@pytest.fixture(scope="module")
def libs():
    rf2_build.build()
    normal = rf2.load(rf2.LIB_PATH)
    checked = rf2.load(rf2.CHECKED_LIB_PATH)
    yield normal, checked
    rf2._lib = normal


def _path(g, wl, q, k, v):
    mask, ws = rf2.alloc_mask(g, wl.keep, q.device)
    qp, kp = rf2.permute_qk_pool(g, q, k, ws)
    rf2.predict_mask_pooled(g, wl.keep, mask, ws)
    vp = rf2.permute(g, v)
    op = rf2.block_sparse_attn(g, qp, kp, vp, mask)
    o = rf2.unpermute(g, op)
    m2 = rf2.predict_mask(g, qp, kp, wl.keep)
    torch.cuda.synchronize()
    return {"qp": qp, "kp": kp, "vp": vp, "row_start": mask.row_start, "row_count": mask.row_count,
            "dense": torch.from_numpy(mask.dense()), "dense_unfused": torch.from_numpy(m2.dense()), "op": op, "o": o}


@pytest.mark.parametrize("name,wl", CASES)
def test_checked_library_matches(libs, name, wl):
    normal, checked = libs
    q, k, v = make_qkv(wl, "cuda", seed=21)
    g = rf2.geometry_of(wl)
    rf2._lib = normal
    a = _path(g, wl, q, k, v)
    assert rf2.device_status() == rf2.RF2_OK
    rf2._lib = checked
    b = _path(g, wl, q, k, v)
    assert rf2.device_status() == rf2.RF2_OK
    rf2._lib = normal
    for key in a:
        x, y = a[key], b[key]
        if x.dtype == torch.bfloat16:
            x, y = x.view(torch.int16), y.view(torch.int16)
        assert torch.equal(x, y), key


def test_checked_library_reports_bad_csr(libs):
    normal, checked = libs
    wl = Workload("r1", 1, 3, 128, 3, 7, 9, 2, 4, 4, 0.3, True, (44, 42, 42))
    q, k, v = make_qkv(wl, "cuda", seed=22)
    g = rf2.geometry_of(wl)
    rf2._lib = checked
    try:
        qp, kp, vp = rf2.permute(g, q), rf2.permute(g, k), rf2.permute(g, v)
        mask = rf2.predict_mask(g, qp, kp, wl.keep)
        torch.cuda.synchronize()
        assert rf2.device_status() == rf2.RF2_OK
        Tb = mask.sizes.num_blocks
        mid = mask.row_count.numel() // 2
        for corrupt in ("count", "value"):
            bad = rf2.BlockMask(mask.row_start.clone(), mask.row_count.clone(), mask.col_idx.clone(), mask.sizes)
            if corrupt == "count":
                bad.row_count[mid] = Tb + 5            # the kernel would clamp it to T_b: inside col_idx
            else:
                bad.col_idx[int(mask.row_start[mid])] = Tb + 3
            rf2.block_sparse_attn(g, qp, kp, vp, bad)
            torch.cuda.synchronize()
            assert rf2.device_status() == rf2.RF2_ERR_RANGE, corrupt
        rf2.block_sparse_attn(g, qp, kp, vp, mask)
        assert rf2.device_status() == rf2.RF2_OK
    finally:
        rf2._lib = normal
