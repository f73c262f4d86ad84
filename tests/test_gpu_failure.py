"""Failure detection on the GPU, without faulting it.

Every wait of the library's kernels on an mbarrier is bounded: when it runs
out, the kernel records RF2_ERR_TIMEOUT in the device status word, raises the
CTA's abort flag so that the CTA's other roles leave their waits too, and
returns.  Here a bounded wait is made to run out on purpose (a barrier that
nothing completes, through the library's self-test entry point), and the
host reads the status; the context must stay usable afterwards.
"""
import time

import pytest
import torch

from image_dits_b200 import build as rf2_build
from image_dits_b200 import rf2
from image_dits_b200.workload import WORKLOADS, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    rf2_build.build()
    rf2.lib()
    yield
    torch.cuda.synchronize()


def test_bounded_wait_times_out_and_context_survives():
    assert rf2.device_status() == rf2.RF2_OK
    rf2.selftest_wait_timeout(1000)                 # first launch: module set-up out of the timing
    assert rf2.device_status() == rf2.RF2_ERR_TIMEOUT
    t0 = time.perf_counter()
    given_up = rf2.selftest_wait_timeout(2000)      # 2 ms
    dt = time.perf_counter() - t0
    # both waits ended without their barrier: the first on its own 2 ms limit,
    # the second through the abort flag (its own limit is 2 s)
    assert given_up == 2
    assert dt < 1.0, dt
    assert rf2.device_status() == rf2.RF2_ERR_TIMEOUT
    assert rf2.device_status() == rf2.RF2_OK        # read and cleared
    # the context is still usable: the whole path runs clean, twice, with equal bits
    wl = WORKLOADS["tiny"]
    q, k, v = make_qkv(wl, "cuda", seed=1)
    g = rf2.geometry_of(wl)
    o1, _ = rf2.rainfusion_attention(g, q, k, v, wl.keep)
    o2, _ = rf2.rainfusion_attention(g, q, k, v, wl.keep)
    torch.cuda.synchronize()
    assert rf2.device_status() == rf2.RF2_OK
    assert torch.isfinite(o1.float()).all()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
