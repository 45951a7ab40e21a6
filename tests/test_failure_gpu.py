"""Failure detection on the GPU without a GPU fault: the library's bounded
waits (the mbarrier waits of the tensor-core router kernels and the grid
barrier of the cooperative dispatch kernel) give up after their limit, raise
the device flag and let the kernel return; the host reads MR_ERR_TIMEOUT and
the context stays usable."""
import time

import numpy as np
import pytest
import torch

import token_dispatch_fp32_b200 as mr
import workloads as wl
from parity import compare_router, oracle_router, router_inputs, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which", [0, 1], ids=["mbarrier", "grid_barrier"])
def test_bounded_wait_gives_up_and_reports_timeout(which):
    assert mr.mr_get_error() == mr.MR_OK
    t0 = time.monotonic()
    assert mr.lib().mr_selftest_bounded_wait(which, None) == mr.MR_OK
    assert mr.mr_get_error() == mr.MR_ERR_TIMEOUT
    elapsed = time.monotonic() - t0
    assert 0.9 < elapsed < 30.0, elapsed  # the limit is one second
    assert mr.mr_get_error() == mr.MR_OK  # read and cleared
    # the context still works: a routing call matches the oracle
    w = wl.TINY
    d = router_inputs(w)
    idx, wt = mr.mr_router_forward(to_dev(d["x_f32"]), to_dev(d["W"]), to_dev(d["b"]),
                                   w.n_group, w.topk_group, w.k, w.route_scale, w.mask_mode)
    assert mr.mr_get_error() == mr.MR_OK
    compare_router(idx.cpu().numpy(), wt.cpu().numpy(), oracle_router(w, np.arange(w.T)))
    torch.cuda.synchronize()
