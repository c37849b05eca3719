"""Failure detection on the GPU without a fault.

The grid-wide token-choice layout waits at a grid barrier for every CTA to
arrive; the wait is bounded (2 s of wall clock) and, when it runs out, the
kernel records EP_DEVERR_TIMEOUT in the workspace's error word and returns.
Here the barrier's arrival counter is set to a value no arrival can reach, so
nothing ever releases the wait: the call must come back with the timeout
flag, and after the workspace is zeroed again the context must still work.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from combine_ep_get_10_b200 import binding as B
from combine_ep_get_10_b200 import workloads as W
from gpu_util import host, to_dev

pytestmark = pytest.mark.gpu

ARRIVE_WORD = 64  # byte offset of the grid barrier's arrival counter in the workspace


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_ep_get_10_b200 import build

    build.build()
    B.lib()
    oracle.build()


def test_grid_barrier_wait_runs_out_and_is_reported():
    inp = W.make_inputs(2, T=4608)  # 36864 (token, k) pairs: the grid-wide layout
    idx = inp["topk_idx"]
    routing = B.Routing.topk(to_dev(idx), 256, 8)
    lay = B.Layout(routing)
    lay.workspace[ARRIVE_WORD:ARRIVE_WORD + 4].view(torch.int32).fill_(1 << 20)
    t0 = time.time()
    B.ep_get_layout(routing, lay)
    flags = B.ep_get_device_error(lay)
    elapsed = time.time() - t0
    assert flags & B.EP_DEVERR_TIMEOUT
    assert 1.0 < elapsed < 60.0

    # the context stays usable: zero the workspace, lay out again, check it
    B.ep_workspace_init(lay.workspace)
    B.ep_get_layout(routing, lay)
    assert B.ep_get_device_error(lay) == 0
    ref = oracle.tc_layout(idx, 256, 8)
    assert np.array_equal(host(lay.slot), ref["slot"])
    assert np.array_equal(host(lay.expert_offsets), ref["expert_offsets"])
