"""The kernels' failure path on the GPU, without a fault: a wait that nothing
completes runs out after ~1 s, records FT_DEV_WAIT_TIMEOUT with where it
happened, raises the CTA's abort flag so the other role leaves too, and the
kernel ends normally; the next layer call on the same context is correct."""
import time

import numpy as np
import pytest
import torch

from moe_expert_layer_renorm_b200 import _lib, inputs
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_the_context_stays_usable(cuda_device):
    _lib.device_status(clear=True)
    out = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    _lib.selftest_wait_timeout(out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    detail = _lib.device_status_detail()          # synchronises
    elapsed = time.perf_counter() - t0
    assert _lib.device_status(clear=True) == _lib.FT_DEV_WAIT_TIMEOUT
    assert out.cpu().tolist() == [1, 1]           # both warps' waits gave up
    # code, block, warp, barrier kind (4: token stage full), counter, unit
    assert detail[:6] == [_lib.FT_DEV_WAIT_TIMEOUT, 0, 0, 4, 7, 3]
    assert 1_000_000 <= detail[6] < 1_500_000     # microseconds waited (warp 1 would give up at 1.5 s)
    assert 0.9 < elapsed < 30.0
    assert _lib.device_status_detail() == [0] * 8  # cleared with the status word

    w = inputs.WORKLOADS["tiny"]
    run = G.run_gpu(w)                             # asserts a clean status itself
    G.check_routing(run, w.k)
    G.check_output(run, w.k)
