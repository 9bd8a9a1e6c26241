"""Failure detection on the GPU without a fault: a kernel whose only wait can never be satisfied
gives up at the bounded-wait limit, the host reads MOE_ERR_TIMEOUT from the device error word,
and the device keeps working (a layer call afterwards matches the one before).  No trap, no
invalid access, no endless loop: the wait is the library's ordinary bounded mbarrier wait."""
import time

import pytest
import torch

import synth
from _util import to_dev_bf16


@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_the_device_stays_usable():
    import moe_layer_router_b200 as moe
    wl = synth.Workload("tiny_to", 64, 256, 8, 2, 256)
    inp = synth.Inputs(wl)
    W = synth.device_tensors(wl, "cuda")
    x = to_dev_bf16(inp.x())
    T, d, E, k, f = wl.T, wl.d, wl.E, wl.k, wl.f
    ws = torch.empty(moe.moe_workspace_bytes(T, d, E, k, f, 0), dtype=torch.uint8, device="cuda")

    def layer():
        out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
        moe.moe_layer_forward(x, W["wg"], None, W["w1"], W["w3"], W["w2"], None, None, None, 0, T, d, E, k, f,
                              1.0, moe.MOE_CAP_NONE, out, ws)
        return out

    before = layer()
    assert moe.moe_get_error() == moe.MOE_OK
    t0 = time.time()
    moe.moe_selftest_wait_timeout()
    assert moe.moe_get_error() == moe.MOE_ERR_TIMEOUT      # synchronises, reads and clears
    assert time.time() - t0 < 30
    assert moe.moe_get_error() == moe.MOE_OK
    after = layer()
    assert moe.moe_get_error() == moe.MOE_OK
    assert torch.equal(before, after)
