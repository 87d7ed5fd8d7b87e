"""Failure paths on the GPU, made to happen without faulting anything.

* A device-side bounded wait that runs out: a test-only kernel leaves the
  plan's scheduling state as an interrupted forward could and then waits, with
  a short poll limit, on a flag that nothing sets.  The wait gives up and sets
  the error word; moe_sync_status must report MOE_ERR_TIMEOUT within a second,
  clear the state, and the next forward must match the oracle.
* Device allocations that fail: MOE_FAIL_ALLOC_AFTER=n makes plan creation's
  (n+1)-th allocation fail on the host side.  moe_plan_create must return
  MOE_ERR_OOM and release everything it had allocated.
"""
import time

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import mxfp4_latent_moe_router_b200 as moe  # noqa: E402
from mxfp4_latent_moe_router_b200 import synth  # noqa: E402
from helpers import assert_close, bf16_to_f32, check_routing  # noqa: E402

pytestmark = pytest.mark.gpu


def _forward(plan, x):
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    out = torch.empty_like(xt)
    plan.forward(xt, out)
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint16)


def test_expired_wait_reports_timeout_and_plan_recovers():
    shape = synth.SHAPES["tiny"]
    w = synth.make_weights(shape)
    plan = moe.MoePlan(moe.config_from_shape(shape, max_tokens=8))
    plan.load(moe.weights_to_device(w))
    x = synth.make_x(shape, tokens=8, step=3)
    _forward(plan, x)
    assert plan.sync_status() == 0
    t0 = time.perf_counter()
    assert moe.moe_debug_expire_wait(plan.handle, 1000) == 0
    st = plan.sync_status()
    dt = time.perf_counter() - t0
    assert st == 6, moe.moe_status_str(st)          # MOE_ERR_TIMEOUT
    assert dt < 1.0, dt
    assert plan.sync_status() == 0                  # reported once, then cleared
    # the state the expired wait left behind is gone: routing and output match
    # the oracle again, on two forwards in a row
    for step in (4, 5):
        x = synth.make_x(shape, tokens=8, step=step)
        out = _forward(plan, x)
        assert plan.sync_status() == 0
        ref = oracle.forward(shape, w, x, intermediates=False)
        ids, wts = plan.routing(8)
        logits = plan.fetch(moe.MOE_DBG_LOGITS, 8)
        near = check_routing(shape, w, x, ids, wts, logits, ref)
        assert not near
        assert_close(bf16_to_f32(out), ref["out"], "out after a timeout")
    assert moe.moe_debug_expire_wait(plan.handle, 0) == 1  # limit out of range
    plan.close()


@pytest.mark.parametrize("n", [0, 1, 2, 5, 12, 20])
def test_failed_allocation_returns_oom_and_leaks_nothing(n, monkeypatch):
    # E=64 experts of I=1024 over L=1024: the packed expert tensors alone are
    # 2 x 53 MB, so any of them left behind shows in the free-memory count
    shape = synth.custom_shape("oom", 16, 2048, 1024, 64, 4, 1024, 512, synth.SCORE_SIGMOID)
    cfg = moe.config_from_shape(shape, max_tokens=16)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    monkeypatch.setenv("MOE_FAIL_ALLOC_AFTER", str(n))
    with pytest.raises(moe.MoeError) as ei:
        moe.MoePlan(cfg)
    assert ei.value.status == 4                     # MOE_ERR_OOM
    monkeypatch.delenv("MOE_FAIL_ALLOC_AFTER")
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    # the driver's accounting moves in 2 MB pages; a leaked packed tensor
    # would hold tens of MB
    assert free0 - free1 < 8 * 1024 * 1024, (free0, free1)
    plan = moe.MoePlan(cfg)                          # without the injection it succeeds
    plan.close()
