"""Failure detection on the GPU without a GPU fault: a forward is told to skip one step (CTA 0
of the fused decode kernel never stores its router logits), every CTA's bounded wait for them
runs out after the shortened bound, the kernel ends on its own, the call reports
MOE_ERR_DEVICE_TIMEOUT, and the next forward on the same context is clean and matches the
oracle.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import mixture_experts_gemv_b200 as moe
from gpu_util import DevLayer, TOL_GEMV, dev, ensure_init, rel_err, run_layer

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_the_next_call_is_clean():
    from mixture_experts_gemv_b200 import build
    build.build()
    import oracle
    E, d, f, k, T = 32, 512, 128, 4, 3
    lw = mi.make_layer(seed=91, d=d, f=f, E=E)
    xb = mi.make_tokens(92, T, d)
    dl = DevLayer(lw)
    ensure_init(T, d, f, E, k)
    moe.moe_set_path(moe.MOE_PATH_GEMV, 16)
    good = run_layer(xb, dl, k, moe.MOE_PATH_GEMV, want_routing=False)["out"]

    moe.moe_debug_set_wait_ns(1_000_000)        # 1 ms
    try:
        moe.moe_debug_inject(moe.MOE_INJECT_SKIP_ROUTER_ARRIVAL)
        out = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda:0")
        moe.moe_layer_forward(dev(xb), dl.router_w, dl.router_scale, dl.gate_up, dl.down,
                              dl.expert_scale, T, d, f, E, k, out)
        with pytest.raises(moe.MoeError) as ei:
            moe.moe_debug_check()
        assert ei.value.code == moe.MOE_ERR_DEVICE_TIMEOUT
        assert "timed out" in moe.moe_last_error()
        moe.moe_debug_check()                    # reported once, then clear
    finally:
        moe.moe_debug_set_wait_ns(0)
        moe.moe_debug_inject(moe.MOE_INJECT_NONE)

    # the context is usable: the next forwards (which first reset the arrival counters) give
    # the same bits as before the fault, and match the oracle
    for _ in range(2):
        again = run_layer(xb, dl, k, moe.MOE_PATH_GEMV, want_routing=False)["out"]
        assert np.array_equal(again.view(np.uint32), good.view(np.uint32))
    ref, _, _, flags = oracle.moe_layer(xb, lw.router_w, lw.router_scale, lw.gate_up, lw.down,
                                        lw.expert_scale, k)
    ok = (flags & 1) == 0
    assert rel_err(good[ok], ref[ok]) <= TOL_GEMV
    moe.moe_set_path(moe.MOE_PATH_AUTO, 16)


def test_static_check_is_clean_after_normal_calls():
    """The static entry's error word stays clear in normal operation."""
    E, d, f, k, T = 16, 256, 64, 2, 4
    lw = mi.make_layer(seed=93, d=d, f=f, E=E)
    dl = DevLayer(lw)
    x = dev(mi.make_tokens(94, T, d))
    out = torch.empty((T, d), dtype=torch.float32, device="cuda:0")
    moe.moe_layer_forward_static(x, dl.router_w, dl.router_scale, dl.gate_up, dl.down, dl.expert_scale,
                                 T, d, f, E, k, out)
    moe.moe_layer_forward_static_check()
    assert torch.isfinite(out).all()
