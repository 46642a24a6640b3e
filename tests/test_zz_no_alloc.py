"""moe_layer_forward_static: the decode path for callers that cannot let a library allocate
device memory (engines that own a fixed memory pool, plugins inside a host that owns every
allocation, loops that cannot afford an allocation's synchronisation). Its scratch is a
static device array; this file checks it against moe_layer_forward on two calls in a row,
and that it rejects shapes beyond the array's limits. It is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import moe_inputs as mi
import mixture_experts_gemv_b200 as moe
from gpu_util import DevLayer, TOL_GEMV, dev, ensure_init, rel_err

pytestmark = pytest.mark.gpu


def test_static_entry_matches_layer_forward_on_two_calls():
    from mixture_experts_gemv_b200 import build
    build.build()
    wl = mi.make_workload("decode_T8")
    lw = wl.layers[0]
    T, d, f, E, k = wl.T, lw.d, lw.f, lw.E, wl.k
    dl = DevLayer(lw)
    ensure_init(T, d, f, E, k)
    moe.moe_set_path(moe.MOE_PATH_GEMV, 16)
    x = dev(wl.x)
    ref = torch.empty((T, d), dtype=torch.float32, device="cuda:0")
    moe.moe_layer_forward(x, dl.router_w, dl.router_scale, dl.gate_up, dl.down, dl.expert_scale,
                          T, d, f, E, k, ref)
    moe.moe_debug_check()
    moe.moe_set_path(moe.MOE_PATH_AUTO, 16)
    r = ref.cpu().numpy().astype(np.float64)
    for _ in range(2):
        out = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda:0")
        moe.moe_layer_forward_static(x, dl.router_w, dl.router_scale, dl.gate_up, dl.down,
                                     dl.expert_scale, T, d, f, E, k, out)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.isfinite(got).all()
        assert rel_err(got, r) <= TOL_GEMV


def test_static_entry_rejects_shapes_beyond_its_scratch():
    L = moe.lib()
    fake = ctypes.c_void_p(4096)
    rc = L.moe_layer_forward_static(fake, fake, fake, fake, fake, fake, 17, 2816, 704, 128, 8, fake, None)
    assert rc == moe.MOE_ERR_BAD_ARG
    assert "exceeds the static scratch limits" in moe.moe_last_error()
    rc = L.moe_layer_forward_static(fake, fake, fake, fake, fake, fake, 8, 8192, 704, 128, 8, fake, None)
    assert rc == moe.MOE_ERR_BAD_ARG
