"""moe_layer_forward_static: the decode path for callers that cannot let a library allocate
device memory (engines that own a fixed memory pool, plugins inside a host that owns every
allocation, loops that cannot afford an allocation's synchronisation). Its scratch is a
static device array; this file checks it against moe_layer_forward on two calls in a row --
bit for bit against both decode paths, which compute a token the same way -- at the
workload shape and at the array's largest shape (also against the FP64 oracle there), and
that it rejects shapes beyond the array's limits. It is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
import mixture_experts_gemv_b200 as moe
from gpu_util import DevLayer, TOL_GEMV, dev, ensure_init, rel_err

pytestmark = pytest.mark.gpu


def _reference(x, dl, T, d, f, E, k, path):
    ensure_init(T, d, f, E, k)
    moe.moe_set_path(path, 16)
    ref = torch.empty((T, d), dtype=torch.float32, device="cuda:0")
    moe.moe_layer_forward(x, dl.router_w, dl.router_scale, dl.gate_up, dl.down, dl.expert_scale,
                          T, d, f, E, k, ref)
    moe.moe_debug_check()
    moe.moe_set_path(moe.MOE_PATH_AUTO, 16)
    return ref


def _static_twice(x, dl, T, d, f, E, k):
    outs = []
    for _ in range(2):
        out = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda:0")
        moe.moe_layer_forward_static(x, dl.router_w, dl.router_scale, dl.gate_up, dl.down,
                                     dl.expert_scale, T, d, f, E, k, out)
        moe.moe_layer_forward_static_check()
        outs.append(out)
    return outs


def test_static_entry_matches_layer_forward_on_two_calls():
    from mixture_experts_gemv_b200 import build
    build.build()
    wl = mi.make_workload("decode_T8")
    lw = wl.layers[0]
    T, d, f, E, k = wl.T, lw.d, lw.f, lw.E, wl.k
    dl = DevLayer(lw)
    x = dev(wl.x)
    refs = [_reference(x, dl, T, d, f, E, k, p) for p in (moe.MOE_PATH_GEMV, moe.MOE_PATH_GEMV_SPLIT)]
    r = refs[0].cpu().numpy().astype(np.float64)
    for out in _static_twice(x, dl, T, d, f, E, k):
        got = out.cpu().numpy()
        assert np.isfinite(got).all()
        assert rel_err(got, r) <= TOL_GEMV
        for ref in refs:
            assert torch.equal(out, ref)


def test_static_entry_at_its_largest_shape():
    """T = 16 tokens, T * k = 128 slots, d = 4096, f = 1024, E = 256: every sub-buffer of the
    array at its limit, tokens 9-16 included; against the oracle and moe_layer_forward."""
    T, d, f, E, k = 16, 4096, 1024, 256, 8
    lw = mi.make_layer(seed=77, d=d, f=f, E=E)
    xb = mi.make_tokens(78, T, d)
    dl = DevLayer(lw)
    x = dev(xb)
    ref = _reference(x, dl, T, d, f, E, k, moe.MOE_PATH_GEMV_SPLIT)
    logits = oracle.router_logits(xb, lw.router_w)
    ids, w, flags = oracle.topk_softmax(logits, k, float(lw.router_scale[0]))
    tok = np.nonzero((flags & 1) == 0)[0]
    want = oracle.experts_combine(xb, lw.gate_up, lw.down, lw.expert_scale, ids, w, d, f, tokens=tok)
    for out in _static_twice(x, dl, T, d, f, E, k):
        assert torch.equal(out, ref)
        assert rel_err(out.cpu().numpy()[tok], want) <= TOL_GEMV


def test_static_entry_rejects_shapes_beyond_its_scratch():
    L = moe.lib()
    fake = ctypes.c_void_p(4096)
    rc = L.moe_layer_forward_static(fake, fake, fake, fake, fake, fake, 17, 2816, 704, 128, 8, fake, None)
    assert rc == moe.MOE_ERR_BAD_ARG
    assert "exceeds the static scratch limits" in moe.moe_last_error()
    rc = L.moe_layer_forward_static(fake, fake, fake, fake, fake, fake, 8, 8192, 704, 128, 8, fake, None)
    assert rc == moe.MOE_ERR_BAD_ARG
