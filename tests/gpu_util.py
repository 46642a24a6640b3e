"""Helpers for the GPU parity tests: upload seeded inputs, run the C ABI, compare with the
FP64 oracle under the layer's parity criteria.

Criteria: expert ids bit-exact for tokens whose k-th and (k+1)-th FP64 logits differ by
more than 1e-6 (closer ones are flagged and excluded; selected logits within 1e-6 of each
other compare as a set); combine weights within 1e-5; the permutation equals the stable
counting sort of the GPU's own ids bit-exactly; outputs within a relative error (max
abs difference over max abs reference) of 1e-3 on the FP32-accumulate GEMV path and
2e-2 on the bf16 tensor-core path.
"""
from __future__ import annotations

import numpy as np
import torch

import moe_inputs as mi
import oracle
import mixture_experts_gemv_b200 as moe

TOL_GEMV = 1e-3
TOL_GEMM = 2e-2
TOL_W = 1e-5

_limits = None
CHUNK = 4096   # the tests' workspace holds at most this many tokens; longer calls run in chunks


def ensure_init(T, d, f, E, k):
    global _limits
    need = (min(T, CHUNK), d, f, E, k)
    if _limits is None or any(n > h for n, h in zip(need, _limits)):
        lim = tuple(max(n, h) for n, h in zip(need, _limits)) if _limits else need
        moe.moe_init(0, *lim)
        _limits = lim


def dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to("cuda:0")


class DevLayer:
    def __init__(self, lw: mi.LayerWeights):
        self.lw = lw
        self.router_w = dev(lw.router_w)
        self.router_scale = dev(lw.router_scale)
        self.gate_up = dev(lw.gate_up)
        self.down = dev(lw.down)
        self.expert_scale = dev(lw.expert_scale)


def run_layer(x_bits, dl: DevLayer, k, path=moe.MOE_PATH_AUTO, want_routing=True):
    lw = dl.lw
    T, d = x_bits.shape
    ensure_init(max(T, 1), d, lw.f, lw.E, k)
    moe.moe_set_path(path, 16)
    x = dev(x_bits)
    out = torch.full((max(T, 1), d), float("nan"), dtype=torch.float32, device="cuda:0")
    moe.moe_layer_forward(x, dl.router_w, dl.router_scale, dl.gate_up, dl.down, dl.expert_scale,
                          T, d, lw.f, lw.E, k, out)
    res = {"out": out[:T]}
    if want_routing and T > 0:
        S = (T - ((T - 1) // CHUNK) * CHUNK) * k   # the routing readers hold the last chunk's
        ids = torch.empty(S, dtype=torch.int32, device="cuda:0")
        w = torch.empty(S, dtype=torch.float32, device="cuda:0")
        counts = torch.empty(lw.E, dtype=torch.int32, device="cuda:0")
        offsets = torch.empty(lw.E + 1, dtype=torch.int32, device="cuda:0")
        perm = torch.empty(S, dtype=torch.int32, device="cuda:0")
        moe.moe_debug_get_routing(ids, w, counts, offsets, perm)
        res.update(ids=ids, w=w, counts=counts, offsets=offsets, perm=perm)
    moe.moe_debug_check()
    return {kk: v.cpu().numpy() for kk, v in res.items()}


def check_routing(res, ref_ids, ref_w, flags, k, E):
    """ids / w against the oracle (unflagged tokens); perm against the GPU's own ids."""
    T = ref_ids.shape[0]
    ids = res["ids"].reshape(T, k)
    w = res["w"].reshape(T, k)
    n_checked = 0
    for t in range(T):
        if flags[t] & 1:
            continue
        n_checked += 1
        if flags[t] & 2:
            assert set(ids[t].tolist()) == set(ref_ids[t].tolist()), f"token {t}: ids {ids[t]} vs {ref_ids[t]}"
            for j in range(k):
                jj = int(np.where(ref_ids[t] == ids[t, j])[0][0])
                assert abs(w[t, j] - ref_w[t, jj]) <= TOL_W
        else:
            assert np.array_equal(ids[t], ref_ids[t]), f"token {t}: ids {ids[t]} vs {ref_ids[t]}"
            assert np.max(np.abs(w[t] - ref_w[t])) <= TOL_W, f"token {t}: w {w[t]} vs {ref_w[t]}"
    # permutation: the stable counting sort of the GPU's own ids
    flat = res["ids"]
    assert ((flat >= 0) & (flat < E)).all()
    for t in range(T):
        assert len(set(ids[t].tolist())) == k, f"token {t}: repeated expert"
    exp_perm = np.argsort(flat, kind="stable").astype(np.int32)
    assert np.array_equal(res["perm"], exp_perm)
    exp_counts = np.bincount(flat, minlength=E)
    assert np.array_equal(res["counts"], exp_counts)
    assert np.array_equal(res["offsets"], np.concatenate([[0], np.cumsum(exp_counts)]).astype(np.int32))
    return n_checked


def rel_err(got, ref, rows=None):
    if rows is not None:
        got, ref = got[rows], ref[rows]
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(got.astype(np.float64) - ref)) / max(den, 1e-300))
