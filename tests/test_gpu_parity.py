"""GPU parity: the CUDA path through the C ABI against the FP64 oracle on seeded inputs.

Small shapes spanning several tiles and ragged tails, every edge case of the routing,
and the five full-size workloads (sampled where the oracle would take minutes).
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
import mixture_experts_gemv_b200 as moe
from gpu_util import (CHUNK, DevLayer, TOL_GEMM, TOL_GEMV, check_routing, dev, ensure_init, rel_err,
                      run_layer)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixture_experts_gemv_b200 import build
    build.build()
    yield
    moe.moe_set_path(moe.MOE_PATH_AUTO, 16)


def _tol(path, T):
    if path in (moe.MOE_PATH_GEMV, moe.MOE_PATH_GEMV_SPLIT):
        return TOL_GEMV
    if path == moe.MOE_PATH_GEMM:
        return TOL_GEMM
    return TOL_GEMV if T <= 16 else TOL_GEMM


def _check_full(x, lw, k, path, tokens=None):
    dl = DevLayer(lw)
    res = run_layer(x, dl, k, path)
    logits = oracle.router_logits(x, lw.router_w)
    ids, w, flags = oracle.topk_softmax(logits, k, float(lw.router_scale[0]))
    T = x.shape[0]
    # a call above the workspace's capacity runs in chunks; the routing readers return the
    # last chunk's
    last = np.arange(((T - 1) // CHUNK) * CHUNK, T) if T > 0 else np.arange(0)
    check_routing(res, ids[last], w[last], flags[last], k, lw.E)
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    tok = tok[(flags[tok] & 1) == 0]
    ref = oracle.experts_combine(x, lw.gate_up, lw.down, lw.expert_scale, ids, w, lw.d, lw.f, tokens=tok)
    err = rel_err(res["out"][tok], ref)
    assert err <= _tol(path, T), f"relative error {err:.3e}"
    return res, err


# ------------------------------------------------------------------ small shapes

SMALL = [  # (E, k, T, d, f)
    (4, 1, 1, 64, 32), (4, 4, 7, 64, 32), (8, 2, 33, 256, 64), (8, 8, 2, 96, 64),
    (128, 8, 1, 256, 96), (128, 8, 33, 512, 128), (128, 2, 300, 256, 64), (128, 128, 3, 64, 32),
    (16, 3, 17, 2816, 64), (6, 2, 16, 320, 704),
    (200, 8, 5, 256, 64),    # E above the CTA count: a CTA computes two router rows
    (256, 16, 3, 128, 64),   # E = 256 with k > 8: eight logits a lane, 64-bit selection keys
]


@pytest.mark.parametrize("E,k,T,d,f", SMALL)
def test_small_shapes_gemv(E, k, T, d, f):
    lw = mi.make_layer(seed=E * 1000 + T, layer=0, d=d, f=f, E=E)
    x = mi.make_tokens(E + T, T, d)
    _check_full(x, lw, k, moe.MOE_PATH_GEMV)


@pytest.mark.parametrize("E,k,T,d,f", SMALL)
def test_small_shapes_gemv_split(E, k, T, d, f):
    """The same shapes through the separate routing / gate_up / down kernels."""
    lw = mi.make_layer(seed=E * 1000 + T, layer=0, d=d, f=f, E=E)
    x = mi.make_tokens(E + T, T, d)
    _check_full(x, lw, k, moe.MOE_PATH_GEMV_SPLIT)


@pytest.mark.parametrize("T", [1, 3, 8])
def test_fused_and_split_decode_agree(T):
    lw = mi.make_layer(seed=40 + T, d=2816, f=704, E=128)
    x = mi.make_tokens(41 + T, T, 2816)
    dl = DevLayer(lw)
    a = run_layer(x, dl, 8, moe.MOE_PATH_GEMV)
    b = run_layer(x, dl, 8, moe.MOE_PATH_GEMV_SPLIT)
    assert np.array_equal(a["ids"], b["ids"]) and np.array_equal(a["perm"], b["perm"])
    assert rel_err(a["out"], b["out"].astype(np.float64)) <= 1e-5
    c = run_layer(x, dl, 8, moe.MOE_PATH_GEMV)
    assert np.array_equal(a["out"].view(np.uint32), c["out"].view(np.uint32))


SMALL_GEMM = [  # (E, k, T, d, f): d % 128 == 0, f % 64 == 0
    (8, 2, 33, 256, 64), (4, 4, 130, 128, 128), (128, 8, 300, 512, 128), (16, 4, 257, 2816, 704),
    (128, 2, 17, 256, 64), (3, 3, 40, 384, 192),
    (2, 2, 600, 256, 64),   # 600 rows per expert: five tiles, two tile pairs and a ragged single
    (256, 8, 200, 256, 64), (200, 4, 150, 512, 128),   # E > 128: the router on the CUDA cores (FP32)
]


@pytest.mark.parametrize("E,k,T,d,f", SMALL_GEMM)
def test_small_shapes_gemm(E, k, T, d, f):
    lw = mi.make_layer(seed=E * 1000 + T + 7, layer=0, d=d, f=f, E=E)
    x = mi.make_tokens(E + T + 7, T, d)
    _check_full(x, lw, k, moe.MOE_PATH_GEMM)


def test_gemm_hidden_matches_oracle():
    E, d, f, k, T = 16, 256, 128, 3, 70
    lw = mi.make_layer(seed=14, d=d, f=f, E=E)
    x = mi.make_tokens(15, T, d)
    run_layer(x, DevLayer(lw), k, moe.MOE_PATH_GEMM)
    h = torch.empty((T * k, f), dtype=torch.float32, device="cuda:0")
    moe.moe_debug_get_hidden(h)
    torch.cuda.synchronize()
    logits = oracle.router_logits(x, lw.router_w)
    ids, w, flags = oracle.topk_softmax(logits, k, 1.0)
    _, href = oracle.experts_combine(x, lw.gate_up, lw.down, lw.expert_scale, ids, w, d, f, want_h=True)
    assert rel_err(h.cpu().numpy().reshape(T, k, f), href) <= TOL_GEMM


def test_gemm_and_gemv_paths_agree():
    E, d, f, k, T = 32, 512, 192, 4, 40
    lw = mi.make_layer(seed=16, d=d, f=f, E=E)
    x = mi.make_tokens(17, T, d)
    dl = DevLayer(lw)
    a = run_layer(x, dl, k, moe.MOE_PATH_GEMV)["out"]
    b = run_layer(x, dl, k, moe.MOE_PATH_GEMM)
    assert rel_err(b["out"], a.astype(np.float64)) <= TOL_GEMM
    c = run_layer(x, dl, k, moe.MOE_PATH_GEMM)["out"]
    assert np.array_equal(b["out"].view(np.uint32), c.view(np.uint32))


def test_zero_tokens_is_a_noop():
    lw = mi.make_layer(seed=1, d=64, f=32, E=4)
    dl = DevLayer(lw)
    ensure_init(1, 64, 32, 4, 2)
    out = torch.full((1, 64), 7.0, device="cuda:0")
    x = torch.zeros((1, 64), dtype=torch.int16, device="cuda:0")
    moe.moe_layer_forward(x, dl.router_w, dl.router_scale, dl.gate_up, dl.down, dl.expert_scale,
                          0, 64, 32, 4, 2, out)
    moe.moe_debug_check()
    assert (out.cpu() == 7.0).all()


def test_tied_logits_pick_lower_index():
    E, d, f, k = 8, 64, 32, 2
    lw = mi.make_layer(seed=3, d=d, f=f, E=E)
    lw.router_w[:] = 0.0
    lw.router_w[[1, 3, 5], 0] = 1.0          # experts 1, 3, 5 tie for the top logit
    x = mi.make_tokens(5, 4, d)
    x[:, 0] = mi.f32_to_bf16_bits(np.array([2.0], np.float32))[0]
    res = run_layer(x, DevLayer(lw), k, moe.MOE_PATH_GEMV)
    assert (res["ids"].reshape(4, k) == np.array([1, 3])).all()


def test_router_scale_and_expert_scale_enter_the_output():
    E, d, f, k, T = 8, 128, 64, 2, 3
    lw = mi.make_layer(seed=4, d=d, f=f, E=E)
    x = mi.make_tokens(6, T, d)
    base = run_layer(x, DevLayer(lw), k, moe.MOE_PATH_GEMV)["out"]
    lw.router_scale[0] = 0.5
    half = run_layer(x, DevLayer(lw), k, moe.MOE_PATH_GEMV)["out"]
    assert np.allclose(half, 0.5 * base, rtol=1e-6, atol=1e-12)
    _check_full(x, lw, k, moe.MOE_PATH_GEMV)


def test_nan_input_propagates():
    E, d, f, k, T = 8, 64, 32, 2, 3
    lw = mi.make_layer(seed=5, d=d, f=f, E=E)
    x = mi.make_tokens(7, T, d)
    x[1, 5] = 0x7FC0    # bf16 NaN in token 1
    out = run_layer(x, DevLayer(lw), k, moe.MOE_PATH_GEMV, want_routing=False)["out"]
    assert np.isnan(out[1]).all()
    assert np.isfinite(out[0]).all() and np.isfinite(out[2]).all()


def test_deterministic_bitwise():
    lw = mi.make_layer(seed=8, d=512, f=128, E=32)
    x = mi.make_tokens(9, 8, 512)
    dl = DevLayer(lw)
    a = run_layer(x, dl, 4, moe.MOE_PATH_GEMV)["out"]
    b = run_layer(x, dl, 4, moe.MOE_PATH_GEMV)["out"]
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


def test_batch_invariant_decode():
    """A token's output does not depend on the other tokens of the call, for every T the
    GEMV path takes (T <= 8: the fused decode kernel; 9 <= T <= 16: the separate decode
    kernels, which cut the router and the down rows as the fused kernel does): the verification
    pass of speculative decoding must give plain decoding's logits bit for bit (page "Gemma 4
    26B-A4B it QAT Q4_0 ... NInfer v3 artifact", "Speculative decoding", "Quality"). Singles,
    pairs, fours, eights, twelves and the reversed batch against the batch of sixteen."""
    E, d, f, k = 64, 1024, 256, 8
    lw = mi.make_layer(seed=21, d=d, f=f, E=E)
    x = mi.make_tokens(22, 16, d)
    dl = DevLayer(lw)
    full = run_layer(x, dl, k, moe.MOE_PATH_AUTO, want_routing=False)["out"].view(np.uint32)
    subsets = ([0], [5], [15], [0, 1], [14, 2], [2, 3, 4, 5], [9, 1, 12, 7], list(range(8)),
               list(range(8, 16)), list(range(9)), list(range(3, 15)), list(range(15, -1, -1)))
    for sel in subsets:
        part = run_layer(x[sel], dl, k, moe.MOE_PATH_AUTO, want_routing=False)["out"].view(np.uint32)
        assert np.array_equal(part, full[sel]), sel


def test_hidden_matches_oracle():
    E, d, f, k, T = 16, 256, 96, 3, 5
    lw = mi.make_layer(seed=12, d=d, f=f, E=E)
    x = mi.make_tokens(13, T, d)
    run_layer(x, DevLayer(lw), k, moe.MOE_PATH_GEMV)
    h = torch.empty((T * k, f), dtype=torch.float32, device="cuda:0")
    moe.moe_debug_get_hidden(h)
    torch.cuda.synchronize()
    logits = oracle.router_logits(x, lw.router_w)
    ids, w, flags = oracle.topk_softmax(logits, k, 1.0)
    _, href = oracle.experts_combine(x, lw.gate_up, lw.down, lw.expert_scale, ids, w, d, f, want_h=True)
    assert rel_err(h.cpu().numpy().reshape(T, k, f), href) <= TOL_GEMV


def test_rmsnorm_matches_oracle_up_to_rounding_ties():
    rng = np.random.default_rng(3)
    y = (rng.standard_normal((4, 2816)) * 0.01).astype(np.float32)
    ensure_init(4, 2816, 704, 128, 8)
    xo = torch.empty((4, 2816), dtype=torch.int16, device="cuda:0")
    moe.moe_rmsnorm_bf16(dev(y), xo, 4, 2816, 1e-6)
    torch.cuda.synchronize()
    got = xo.cpu().numpy().view(np.uint16)
    ref = oracle.rmsnorm_bf16(y.astype(np.float64), 1e-6)
    diff = got != ref
    # a differing element must sit within FP32 error of a bf16 rounding midpoint
    yd = y.astype(np.float64)
    val = yd / np.sqrt((yd ** 2).mean(1, keepdims=True) + 1e-6)
    for t, i in zip(*np.nonzero(diff)):
        a, b = int(got[t, i]), int(ref[t, i])
        assert abs(a - b) == 1
        lo, hi = sorted([a, b])
        mid = (mi.bf16_bits_to_f32(np.array([lo], np.uint16))[0].astype(np.float64) +
               mi.bf16_bits_to_f32(np.array([hi], np.uint16))[0].astype(np.float64)) / 2
        assert abs(val[t, i] - mid) <= 1e-6 * abs(mid)
    assert diff.mean() < 1e-3


# ------------------------------------------------------------------ full-size workloads

def test_layer_T1():
    wl = mi.make_workload("layer_T1")
    _check_full(wl.x, wl.layers[0], wl.k, moe.MOE_PATH_AUTO)


def test_decode_T8():
    wl = mi.make_workload("decode_T8")
    _check_full(wl.x, wl.layers[0], wl.k, moe.MOE_PATH_AUTO)


def _near_tie_band(x, lw, k, lo=1e-6, hi=1e-4):
    """Unflagged tokens whose FP64 gap between the k-th and (k+1)-th logit lies in (lo, hi]:
    at logits of magnitude ~58 one FP32 ulp is 3.8e-6, so a gap just above the 1e-6 flag
    can be below the FP32 router's own rounding. Reported, and still compared exactly."""
    lg = np.sort(oracle.router_logits(x, lw.router_w), axis=1)[:, ::-1]
    gap = lg[:, k - 1] - lg[:, k]
    return int(((gap > lo) & (gap <= hi)).sum()), float(np.abs(lg).max())


def test_skewed_T512_every_token():
    """Every one of the 512 tokens against the oracle (2e-2 on the tensor-core path), plus
    the skew the workload is meant to have: a few experts above 100 rows, most near empty."""
    wl = mi.make_workload("skewed_T512")
    lw = wl.layers[0]
    band, lmax = _near_tie_band(wl.x, lw, wl.k)
    print(f"skewed_T512: {band} unflagged tokens with a k-th / (k+1)-th FP64 logit gap in "
          f"(1e-6, 1e-4]; max |logit| {lmax:.2f}")
    res, err = _check_full(wl.x, lw, wl.k, moe.MOE_PATH_AUTO)
    counts = res["counts"]
    assert (counts > 100).sum() >= 3 and (counts <= 2).sum() >= 64
    print(f"skewed_T512: max relative error {err:.3e} over all tokens")


def test_skewed_T512_every_token_on_the_gemv_path():
    """The same 512 tokens forced onto the FP32-accumulate GEMV path, at 1e-3."""
    wl = mi.make_workload("skewed_T512")
    _check_full(wl.x, wl.layers[0], wl.k, moe.MOE_PATH_GEMV_SPLIT)


def test_prefill_T4096_every_token():
    """All 4,096 tokens (every row of every tile pair and every ragged tail) against the
    oracle, element by element, at 2e-2."""
    wl = mi.make_workload("prefill_T4096")
    res, err = _check_full(wl.x, wl.layers[0], wl.k, moe.MOE_PATH_AUTO)
    print(f"prefill_T4096: max relative error {err:.3e} over all tokens")


@pytest.fixture(scope="module")
def stack30():
    wl = mi.make_workload("stack30_T1")
    return wl, [DevLayer(lw) for lw in wl.layers]


def test_stack_in_kernel_norm_matches_separate_norm(stack30):
    """In a stack, the fused decode kernel normalises the previous layer's output itself; the
    separate path launches moe_rmsnorm_bf16 and the separate decode kernels. Same bits for
    every layer's x and for the output, over all 30 layers."""
    wl, dls = stack30
    L = len(wl.layers)
    d, f, E, k = mi.D_MODEL, mi.D_FF, mi.N_EXPERTS, wl.k
    ensure_init(1, d, f, E, k)
    res = []
    for path in (moe.MOE_PATH_AUTO, moe.MOE_PATH_GEMV_SPLIT):
        moe.moe_set_path(path, 16)
        out = torch.empty((1, d), dtype=torch.float32, device="cuda:0")
        trace = torch.empty((L, 1, d), dtype=torch.int16, device="cuda:0")
        moe.moe_stack_forward(dev(wl.x), [q.router_w for q in dls], [q.router_scale for q in dls],
                              [q.gate_up for q in dls], [q.down for q in dls], [q.expert_scale for q in dls],
                              1, d, f, E, k, 1e-6, out, trace)
        moe.moe_debug_check()
        res.append((out.cpu().numpy().view(np.uint32), trace.cpu().numpy()))
    moe.moe_set_path(moe.MOE_PATH_AUTO, 16)
    assert np.array_equal(res[0][1], res[1][1])
    assert np.array_equal(res[0][0], res[1][0])


def test_stack_teacher_forced(stack30):
    """All 30 layers: layer i's oracle consumes the GPU's own bf16 input x_i (recorded by
    x_trace); each layer's output is checked through the next layer's input, the last one
    directly."""
    wl, dls = stack30
    L = len(wl.layers)
    d, f, E, k = mi.D_MODEL, mi.D_FF, mi.N_EXPERTS, wl.k
    ensure_init(1, d, f, E, k)
    moe.moe_set_path(moe.MOE_PATH_AUTO, 16)
    out = torch.empty((1, d), dtype=torch.float32, device="cuda:0")
    trace = torch.empty((L, 1, d), dtype=torch.int16, device="cuda:0")
    moe.moe_stack_forward(dev(wl.x), [q.router_w for q in dls], [q.router_scale for q in dls],
                          [q.gate_up for q in dls], [q.down for q in dls], [q.expert_scale for q in dls],
                          1, d, f, E, k, 1e-6, out, trace)
    moe.moe_debug_check()
    xs = trace.cpu().numpy().view(np.uint16)
    assert np.array_equal(xs[0], wl.x)
    for i, lw in enumerate(wl.layers):
        ref, ids, w, flags = oracle.moe_layer(xs[i], lw.router_w, lw.router_scale, lw.gate_up, lw.down,
                                              lw.expert_scale, k)
        if i + 1 < L:
            # x_{i+1} = bf16(rmsnorm(out_i)), element by element: the 1e-3 output bound (with
            # the norm's own scale, 1.1e-3 of the largest element) plus at most one bf16 ulp
            # of rounding difference, and one ulp of a bf16 value v is at most 2^-7 |v|
            nxt = mi.bf16_bits_to_f32(oracle.rmsnorm_bf16(ref)).astype(np.float64)
            got = mi.bf16_bits_to_f32(xs[i + 1]).astype(np.float64)
            bound = 1.1e-3 * np.abs(nxt).max() + 2.0 ** -7 * np.abs(nxt)
            assert (np.abs(got - nxt) <= bound).all(), f"layer {i}: x_{i + 1} outside the bound"
        else:
            assert rel_err(out.cpu().numpy(), ref) <= TOL_GEMV


# ------------------------------------------------------------------ long prompts (chunked)

def _tile_boundary_tokens(T, chunk, k, rng, n_random):
    """Tokens at the chunk boundaries (the first and last 128 of every chunk) plus n_random
    others."""
    edges = set()
    for c0 in range(0, T, chunk):
        c1 = min(T, c0 + chunk)
        edges.update(range(c0, min(c1, c0 + 128)))
        edges.update(range(max(c0, c1 - 128), c1))
    rest = np.setdiff1d(np.arange(T), np.fromiter(edges, dtype=np.int64))
    pick = rng.choice(rest, min(n_random, rest.size), replace=False)
    return np.sort(np.concatenate([np.fromiter(edges, dtype=np.int64), pick]))


def test_chunked_prefill_is_bitwise_one_pass():
    """A 4,096-token prefill through a workspace of 1,024 tokens (four chunks) gives the bits
    of one 4,096-token pass: chunking bounds the workspace without changing any output."""
    import gpu_util
    wl = mi.make_workload("prefill_T4096")
    lw = wl.layers[0]
    d, f, E, k = lw.d, lw.f, lw.E, wl.k
    dl = DevLayer(lw)
    x = dev(wl.x)
    outs = []
    for cap in (4096, 1024):
        moe.moe_init(0, cap, d, f, E, k)
        gpu_util._limits = (cap, d, f, E, k)
        moe.moe_set_path(moe.MOE_PATH_AUTO, 16)
        o = torch.full((wl.T, d), float("nan"), dtype=torch.float32, device="cuda:0")
        moe.moe_layer_forward(x, dl.router_w, dl.router_scale, dl.gate_up, dl.down, dl.expert_scale,
                              wl.T, d, f, E, k, o)
        moe.moe_debug_check()
        outs.append(o)
    assert torch.equal(outs[0], outs[1])
    assert moe.moe_workspace_bytes(1024, d, f, E, k) < moe.moe_workspace_bytes(4096, d, f, E, k)


def test_prefill_T10000_every_token():
    """The 10,000-token prompt (three 4,096-token chunks, the last one ragged): every token
    against the oracle at 2e-2."""
    wl = mi.make_workload("prefill_T10000")
    _, err = _check_full(wl.x, wl.layers[0], wl.k, moe.MOE_PATH_AUTO)
    print(f"prefill_T10000: max relative error {err:.3e} over all tokens")


def test_prefill_T40000_boundaries_and_sample():
    """The 40,000-token prompt (ten chunks): every token of the first and last 128-row tile of
    each chunk, plus 1,000 random tokens, against the oracle at 2e-2."""
    wl = mi.make_workload("prefill_T40000")
    tok = _tile_boundary_tokens(wl.T, 4096, wl.k, np.random.default_rng(2), 1000)
    _, err = _check_full(wl.x, wl.layers[0], wl.k, moe.MOE_PATH_AUTO, tokens=tok)
    print(f"prefill_T40000: max relative error {err:.3e} over {tok.size} tokens")


# ------------------------------------------------------------------ the block's dense MLP

def _run_block(x_bits, dl, dense, k, path, f_dense):
    lw = dl.lw
    T, d = x_bits.shape
    ensure_init(max(T, 1), d, max(lw.f, f_dense), lw.E, k)
    moe.moe_set_path(path, 16)
    gud, dnd = dev(dense[0]), dev(dense[1])
    out = torch.full((max(T, 1), d), float("nan"), dtype=torch.float32, device="cuda:0")
    moe.moe_block_forward(dev(x_bits), dl.router_w, dl.router_scale, dl.gate_up, dl.down, dl.expert_scale,
                          gud, dnd, T, d, lw.f, f_dense, lw.E, k, out)
    moe.moe_debug_check()
    return out[:T].cpu().numpy()


BLOCK = [  # (E, k, T, d, f, f_dense)
    (8, 2, 5, 256, 64, 64), (16, 4, 3, 512, 128, 192), (128, 8, 8, 2816, 704, 704),
    (32, 4, 40, 512, 128, 256), (16, 3, 300, 256, 64, 128),
]


@pytest.mark.parametrize("E,k,T,d,f,fd", BLOCK)
@pytest.mark.parametrize("path", [moe.MOE_PATH_AUTO, moe.MOE_PATH_GEMV_SPLIT, moe.MOE_PATH_GEMM])
def test_block_with_dense_mlp_matches_oracle(E, k, T, d, f, fd, path):
    """Routed layer plus the dense MLP, on the fused decode, split decode and grouped-GEMM paths,
    against the oracle's block (routed combine + dense GeGLU)."""
    lw = mi.make_layer(seed=E * 7 + T, d=d, f=f, E=E)
    dense = mi.make_dense(seed=E * 7 + T, d=d, f_dense=fd)
    x = mi.make_tokens(E + 3 * T, T, d)
    got = _run_block(x, DevLayer(lw), dense, k, path, fd)
    ref, ids, w, flags = oracle.block_ffn(x, lw.router_w, lw.router_scale, lw.gate_up, lw.down, lw.expert_scale,
                                          dense[0], dense[1], k)
    ok = (flags & 1) == 0
    tol = TOL_GEMM if path == moe.MOE_PATH_GEMM else _tol(path, T)
    assert rel_err(got[ok], ref[ok]) <= tol


def test_block_with_zero_dense_mlp_is_the_routed_layer():
    """Zero dense weights (code 8) add exactly nothing: the block equals moe_layer_forward."""
    E, k, T, d, f, fd = 16, 4, 6, 512, 128, 128
    lw = mi.make_layer(seed=61, d=d, f=f, E=E)
    gu0 = np.zeros((2 * fd, d // 32, 18), np.uint8)
    gu0[..., 1] = 0x24                                   # scale 1/64, every code 8
    gu0[..., 2:] = 0x88
    dn0 = np.zeros((d, fd // 32, 18), np.uint8)
    dn0[..., 1] = 0x24
    dn0[..., 2:] = 0x88
    x = mi.make_tokens(62, T, d)
    dl = DevLayer(lw)
    got = _run_block(x, dl, (gu0.reshape(2 * fd, -1), dn0.reshape(d, -1)), k, moe.MOE_PATH_AUTO, fd)
    base = run_layer(x, dl, k, moe.MOE_PATH_AUTO, want_routing=False)["out"]
    assert np.array_equal(got, base)
