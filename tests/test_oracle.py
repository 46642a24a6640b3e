"""Pins of the FP64 CPU oracle against things other than itself.

Each test ties one oracle function to a hand-worked value, a library routine,
brute force, a closed form or an invariant, chosen so that a plausible slip
(a dropped term, a swapped nibble, a wrong sign, a transposed operand) fails.
Source of the layer's definition: the page "Gemma 4 26B-A4B it QAT Q4_0 ...
NInfer v3 artifact" ("What is inside": Q4_0 expert-major [gate; up] 2 x 704 rows,
down 2,816 rows, FP32 router / router scale / expert scales; intro: blocks
multiplied in place, no requantisation).
"""
import itertools
import math

import numpy as np
import pytest
import scipy.special

import moe_inputs as mi
import np_ref


# ------------------------------------------------------------------ fp16 / bf16

@pytest.mark.parametrize("bits,val", [
    (0x3C00, 1.0), (0xBC00, -1.0), (0x2C00, 0.0625), (0x1C00, 2.0 ** -8),
    (0x0001, 2.0 ** -24), (0x03FF, 1023 * 2.0 ** -24), (0x0400, 2.0 ** -14),
    (0x7BFF, 65504.0), (0x3555, 1365 / 4096), (0x0000, 0.0), (0xC500, -5.0),
    (0x7C00, math.inf), (0xFC00, -math.inf),
])
def test_fp16_hand_values(orc, bits, val):
    assert orc.fp16_to_double(bits) == val


def test_fp16_all_patterns_match_numpy(orc):
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.fp16_to_double(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_bf16_all_patterns_match_field_definition(orc):
    bits = np.arange(65536, dtype=np.uint16)
    ref = np_ref.bf16_field_decode(bits)
    got = np.array([orc.bf16_to_double(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


@pytest.mark.parametrize("v,bits", [
    (1.0, 0x3F80), (1.0 + 2.0 ** -8, 0x3F80),            # tie -> even (0x3F80)
    (1.0 + 3 * 2.0 ** -8, 0x3F82),                        # tie -> even (0x3F82)
    (1.0 + 2.0 ** -8 + 2.0 ** -30, 0x3F81),               # just above the tie
    (-2.5, 0xC020), (0.0, 0x0000), (2.0 ** -133, 0x0001),
    (2.0 ** -134, 0x0000), (3 * 2.0 ** -134, 0x0002),     # subnormal ties
    ((2 - 2.0 ** -8) * 2.0 ** 127, 0x7F80),               # rounds up to inf
    ((2 - 2.0 ** -7) * 2.0 ** 127, 0x7F7F),               # max finite
])
def test_bf16_rne_hand_values(orc, v, bits):
    assert orc.double_to_bf16(v) == bits


def test_bf16_rne_brute_force(orc):
    """Nearest bf16 by search over every positive finite bf16, ties to even."""
    pos = np.arange(0, 0x7F80, dtype=np.uint16)
    vals = np_ref.bf16_field_decode(pos)
    rng = np.random.default_rng(123)
    samples = np.concatenate([
        rng.standard_normal(3000) * 10.0 ** rng.integers(-5, 5, 3000),
        rng.standard_normal(200) * 1e-39,
    ])
    for v in samples:
        a = abs(float(v))
        i = int(np.searchsorted(vals, a))
        cands = [j for j in (i - 1, i) if 0 <= j < len(vals)]
        best = min(cands, key=lambda j: (abs(vals[j] - a), int(pos[j]) & 1))
        exp_bits = int(pos[best]) | (0x8000 if v < 0 else 0)
        assert orc.double_to_bf16(float(v)) == exp_bits, v


# ------------------------------------------------------------------ Q4_0 blocks

def _block(d_lo, d_hi, qs):
    return np.array([d_lo, d_hi] + list(qs), dtype=np.uint8)


def test_q4_0_block_minus8_zero(orc):
    # d = 0x3C00 = 1.0; every code byte 0x80: low nibble 0 -> -8, high nibble 8 -> 0
    got = orc.q4_0_decode_block(_block(0x00, 0x3C, [0x80] * 16))
    assert got.tolist() == [-8.0] * 16 + [0.0] * 16


def test_q4_0_block_nibble_order(orc):
    # d = 0x2C00 = 1/16; byte i = i | (15 - i) << 4
    # element i = (i - 8)/16 (low nibble), element 16 + i = (7 - i)/16 (high nibble)
    got = orc.q4_0_decode_block(_block(0x00, 0x2C, [i | ((15 - i) << 4) for i in range(16)]))
    exp = [(i - 8) / 16 for i in range(16)] + [(7 - i) / 16 for i in range(16)]
    assert got.tolist() == exp


def test_q4_0_block_max_code_small_scale(orc):
    # d = 0x1C00 = 2^-8 (inside U(0.001, 0.004)); all nibbles 15 -> 7 * 2^-8
    got = orc.q4_0_decode_block(_block(0x00, 0x1C, [0xFF] * 16))
    assert got.tolist() == [0.02734375] * 32


def test_q4_0_block_negative_scale(orc):
    # d = 0xBC00 = -1.0; byte 0x97: low 7 -> (7-8)(-1) = 1, high 9 -> (9-8)(-1) = -1
    got = orc.q4_0_decode_block(_block(0x00, 0xBC, [0x97] * 16))
    assert got.tolist() == [1.0] * 16 + [-1.0] * 16


def test_q4_0_block_subnormal_scale_and_byte_index(orc):
    # d = 0x3555 = 1365/4096 (little-endian bytes 55 35); byte i = (5i & 15) | ((3i+1) & 15) << 4
    qs = [((5 * i) & 15) | (((3 * i + 1) & 15) << 4) for i in range(16)]
    got = orc.q4_0_decode_block(_block(0x55, 0x35, qs))
    exp = [(((5 * i) & 15) - 8) * 1365 / 4096 for i in range(16)] + \
          [(((3 * i + 1) & 15) - 8) * 1365 / 4096 for i in range(16)]
    assert got.tolist() == exp
    # subnormal d = 0x0001 = 2^-24; byte 0x0F: low 15 -> 7 * 2^-24, high 0 -> -8 * 2^-24
    got = orc.q4_0_decode_block(_block(0x01, 0x00, [0x0F] * 16))
    assert got.tolist() == [7 * 2.0 ** -24] * 16 + [-8 * 2.0 ** -24] * 16


def test_q4_0_block_matches_numpy_float16_decode(orc):
    rng = np.random.default_rng(5)
    blocks = mi.random_q4_0(rng, 64, 32)            # 64 rows of one block each
    ref = np_ref.decode_q4_0(blocks, 32)
    for r in range(64):
        assert np.array_equal(orc.q4_0_decode_block(blocks[r]), ref[r])


# ------------------------------------------------------------------ GELU-tanh

def test_gelu_zero_and_odd_part(orc):
    assert orc.gelu_tanh(0.0) == 0.0
    for z in np.linspace(-7, 7, 141):
        # gelu(z) = z * s(z) with s(z) + s(-z) = 1, so gelu(z) - gelu(-z) = z
        assert abs(orc.gelu_tanh(z) - orc.gelu_tanh(-z) - z) <= 1e-14 * max(1.0, abs(z))


def test_gelu_tanh_close_to_erf_gelu(orc):
    # The tanh form approximates z * Phi(z); a dropped cubic term or a wrong
    # sqrt(2/pi) constant moves it by > 1e-2 somewhere in [-6, 6].
    worst = max(abs(orc.gelu_tanh(z) - np_ref.gelu_erf(z)) for z in np.linspace(-6, 6, 1201))
    assert worst < 5e-4


def test_gelu_asymptotes_and_slope(orc):
    assert abs(orc.gelu_tanh(12.0) - 12.0) < 1e-12
    assert abs(orc.gelu_tanh(-12.0)) < 1e-12
    h = 1e-6
    assert abs((orc.gelu_tanh(h) - orc.gelu_tanh(-h)) / (2 * h) - 0.5) < 1e-9


# ------------------------------------------------------------------ router

def test_router_logits_match_numpy_matmul(orc):
    rng = np.random.default_rng(7)
    x = mi.f32_to_bf16_bits(rng.standard_normal((5, 96)).astype(np.float32))
    W = (rng.standard_normal((12, 96)) / np.sqrt(96)).astype(np.float32)
    got = orc.router_logits(x, W)
    ref = np_ref.bf16_field_decode(x) @ W.astype(np.float64).T
    assert np.allclose(got, ref, rtol=0, atol=1e-13)
    # a transposed operand would not even match this shape-asymmetric case
    assert got.shape == (5, 12)


def _valid_topk(l32, sel):
    inside = set(sel)
    for e in sel:
        for o in range(len(l32)):
            if o in inside:
                continue
            if not (l32[e] > l32[o] or (l32[e] == l32[o] and e < o)):
                return False
    return True


@pytest.mark.parametrize("E", [4, 6, 8])
def test_topk_brute_force_subsets(orc, E):
    rng = np.random.default_rng(E)
    for trial in range(20):
        l = rng.standard_normal((1, E))
        if trial % 4 == 1:
            l[0, rng.integers(E)] = l[0, rng.integers(E)]            # exact tie
        if trial % 4 == 2:
            l[0, :] = np.round(l[0, :])                               # many ties
        l32 = l[0].astype(np.float32)
        for k in range(1, E + 1):
            ids, w, fl = orc.topk_softmax(l, k, 1.0)
            valid = [s for s in itertools.combinations(range(E), k) if _valid_topk(l32, s)]
            assert len(valid) == 1
            assert set(ids[0]) == set(valid[0])
            # order: logit descending, equal logits by ascending index
            keys = [(-float(l32[e]), int(e)) for e in ids[0]]
            assert keys == sorted(keys)


def test_topk_ties_take_lower_index(orc):
    l = np.array([[0.5, 1.0, 1.0, 1.0, 0.2, 1.0]])
    ids, w, fl = orc.topk_softmax(l, 2, 1.0)
    assert ids.tolist() == [[1, 2]]
    assert fl[0] & 1                       # 3rd-largest equals the 2nd: flagged
    assert np.allclose(w, [[0.5, 0.5]], atol=1e-15)


def test_tie_flag_threshold(orc):
    l = np.array([[3.0, 2.0, 2.0 - 5e-7, 0.0], [3.0, 2.0, 2.0 - 2e-6, 0.0]])
    ids, w, fl = orc.topk_softmax(l, 2, 1.0)
    assert fl[0] & 1 and not fl[1] & 1
    assert ids.tolist() == [[0, 1], [0, 1]]


def test_softmax_sums_to_router_scale_and_is_ordered(orc):
    rng = np.random.default_rng(11)
    l = rng.standard_normal((50, 128)) * 3
    for scale in (1.0, 0.37, 2.5):
        ids, w, fl = orc.topk_softmax(l, 8, scale)
        assert np.allclose(w.sum(1), scale, rtol=0, atol=1e-12 * scale)
        assert (w > 0).all()
        assert (np.diff(w, axis=1) <= 1e-15).all()          # ordered like the logits
        ref = scipy.special.softmax(np.take_along_axis(l, ids, 1), axis=1) * scale
        assert np.allclose(w, ref, rtol=1e-13, atol=0)


def test_k_equals_E_is_full_softmax(orc):
    rng = np.random.default_rng(12)
    l = rng.standard_normal((4, 16))
    ids, w, fl = orc.topk_softmax(l, 16, 1.0)
    full = scipy.special.softmax(l, axis=1)
    for t in range(4):
        assert sorted(ids[t].tolist()) == list(range(16))
        assert np.allclose(w[t], full[t, ids[t]], rtol=1e-13, atol=0)


# ------------------------------------------------------------------ permutation

def test_permutation_matches_stable_argsort(orc):
    rng = np.random.default_rng(13)
    for T, k, E in [(1, 8, 128), (33, 8, 128), (300, 2, 8), (7, 4, 4), (64, 1, 3)]:
        ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        counts, offsets, perm, inv = orc.permutation(ids, E)
        assert np.array_equal(perm, np.argsort(ids.ravel(), kind="stable"))
        assert np.array_equal(counts, np.bincount(ids.ravel(), minlength=E))
        assert offsets[0] == 0 and offsets[-1] == T * k
        assert np.array_equal(np.diff(offsets), counts)
        assert np.array_equal(inv[perm], np.arange(T * k))          # round trip
        assert np.array_equal(perm[inv], np.arange(T * k))
        for e in range(E):                                          # stable per expert
            rows = perm[offsets[e]:offsets[e + 1]]
            assert (np.diff(rows) > 0).all()
            assert (ids.ravel()[rows] == e).all()


# ------------------------------------------------------------------ experts + combine

def _tiny_layer(seed, E=6, d=64, f=32, d_lo=0.001, d_hi=0.004):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((E, d)) / np.sqrt(d)).astype(np.float32)
    gu = mi.random_q4_0(rng, 2 * f, d, d_lo, d_hi, lead=(E,))
    dn = mi.random_q4_0(rng, d, f, d_lo, d_hi, lead=(E,))
    es = rng.uniform(0.5, 1.5, E).astype(np.float32)
    return W, gu, dn, es


@pytest.mark.parametrize("E,d,f,k,T", [(6, 64, 32, 2, 5), (4, 32, 64, 4, 3), (8, 96, 64, 3, 4)])
def test_layer_matches_dense_brute_force(orc, E, d, f, k, T):
    # larger block scales so the expert outputs are far from zero
    W, gu, dn, es = _tiny_layer(100 + E, E, d, f, 0.05, 0.2)
    rng = np.random.default_rng(200 + E)
    x = mi.f32_to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    out, ids, w, fl = orc.moe_layer(x, W, 0.8, gu, dn, es, k)
    ref, ref_ids, _ = np_ref.dense_moe(x, W, 0.8, gu, dn, es, k)
    assert np.array_equal(ids, ref_ids)
    assert np.max(np.abs(out - ref)) <= 1e-12 * np.max(np.abs(ref))


def _const_q4(rows, cols, code, d_bits=0x2400):
    nb = cols // 32
    b = np.zeros((rows, nb, 18), dtype=np.uint8)
    b[..., 0] = d_bits & 0xFF
    b[..., 1] = d_bits >> 8
    b[..., 2:] = (code & 15) | ((code & 15) << 4)
    return b.reshape(rows, nb * 18)


def test_zero_codes_and_zero_input_give_zero(orc):
    E, d, f, k = 4, 64, 32, 2
    W, gu, dn, es = _tiny_layer(1, E, d, f)
    x = mi.f32_to_bf16_bits(np.random.default_rng(2).standard_normal((3, d)).astype(np.float32))
    zero_gu = np.stack([_const_q4(2 * f, d, 8)] * E)     # code 8 -> weight 0
    out, *_ = orc.moe_layer(x, W, 1.0, zero_gu, dn, es, k)
    assert (out == 0).all()
    out, *_ = orc.moe_layer(np.zeros_like(x), W, 1.0, gu, dn, es, k)
    assert (out == 0).all()


def test_constant_codes_closed_form_pins_gate_up_and_down_layout(orc):
    # All block scales 1/64 (fp16 0x2400). Gate rows code 9 -> weight 1/64,
    # up rows code 10 -> 2/64, so g = s, u = 2s with s = sum(x)/64 and
    # h = gelu(s) * 2s for every c. Down row r has code (r % 16), weight
    # (r % 16 - 8)/64, so y[r] = (r % 16 - 8)/64 * f * h. With identical experts,
    # expert scales 1 and router scale 1, out = y. Swapping gate and up would
    # give gelu(2s) * s instead.
    E, d, f, k = 4, 64, 32, 2
    gate = _const_q4(f, d, 9)
    up = _const_q4(f, d, 10)
    gu = np.stack([np.concatenate([gate, up])] * E)
    dn_rows = np.stack([_const_q4(1, f, r % 16)[0] for r in range(d)])
    dn = np.stack([dn_rows] * E)
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((E, d)) / 8).astype(np.float32)
    x = mi.f32_to_bf16_bits((rng.standard_normal((2, d)) * 0.5).astype(np.float32))
    out, *_ = orc.moe_layer(x, W, 1.0, gu, dn, np.ones(E, np.float32), k)
    xv = np_ref.bf16_field_decode(x)
    for t in range(2):
        s = xv[t].sum() / 64
        h = float(np_ref.gelu_tanh(s)) * 2 * s
        exp = np.array([(r % 16 - 8) / 64 * f * h for r in range(d)])
        assert np.allclose(out[t], exp, rtol=1e-13, atol=1e-300)
        swapped = float(np_ref.gelu_tanh(2 * s)) * s
        assert not np.isclose(h, swapped, rtol=1e-6)


def test_one_hot_router_reproduces_single_expert(orc):
    E, d, f = 8, 64, 32
    W, gu, dn, es = _tiny_layer(21, E, d, f, 0.05, 0.2)
    x = mi.f32_to_bf16_bits(np.random.default_rng(22).standard_normal((1, d)).astype(np.float32))
    e_star = 5
    W = W * 0.01
    W[e_star] = 1000.0 * np_ref.bf16_field_decode(x[0]).astype(np.float32)
    for scale in (1.0, 0.5):
        out, ids, w, fl = orc.moe_layer(x, W, scale, gu, dn, es, 1)
        assert ids[0, 0] == e_star and w[0, 0] == scale
        _, y = orc.expert_ffn(x[0], gu[e_star], dn[e_star], d, f)
        assert np.allclose(out[0], scale * es[e_star] * y, rtol=1e-15, atol=0)


def test_ffn_matches_numpy_decode_and_matmul(orc):
    E, d, f = 2, 96, 64
    W, gu, dn, es = _tiny_layer(31, E, d, f, 0.05, 0.2)
    x = mi.f32_to_bf16_bits(np.random.default_rng(32).standard_normal(d).astype(np.float32))
    h, y = orc.expert_ffn(x, gu[1], dn[1], d, f)
    Wg = np_ref.decode_q4_0(gu[1], d)
    Wd = np_ref.decode_q4_0(dn[1], f)
    xv = np_ref.bf16_field_decode(x)
    g, u = Wg[:f] @ xv, Wg[f:] @ xv
    # 1 + tanh(.) cancels for very negative gates: compare against the tensor's max
    h_ref = np_ref.gelu_tanh(g) * u
    y_ref = Wd @ h_ref
    assert np.max(np.abs(h - h_ref)) <= 1e-13 * np.max(np.abs(h_ref))
    assert np.max(np.abs(y - y_ref)) <= 1e-13 * np.max(np.abs(y_ref))


def test_results_do_not_depend_on_thread_count(orc):
    E, d, f, k, T = 8, 64, 32, 3, 9
    W, gu, dn, es = _tiny_layer(41, E, d, f)
    x = mi.f32_to_bf16_bits(np.random.default_rng(42).standard_normal((T, d)).astype(np.float32))
    n0 = orc.num_threads()
    try:
        orc.set_num_threads(1)
        a = orc.moe_layer(x, W, 1.0, gu, dn, es, k)[0]
        orc.set_num_threads(4)
        b = orc.moe_layer(x, W, 1.0, gu, dn, es, k)[0]
    finally:
        orc.set_num_threads(n0)
    assert np.array_equal(a, b)


# ------------------------------------------------------------------ RMSNorm + cast

def test_rmsnorm_hand_value_and_invariants(orc):
    # y = [3, 4]: mean square 12.5, eps 0 -> [3, 4] / sqrt(12.5)
    x = orc.rmsnorm_bf16(np.array([[3.0, 4.0]]), eps=0.0)
    vals = np_ref.bf16_field_decode(x[0])
    assert np.allclose(vals, [3 / math.sqrt(12.5), 4 / math.sqrt(12.5)], rtol=2 ** -8)
    # constant vector: every element rounds from c / sqrt(c^2 + eps)
    c = 0.25
    x = orc.rmsnorm_bf16(np.full((1, 64), c), eps=1e-6)
    assert (x == orc.double_to_bf16(c / math.sqrt(c * c + 1e-6))).all()
    # scale invariance (eps = 0): rmsnorm(a y) == rmsnorm(y) for a power of two
    y = np.random.default_rng(51).standard_normal((3, 128))
    assert np.array_equal(orc.rmsnorm_bf16(y, 0.0), orc.rmsnorm_bf16(8.0 * y, 0.0))
    # result has unit RMS up to bf16 rounding
    xv = np_ref.bf16_field_decode(orc.rmsnorm_bf16(y, 1e-6))
    assert np.allclose(np.sqrt((xv ** 2).mean(1)), 1.0, atol=3e-3)


def test_oracle_regression_fixture(orc):
    """Unchanged arithmetic: the oracle reproduces its own stored tiny-case output."""
    import os
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden"))
    import make_oracle_regression as mk
    rows = {}
    for line in open(mk.OUT):
        if line.startswith("#"):
            continue
        key, *vals = line.split()
        rows[key] = vals
    lw, x = mk.tiny_case()
    out, ids, w, fl = orc.moe_layer(x, lw.router_w, lw.router_scale, lw.gate_up, lw.down,
                                    lw.expert_scale, k=3)
    assert ids.ravel().tolist() == [int(v) for v in rows["ids"]]
    assert w.ravel().tolist() == [float(v) for v in rows["w"]]
    assert out.ravel().tolist() == [float(v) for v in rows["out"]]


# ------------------------------------------------------------------ the block's dense MLP

def test_dense_mlp_matches_numpy_decode_and_matmul(orc):
    """The dense MLP (gate rows first in the one [gate; up] parent, GELU-tanh GeGLU, down)
    against NumPy's float16 decode and matmuls, on every token and on a token subset."""
    d, fd, T = 96, 64, 5
    gu, dn = mi.make_dense(11, 0, d, fd)
    x = mi.make_tokens(12, T, d)
    got = orc.dense_mlp(x, gu, dn)
    xv = np_ref.bf16_field_decode(x)
    Wg = np_ref.decode_q4_0(gu, d)
    Wd = np_ref.decode_q4_0(dn, fd)
    ref = (np_ref.gelu_tanh(xv @ Wg[:fd].T) * (xv @ Wg[fd:].T)) @ Wd.T
    assert got.shape == (T, d)
    assert np.max(np.abs(got - ref)) <= 1e-13 * np.max(np.abs(ref))
    sub = orc.dense_mlp(x, gu, dn, tokens=np.array([4, 1]))
    assert np.array_equal(sub, got[[4, 1]])


def test_block_is_routed_layer_plus_dense_mlp(orc):
    """The block's output is the routed layer's plus the dense MLP's: zero dense weights (code
    8) leave the routed layer's bits, zero expert weights leave the dense MLP's, and in general
    the two add up (to FP64 rounding)."""
    E, d, f, fd, k, T = 6, 64, 32, 96, 2, 4
    W, gu, dn, es = _tiny_layer(51, E, d, f, 0.05, 0.2)
    gud, dnd = mi.make_dense(52, 0, d, fd)
    x = mi.make_tokens(53, T, d)
    routed, ids, w, fl = orc.moe_layer(x, W, 0.7, gu, dn, es, k)
    out, ids2, w2, fl2 = orc.block_ffn(x, W, 0.7, gu, dn, es, gud, dnd, k)
    assert np.array_equal(ids, ids2) and np.array_equal(w, w2)
    dense = orc.dense_mlp(x, gud, dnd)
    assert np.max(np.abs(out - (routed + dense))) <= 1e-14 * np.max(np.abs(out))
    zero_gud = _const_q4(2 * fd, d, 8)
    out0, *_ = orc.block_ffn(x, W, 0.7, gu, dn, es, zero_gud, dnd, k)
    assert np.array_equal(out0, routed)
    zero_gu = np.stack([_const_q4(2 * f, d, 8)] * E)
    out1, *_ = orc.block_ffn(x, W, 0.7, zero_gu, dn, es, gud, dnd, k)
    assert np.array_equal(out1, dense)
