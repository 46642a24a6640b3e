"""Seeded input generator: determinism, the page's storage facts, the skew recipe."""
import os

import numpy as np
import pytest

import moe_inputs as mi
import np_ref

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _facts():
    facts = {}
    for line in open(os.path.join(GOLDEN, "model_card_shapes.txt")):
        line = line.split("#")[0].strip()
        if line:
            key, val = line.split()
            facts[key] = int(val) if val.isdigit() else val
    return facts


def test_generator_matches_model_card_storage_facts():
    f = _facts()
    assert mi.N_EXPERTS == f["experts_per_block"]
    assert 2 * mi.D_FF == f["gate_up_rows"] and mi.D_FF == f["gate_rows"]
    assert mi.D_MODEL == f["down_rows"]
    assert mi.Q4_0_BLOCK == f["q4_0_weights_per_block"]
    assert mi.Q4_0_BYTES == f["q4_0_bytes_per_block"]
    lw = mi.make_layer(0, 0, d=256, f=64, E=4)
    assert lw.gate_up.shape == (4, 128, 256 // 32 * 18)
    assert lw.down.shape == (4, 256, 64 // 32 * 18)
    assert lw.router_w.dtype == np.float32 and lw.expert_scale.dtype == np.float32
    # full-size per-expert bytes: [gate; up] 1408 x 88 blocks, down 2816 x 22 blocks
    assert f["gate_up_rows"] * (mi.D_MODEL // 32) * 18 == 2_230_272
    assert f["down_rows"] * (mi.D_FF // 32) * 18 == 1_115_136


def test_generator_is_deterministic_and_order_free():
    a = mi.make_layer(3, 2, d=128, f=64, E=4)
    b = mi.make_layer(3, 2, d=128, f=64, E=4)
    for name in ("router_w", "gate_up", "down", "expert_scale"):
        assert mi.sha256(getattr(a, name)) == mi.sha256(getattr(b, name))
    c = mi.make_layer(3, 3, d=128, f=64, E=4)
    assert mi.sha256(a.gate_up) != mi.sha256(c.gate_up)
    assert np.array_equal(mi.make_tokens(5, 4, 128), mi.make_tokens(5, 4, 128))


def test_q4_0_scale_range_and_code_uniformity():
    rng = np.random.default_rng(0)
    q = mi.random_q4_0(rng, 256, 1024)
    blocks = q.reshape(-1, 18)
    d = blocks[:, 0:2].copy().view(np.float16).astype(np.float64)
    assert d.min() >= 0.001 - 2e-6 and d.max() <= 0.004 + 2e-6     # fp16 half-ulp
    codes = np.concatenate([blocks[:, 2:] & 15, blocks[:, 2:] >> 4]).ravel()
    hist = np.bincount(codes, minlength=16)
    assert hist.min() > 0.9 * hist.mean()


def test_bf16_input_rounding_is_nearest_even():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -3.14159], dtype=np.float32)
    bits = mi.f32_to_bf16_bits(v)
    assert bits.tolist()[:3] == [0x3F80, 0x3F80, 0x3F82]
    back = np_ref.bf16_field_decode(bits)
    assert abs(back[3] + 3.14159) <= 2 ** -8 * 4


def test_decode_requests_use_one_seed_each():
    x = mi.make_tokens_per_seed([1, 2, 3], d=64)
    assert np.array_equal(x[1], mi.make_tokens_per_seed([2], d=64)[0])


def test_zipf_reading_gives_few_hot_many_cold_experts(orc):
    """skewed_T512: a few experts above 100 tokens, many with 0-2 (oracle routing)."""
    wl = mi.make_workload("skewed_T512")
    lw = wl.layers[0]
    logits = orc.router_logits(wl.x, lw.router_w)
    ids, w, fl = orc.topk_softmax(logits, wl.k, 1.0)
    counts = np.bincount(ids.ravel(), minlength=lw.E)
    assert (counts > 100).sum() >= 3
    assert (counts <= 2).sum() >= 64
    assert counts.sum() == wl.T * wl.k
