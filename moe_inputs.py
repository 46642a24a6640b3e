"""Seeded synthetic inputs for the routed MoE layer.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark. It only draws random numbers and lays them out in the storage formats
the layer consumes; it holds none of the layer's arithmetic (no decode, no dot
products, no routing).

Storage formats (Gemma 4 26B-A4B NInfer v3 model card, "What is inside"):
  * routed expert weights are ggml Q4_0 blocks, expert-major:
      gate_up  uint8 [E][2f][d/32][18]   rows 0..f-1 = gate, f..2f-1 = up
      down     uint8 [E][d][f/32][18]
    one block = fp16 scale (2 bytes, little-endian) followed by 16 bytes of
    packed 4-bit codes;
  * router weights, router scale and per-expert scales are FP32;
  * activations x are bf16, carried here as their uint16 bit patterns.

Each tensor is drawn from its own generator, seeded with
``[config_seed, tensor_id, layer]`` (NumPy PCG64), so tensors do not depend on
the order in which they are generated.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field

import numpy as np

# Gemma-4-26B-A4B routed-expert shapes (model card, "What is inside").
D_MODEL = 2816
D_FF = 704
N_EXPERTS = 128
TOP_K = 8
Q4_0_BLOCK = 32
Q4_0_BYTES = 18

TENSOR_X = 0
TENSOR_ROUTER_W = 1
TENSOR_GATE_UP = 2
TENSOR_DOWN = 3
TENSOR_EXPERT_SCALE = 4
TENSOR_DENSE_GATE_UP = 5
TENSOR_DENSE_DOWN = 6
# Width of the block's dense MLP in the benchmark and full-size tests: the page stores its gate
# and up rows as one Q4_0 parent but gives no width; the one MLP width it gives for this
# block is a routed expert's, 704.
D_FF_DENSE = 704


def _rng(config_seed: int, tensor_id: int, layer: int = 0) -> np.random.Generator:
    return np.random.default_rng([int(config_seed), int(tensor_id), int(layer)])


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); uint16 bits.

    Used only to quantise freshly drawn inputs; both paths consume the bytes.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = (u + 0x7FFF + lsb) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def random_q4_0(rng: np.random.Generator, rows: int, cols: int,
                d_lo: float = 0.001, d_hi: float = 0.004,
                lead: tuple = ()) -> np.ndarray:
    """Random Q4_0 matrix bytes: shape lead + (rows, cols/32*18), uint8.

    Codes are uniform over 0..15 (uniform bytes give uniform nibbles in both
    halves); the fp16 block scale is drawn U(d_lo, d_hi) and rounded to fp16.
    """
    assert cols % Q4_0_BLOCK == 0
    nb = cols // Q4_0_BLOCK
    shape = tuple(lead) + (rows, nb)
    out = np.empty(shape + (Q4_0_BYTES,), dtype=np.uint8)
    scale = rng.uniform(d_lo, d_hi, size=shape).astype(np.float16)
    out[..., 0:2] = scale.view(np.uint8).reshape(shape + (2,))
    n = int(np.prod(shape)) * 16           # multiple of 8
    raw = rng.bit_generator.random_raw(n // 8).astype('<u8', copy=False)
    out[..., 2:18] = raw.view(np.uint8).reshape(shape + (16,))
    return out.reshape(tuple(lead) + (rows, nb * Q4_0_BYTES))


@dataclass
class LayerWeights:
    router_w: np.ndarray       # float32 [E, d]
    router_scale: np.ndarray   # float32 [1]
    gate_up: np.ndarray        # uint8 [E, 2f, d/32*18]
    down: np.ndarray           # uint8 [E, d, f/32*18]
    expert_scale: np.ndarray   # float32 [E]
    d: int = D_MODEL
    f: int = D_FF
    E: int = N_EXPERTS

    def nbytes_expert(self) -> int:
        return (self.gate_up.nbytes + self.down.nbytes) // self.E


def make_layer(seed: int = 0, layer: int = 0, d: int = D_MODEL, f: int = D_FF,
               E: int = N_EXPERTS, router_scale: float = 1.0) -> LayerWeights:
    """One layer of random weights with the model card's storage formats."""
    rw = _rng(seed, TENSOR_ROUTER_W, layer).standard_normal((E, d)) / np.sqrt(d)
    gu = random_q4_0(_rng(seed, TENSOR_GATE_UP, layer), 2 * f, d, lead=(E,))
    dn = random_q4_0(_rng(seed, TENSOR_DOWN, layer), d, f, lead=(E,))
    es = _rng(seed, TENSOR_EXPERT_SCALE, layer).uniform(0.5, 1.5, size=E)
    return LayerWeights(router_w=rw.astype(np.float32),
                        router_scale=np.array([router_scale], dtype=np.float32),
                        gate_up=gu, down=dn, expert_scale=es.astype(np.float32),
                        d=d, f=f, E=E)


def make_dense(seed: int = 0, layer: int = 0, d: int = D_MODEL, f_dense: int = D_FF_DENSE):
    """The block's dense MLP weights with the experts' recipe: (gate_up [2 f_dense, d/32*18],
    down [d, f_dense/32*18]) Q4_0 bytes, gate rows first in the one [gate; up] parent."""
    gu = random_q4_0(_rng(seed, TENSOR_DENSE_GATE_UP, layer), 2 * f_dense, d)
    dn = random_q4_0(_rng(seed, TENSOR_DENSE_DOWN, layer), d, f_dense)
    return gu, dn


def make_tokens(seed: int, T: int, d: int = D_MODEL) -> np.ndarray:
    """x [T, d] ~ N(0,1) as bf16 bits, all tokens from one seed."""
    x = _rng(seed, TENSOR_X, 0).standard_normal((T, d)).astype(np.float32)
    return f32_to_bf16_bits(x)


def make_tokens_per_seed(seeds, d: int = D_MODEL) -> np.ndarray:
    """x with token t drawn from its own seed seeds[t] (decode requests)."""
    rows = [_rng(s, TENSOR_X, 0).standard_normal(d).astype(np.float32) for s in seeds]
    return f32_to_bf16_bits(np.stack(rows))


def zipf_mean_one(E: int = N_EXPERTS, s: float = 1.1) -> np.ndarray:
    """z_e = E * (e+1)^-s / H, H = sum_{r=1..E} r^-s (mean-one Zipf pmf)."""
    r = np.arange(1, E + 1, dtype=np.float64)
    p = r ** (-s)
    return E * p / p.sum()


def apply_router_bias(lw: LayerWeights, x: np.ndarray, bias: np.ndarray) -> None:
    """Make the router logits carry +bias[e] through the plain router product.

    The last hidden coordinate of every token is set to exactly 1.0 and the
    router's last column to bias[e], so logit_e = sum_{i<d-1} W[e,i] x[i] + bias[e].
    """
    x[:, -1] = f32_to_bf16_bits(np.array([1.0], dtype=np.float32))[0]
    lw.router_w[:, -1] = bias.astype(np.float32)


@dataclass
class Workload:
    name: str
    x: np.ndarray                 # uint16 bf16 bits [T, d]
    layers: list = field(default_factory=list)   # list[LayerWeights]
    k: int = TOP_K

    @property
    def T(self) -> int:
        return int(self.x.shape[0])


# The layer's five workloads, named by what they are.
WORKLOADS = (
    "layer_T1",         # one token, x from seed 0
    "decode_T8",        # eight decode requests, token t from seed t (t = 1..8)
    "stack30_T1",       # 30 independent layers of the same shapes, one token
    "prefill_T4096",    # 4,096-token prefill, x from seed 3, unskewed router
    "skewed_T512",      # 512 tokens, x from seed 4, Zipf-biased router
    "prefill_T10000",   # 10,000-token prefill, x from seed 5 (a long prompt)
    "prefill_T40000",   # 40,000-token prefill, x from seed 6 (the longest prompt)
    "block_T8",         # decode_T8 through the routed experts plus the block's dense MLP
)


def make_layers(indices, seed: int = 0, threads: int = 8) -> list:
    """make_layer(seed, i) for every i of `indices`, drawn on a few threads at once (each
    layer has its own generators, so the bytes do not depend on the threading)."""
    idx = list(indices)
    if len(idx) <= 1 or threads <= 1:
        return [make_layer(seed, i) for i in idx]
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=min(threads, len(idx))) as ex:
        return list(ex.map(lambda i: make_layer(seed, i), idx))


def make_workload(name: str, n_layers: int | None = None, layer_fn=None) -> Workload:
    """Build one named workload; weights always come from seed 0 (layer i: [0, id, i]).

    skewed_T512 biases the router logits by 2.0 * z_e, z the mean-one
    Zipf(s = 1.1) pmf over expert ids (on a copy of the router weights).
    `layer_fn(i)`, when given, returns layer i of seed 0 (e.g. from a cache); it must
    return make_layer(0, i).
    """
    get = layer_fn if layer_fn is not None else (lambda i: make_layer(0, i))
    if name == "layer_T1":
        return Workload(name, make_tokens(0, 1), [get(0)])
    if name in ("decode_T8", "block_T8"):
        return Workload(name, make_tokens_per_seed(range(1, 9)), [get(0)])
    if name == "stack30_T1":
        L = 30 if n_layers is None else n_layers
        layers = [get(i) for i in range(L)] if layer_fn is not None else make_layers(range(L))
        return Workload(name, make_tokens(0, 1), layers)
    if name == "prefill_T4096":
        return Workload(name, make_tokens(3, 4096), [get(0)])
    if name == "prefill_T10000":
        return Workload(name, make_tokens(5, 10000), [get(0)])
    if name == "prefill_T40000":
        return Workload(name, make_tokens(6, 40000), [get(0)])
    if name == "skewed_T512":
        lw = get(0)
        lw = LayerWeights(router_w=lw.router_w.copy(), router_scale=lw.router_scale, gate_up=lw.gate_up,
                          down=lw.down, expert_scale=lw.expert_scale, d=lw.d, f=lw.f, E=lw.E)
        x = make_tokens(4, 512)
        apply_router_bias(lw, x, 2.0 * zipf_mean_one(lw.E, 1.1))
        return Workload(name, x, [lw])
    raise ValueError(f"unknown workload {name!r}")


def sha256(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()
