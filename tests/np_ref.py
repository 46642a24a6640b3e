"""Independent NumPy restatements used to pin the oracle in tests.

These are written separately from the C oracle (vectorised NumPy, library
float16 / matmul / argsort / softmax) so that a slip in one does not repeat in
the other. They are test helpers only.
"""
from __future__ import annotations

import math

import numpy as np


def decode_q4_0(mat: np.ndarray, cols: int) -> np.ndarray:
    """[..., rows, cols/32*18] uint8 -> [..., rows, cols] float64 via numpy float16."""
    nb = cols // 32
    lead = mat.shape[:-1]
    b = np.ascontiguousarray(mat).reshape(lead + (nb, 18))
    d = b[..., 0:2].copy().view(np.float16).astype(np.float64)      # [..., nb, 1]
    qs = b[..., 2:18].astype(np.int64)
    vals = np.concatenate([(qs & 15) - 8, (qs >> 4) - 8], axis=-1) * d
    return vals.reshape(lead + (cols,))


def bf16_field_decode(bits: np.ndarray) -> np.ndarray:
    """bf16 bits -> float64 from the field definition (1 sign, 8 exponent, 7 mantissa)."""
    b = np.asarray(bits, dtype=np.int64)
    s = np.where((b >> 15) & 1, -1.0, 1.0)
    ex = (b >> 7) & 0xFF
    m = (b & 0x7F).astype(np.float64)
    normal = s * np.ldexp(1.0 + m / 128.0, (ex - 127).astype(np.int64))
    sub = s * np.ldexp(m / 128.0, -126)
    out = np.where(ex == 0, sub, normal)
    out = np.where((ex == 255) & (m == 0), s * np.inf, out)
    out = np.where((ex == 255) & (m != 0), np.nan, out)
    return out


def gelu_tanh(z):
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)))


def gelu_erf(z: float) -> float:
    return 0.5 * z * (1.0 + math.erf(z / math.sqrt(2.0)))


def topk_sorted(logits32: np.ndarray, k: int) -> np.ndarray:
    """Top-k by a stable sort on -logit (so equal values keep the lower index)."""
    order = np.argsort(-logits32.astype(np.float64), axis=-1, kind="stable")
    return order[..., :k]


def dense_moe(x_bits, router_w, router_scale, gate_up, down, expert_scale, k):
    """Every expert on every token, then a top-k mask: the dense formulation."""
    x = bf16_field_decode(x_bits)
    E, two_f, _ = gate_up.shape
    f = two_f // 2
    d = x.shape[1]
    Wg = decode_q4_0(gate_up, d)                   # [E, 2f, d]
    Wd = decode_q4_0(down, f)                      # [E, d, f]
    logits = x @ router_w.astype(np.float64).T     # [T, E]
    g = np.einsum("ecd,td->tec", Wg[:, :f], x)
    u = np.einsum("ecd,td->tec", Wg[:, f:], x)
    h = gelu_tanh(g) * u                           # [T, E, f]
    y = np.einsum("erc,tec->ter", Wd, h)           # [T, E, d]
    ids = topk_sorted(logits.astype(np.float32), k)
    T = x.shape[0]
    mask = np.zeros((T, E))
    for t in range(T):
        sel = logits[t, ids[t]]
        p = np.exp(sel - sel.max())
        p /= p.sum()
        mask[t, ids[t]] = float(router_scale) * p
    out = np.einsum("te,ter->tr", mask * expert_scale.astype(np.float64)[None, :], y)
    return out, ids, logits
