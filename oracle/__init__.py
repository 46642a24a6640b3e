"""ctypes wrapper around the FP64 CPU oracle (moe_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and the
benchmark's CPU-baseline leg, never by the CUDA library or its binding.

Every function takes and returns NumPy arrays; bf16 activations travel as their
uint16 bit patterns and Q4_0 weights as raw bytes, exactly as the CUDA path
receives them.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build_oracle, LIB_PATH

_lib = None

_p = ctypes.c_void_p
_i = ctypes.c_int
_d = ctypes.c_double


def lib():
    global _lib
    if _lib is None:
        path = os.environ.get("MOE_ORACLE_LIB", LIB_PATH)   # a planted-mistake copy in tests
        if path == LIB_PATH:
            build_oracle()
        L = ctypes.CDLL(path)
        L.oracle_fp16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_fp16_to_double.restype = _d
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_double.restype = _d
        L.oracle_double_to_bf16_rne.argtypes = [_d]
        L.oracle_double_to_bf16_rne.restype = ctypes.c_uint16
        L.oracle_gelu_tanh.argtypes = [_d]
        L.oracle_gelu_tanh.restype = _d
        L.oracle_q4_0_decode_block.argtypes = [_p, _p]
        L.oracle_q4_0_decode_block.restype = None
        L.oracle_router_logits.argtypes = [_p, _p, _i, _i, _i, _p]
        L.oracle_router_logits.restype = None
        L.oracle_topk_softmax.argtypes = [_p, _i, _i, _i, _d, _d, _p, _p, _p]
        L.oracle_topk_softmax.restype = None
        L.oracle_permutation.argtypes = [_p, _i, _i, _i, _p, _p, _p, _p]
        L.oracle_permutation.restype = None
        L.oracle_expert_ffn.argtypes = [_p, _p, _p, _i, _i, _p, _p]
        L.oracle_expert_ffn.restype = None
        L.oracle_experts_combine.argtypes = [_p, _p, _p, _p, _p, _p, _i, _i, _i, _p, _i, _p, _p]
        L.oracle_experts_combine.restype = None
        L.oracle_moe_layer.argtypes = [_p, _p, _d, _p, _p, _p, _i, _i, _i, _i, _i, _d,
                                       _p, _p, _p, _p]
        L.oracle_moe_layer.restype = _i
        L.oracle_dense_mlp.argtypes = [_p, _p, _p, _i, _i, _p, _i, _p]
        L.oracle_dense_mlp.restype = None
        L.oracle_block_ffn.argtypes = [_p, _p, _d, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _d,
                                       _p, _p, _p, _p]
        L.oracle_block_ffn.restype = _i
        L.oracle_rmsnorm_bf16.argtypes = [_p, _i, _i, _d, _p]
        L.oracle_rmsnorm_bf16.restype = None
        L.oracle_num_threads.argtypes = []
        L.oracle_num_threads.restype = _i
        L.oracle_set_num_threads.argtypes = [_i]
        L.oracle_set_num_threads.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


TIE_EPS = 1e-6


def fp16_to_double(bits: int) -> float:
    return lib().oracle_fp16_to_double(int(bits))


def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(int(bits))


def double_to_bf16(v: float) -> int:
    return int(lib().oracle_double_to_bf16_rne(float(v)))


def gelu_tanh(z: float) -> float:
    return lib().oracle_gelu_tanh(float(z))


def q4_0_decode_block(blk) -> np.ndarray:
    b = _c(np.asarray(blk, dtype=np.uint8).reshape(18), np.uint8)
    out = np.empty(32, dtype=np.float64)
    lib().oracle_q4_0_decode_block(_ptr(b), _ptr(out))
    return out


def router_logits(x_bits, router_w) -> np.ndarray:
    x = _c(x_bits, np.uint16)
    W = _c(router_w, np.float32)
    T, d = x.shape
    E = W.shape[0]
    out = np.empty((T, E), dtype=np.float64)
    lib().oracle_router_logits(_ptr(x), _ptr(W), T, d, E, _ptr(out))
    return out


def topk_softmax(logits, k: int, router_scale: float, tie_eps: float = TIE_EPS):
    l = _c(logits, np.float64)
    T, E = l.shape
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    flags = np.empty(T, dtype=np.uint8)
    lib().oracle_topk_softmax(_ptr(l), T, E, k, float(router_scale), float(tie_eps),
                              _ptr(ids), _ptr(w), _ptr(flags))
    return ids, w, flags


def permutation(ids, E: int):
    i = _c(ids, np.int32)
    T, k = i.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    perm = np.empty(T * k, dtype=np.int32)
    inv = np.empty(T * k, dtype=np.int32)
    lib().oracle_permutation(_ptr(i), T, k, E, _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv))
    return counts, offsets, perm, inv


def expert_ffn(x_row_bits, gate_up_e, down_e, d: int, f: int):
    x = _c(x_row_bits, np.uint16).reshape(d)
    gu = _c(gate_up_e, np.uint8)
    dn = _c(down_e, np.uint8)
    h = np.empty(f, dtype=np.float64)
    y = np.empty(d, dtype=np.float64)
    lib().oracle_expert_ffn(_ptr(x), _ptr(gu), _ptr(dn), d, f, _ptr(h), _ptr(y))
    return h, y


def experts_combine(x_bits, gate_up, down, expert_scale, ids, w, d: int, f: int,
                    tokens=None, want_h: bool = False):
    x = _c(x_bits, np.uint16)
    ids_ = _c(ids, np.int32)
    w_ = _c(w, np.float64)
    k = ids_.shape[1]
    tok = _c(np.arange(x.shape[0]) if tokens is None else tokens, np.int32)
    n = tok.shape[0]
    out = np.empty((n, d), dtype=np.float64)
    h = np.empty((n, k, f), dtype=np.float64) if want_h else None
    lib().oracle_experts_combine(_ptr(x), _ptr(_c(gate_up, np.uint8)), _ptr(_c(down, np.uint8)),
                                 _ptr(_c(expert_scale, np.float32)), _ptr(ids_), _ptr(w_),
                                 d, f, k, _ptr(tok), n, _ptr(out),
                                 _ptr(h) if want_h else None)
    return (out, h) if want_h else out


def moe_layer(x_bits, router_w, router_scale, gate_up, down, expert_scale, k: int,
              tie_eps: float = TIE_EPS):
    """Full layer for all tokens: (out [T,d] f64, ids [T,k], w [T,k] f64, flags [T])."""
    x = _c(x_bits, np.uint16)
    T, d = x.shape
    W = _c(router_w, np.float32)
    E = W.shape[0]
    gu = _c(gate_up, np.uint8)
    f = gu.shape[1] // 2
    out = np.empty((T, d), dtype=np.float64)
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    flags = np.empty(T, dtype=np.uint8)
    lib().oracle_moe_layer(_ptr(x), _ptr(W), float(np.asarray(router_scale).reshape(-1)[0]),
                           _ptr(gu), _ptr(_c(down, np.uint8)),
                           _ptr(_c(expert_scale, np.float32)), T, d, f, E, k, float(tie_eps),
                           _ptr(out), _ptr(ids), _ptr(w), _ptr(flags))
    return out, ids, w, flags


def dense_mlp(x_bits, gate_up_dense, down_dense, tokens=None):
    """The block's dense MLP (GELU-tanh GeGLU of width f_dense) on the given tokens: [n, d] f64."""
    x = _c(x_bits, np.uint16)
    T, d = x.shape
    gu = _c(gate_up_dense, np.uint8)
    f_dense = gu.shape[0] // 2
    tok = _c(np.arange(T) if tokens is None else tokens, np.int32)
    out = np.empty((tok.shape[0], d), dtype=np.float64)
    lib().oracle_dense_mlp(_ptr(x), _ptr(gu), _ptr(_c(down_dense, np.uint8)), d, f_dense, _ptr(tok),
                           tok.shape[0], _ptr(out))
    return out


def block_ffn(x_bits, router_w, router_scale, gate_up, down, expert_scale, gate_up_dense, down_dense, k: int,
              tie_eps: float = TIE_EPS):
    """Routed layer plus dense MLP for all tokens: (out [T,d] f64, ids, w, flags)."""
    x = _c(x_bits, np.uint16)
    T, d = x.shape
    W = _c(router_w, np.float32)
    E = W.shape[0]
    gu = _c(gate_up, np.uint8)
    f = gu.shape[1] // 2
    gud = _c(gate_up_dense, np.uint8)
    f_dense = gud.shape[0] // 2
    out = np.empty((T, d), dtype=np.float64)
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    flags = np.empty(T, dtype=np.uint8)
    lib().oracle_block_ffn(_ptr(x), _ptr(W), float(np.asarray(router_scale).reshape(-1)[0]), _ptr(gu),
                           _ptr(_c(down, np.uint8)), _ptr(_c(expert_scale, np.float32)), _ptr(gud),
                           _ptr(_c(down_dense, np.uint8)), T, d, f, f_dense, E, k, float(tie_eps),
                           _ptr(out), _ptr(ids), _ptr(w), _ptr(flags))
    return out, ids, w, flags


def rmsnorm_bf16(y, eps: float = 1e-6) -> np.ndarray:
    yy = _c(y, np.float64)
    T, d = yy.shape
    out = np.empty((T, d), dtype=np.uint16)
    lib().oracle_rmsnorm_bf16(_ptr(yy), T, d, float(eps), _ptr(out))
    return out


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))
