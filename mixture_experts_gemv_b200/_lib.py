"""ctypes binding of libmoe.so: same names as the C ABI in include/moe.h.

Argument marshalling only. Tensors are torch tensors (device memory and streams come from
PyTorch); their data pointers and the current CUDA stream are passed straight to the
library. The binding raises MoeError on any non-zero return, and fails loudly at import
of the library if libmoe.so has not been built: there is no other implementation.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

MOE_OK = 0
MOE_ERR_NOT_INIT = -1
MOE_ERR_BAD_ARG = -2
MOE_ERR_BAD_ALIGN = -3
MOE_ERR_CUDA = -4
MOE_ERR_DEVICE_TIMEOUT = -5
MOE_ERR_UNSUPPORTED_DEVICE = -6
MOE_PATH_AUTO = 0
MOE_PATH_GEMV = 1
MOE_PATH_GEMM = 2
MOE_PATH_GEMV_SPLIT = 3

# Every symbol include/moe.h declares.
EXPORTED = (
    "moe_init", "moe_layer_forward", "moe_rmsnorm_bf16", "moe_stack_forward", "moe_set_path",
    "moe_destroy", "moe_last_error", "moe_debug_get_routing", "moe_debug_get_hidden",
    "moe_debug_check", "moe_workspace_bytes", "moe_profile_begin", "moe_profile_end",
    "moe_layer_forward_static", "moe_profile_kernel_launches", "moe_layer_forward_static_check",
    "moe_debug_set_wait_ns", "moe_debug_inject", "moe_block_forward", "moe_route", "moe_experts_forward",
    "moe_gather_rows", "moe_combine_slots",
)
MOE_INJECT_NONE = 0
MOE_INJECT_SKIP_ROUTER_ARRIVAL = 1
PROF_GROUPS = ("route", "gateup_gemv", "down_gemv", "gateup_gemm", "down_gemm", "combine", "rmsnorm",
               "fused_decode")


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libmoe error {code}: {msg}")
        self.code = code


_lib = None
_p = ctypes.c_void_p
_i = ctypes.c_int


def lib():
    """Load libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m mixture_experts_gemv_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        L.moe_init.argtypes = [_i, _i, _i, _i, _i, _i]
        L.moe_init.restype = _i
        L.moe_layer_forward.argtypes = [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p, _p]
        L.moe_layer_forward.restype = _i
        L.moe_route.argtypes = [_p, _p, _p, _i, _i, _i, _i, _p, _p, _p]
        L.moe_route.restype = _i
        L.moe_experts_forward.argtypes = [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _p, _p]
        L.moe_experts_forward.restype = _i
        L.moe_gather_rows.argtypes = [_p, _p, _i, ctypes.c_size_t, _p, _p]
        L.moe_gather_rows.restype = _i
        L.moe_combine_slots.argtypes = [_p, _i, _i, _i, _p, _p]
        L.moe_combine_slots.restype = _i
        L.moe_block_forward.argtypes = [_p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p, _p]
        L.moe_block_forward.restype = _i
        L.moe_rmsnorm_bf16.argtypes = [_p, _p, _i, _i, ctypes.c_float, _p]
        L.moe_rmsnorm_bf16.restype = _i
        L.moe_stack_forward.argtypes = [_p, _i, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i,
                                        ctypes.c_float, _p, _p, _p]
        L.moe_stack_forward.restype = _i
        L.moe_set_path.argtypes = [_i, _i]
        L.moe_set_path.restype = _i
        L.moe_destroy.argtypes = []
        L.moe_destroy.restype = None
        L.moe_last_error.argtypes = []
        L.moe_last_error.restype = ctypes.c_char_p
        L.moe_debug_get_routing.argtypes = [_p, _p, _p, _p, _p, _p]
        L.moe_debug_get_routing.restype = _i
        L.moe_debug_get_hidden.argtypes = [_p, _p]
        L.moe_debug_get_hidden.restype = _i
        L.moe_debug_check.argtypes = [_p]
        L.moe_debug_check.restype = _i
        L.moe_profile_begin.argtypes = []
        L.moe_profile_begin.restype = _i
        L.moe_profile_end.argtypes = [_p, _p]
        L.moe_profile_end.restype = _i
        L.moe_layer_forward_static.argtypes = [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p, _p]
        L.moe_layer_forward_static.restype = _i
        L.moe_layer_forward_static_check.argtypes = [_p]
        L.moe_layer_forward_static_check.restype = _i
        L.moe_debug_set_wait_ns.argtypes = [ctypes.c_ulonglong]
        L.moe_debug_set_wait_ns.restype = _i
        L.moe_debug_inject.argtypes = [_i]
        L.moe_debug_inject.restype = _i
        L.moe_profile_kernel_launches.argtypes = []
        L.moe_profile_kernel_launches.restype = ctypes.c_longlong
        L.moe_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
        L.moe_workspace_bytes.restype = ctypes.c_size_t
        _lib = L
    return _lib


def _check(rc: int) -> int:
    if rc != MOE_OK:
        raise MoeError(rc, lib().moe_last_error().decode(errors="replace"))
    return rc


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def moe_init(device: int, max_tokens: int, max_d: int, max_f: int, max_E: int, max_k: int) -> None:
    _check(lib().moe_init(device, max_tokens, max_d, max_f, max_E, max_k))


def moe_layer_forward(x, router_w, router_scale, gate_up_q4, down_q4, expert_scale,
                      T: int, d: int, f: int, E: int, k: int, out, stream=None) -> None:
    _check(lib().moe_layer_forward(_ptr(x), _ptr(router_w), _ptr(router_scale), _ptr(gate_up_q4),
                                   _ptr(down_q4), _ptr(expert_scale), T, d, f, E, k, _ptr(out),
                                   _stream(stream)))


def moe_block_forward(x, router_w, router_scale, gate_up_q4, down_q4, expert_scale, gate_up_dense_q4,
                      down_dense_q4, T: int, d: int, f: int, f_dense: int, E: int, k: int, out, stream=None) -> None:
    _check(lib().moe_block_forward(_ptr(x), _ptr(router_w), _ptr(router_scale), _ptr(gate_up_q4),
                                   _ptr(down_q4), _ptr(expert_scale), _ptr(gate_up_dense_q4),
                                   _ptr(down_dense_q4), T, d, f, f_dense, E, k, _ptr(out), _stream(stream)))


def moe_route(x, router_w, router_scale, T: int, d: int, E: int, k: int, ids, w, stream=None) -> None:
    _check(lib().moe_route(_ptr(x), _ptr(router_w), _ptr(router_scale), T, d, E, k, _ptr(ids), _ptr(w),
                           _stream(stream)))


def moe_experts_forward(x_rows, row_expert, row_weight, gate_up_q4, down_q4, expert_scale, R: int, d: int,
                        f: int, E: int, out_rows, stream=None) -> None:
    _check(lib().moe_experts_forward(_ptr(x_rows), _ptr(row_expert), _ptr(row_weight), _ptr(gate_up_q4),
                                     _ptr(down_q4), _ptr(expert_scale), R, d, f, E, _ptr(out_rows),
                                     _stream(stream)))


def moe_gather_rows(src, index, n: int, row_bytes: int, dst, stream=None) -> None:
    _check(lib().moe_gather_rows(_ptr(src), _ptr(index), n, row_bytes, _ptr(dst), _stream(stream)))


def moe_combine_slots(y_slots, T: int, d: int, k: int, out, stream=None) -> None:
    _check(lib().moe_combine_slots(_ptr(y_slots), T, d, k, _ptr(out), _stream(stream)))


def moe_rmsnorm_bf16(y, x_out, T: int, d: int, eps: float, stream=None) -> None:
    _check(lib().moe_rmsnorm_bf16(_ptr(y), _ptr(x_out), T, d, eps, _stream(stream)))


def _ptr_array(ts):
    arr = (ctypes.c_void_p * len(ts))(*[_ptr(t) for t in ts])
    return arr


def moe_stack_forward(x_in, router_w, router_scale, gate_up_q4, down_q4, expert_scale,
                      T: int, d: int, f: int, E: int, k: int, eps: float, out, x_trace=None,
                      stream=None) -> None:
    """router_w ... expert_scale are sequences of per-layer tensors (length L)."""
    L = len(router_w)
    keep = [_ptr_array(v) for v in (router_w, router_scale, gate_up_q4, down_q4, expert_scale)]
    _check(lib().moe_stack_forward(_ptr(x_in), L, *[ctypes.cast(a, _p) for a in keep], T, d, f, E, k,
                                   eps, _ptr(out), _ptr(x_trace), _stream(stream)))


def moe_set_path(path: int, gemv_max_tokens: int = 16) -> None:
    _check(lib().moe_set_path(path, gemv_max_tokens))


def moe_destroy() -> None:
    lib().moe_destroy()


def moe_last_error() -> str:
    return lib().moe_last_error().decode(errors="replace")


def moe_debug_get_routing(ids=None, w=None, counts=None, offsets=None, perm=None, stream=None) -> None:
    _check(lib().moe_debug_get_routing(_ptr(ids), _ptr(w), _ptr(counts), _ptr(offsets), _ptr(perm),
                                       _stream(stream)))


def moe_debug_get_hidden(h, stream=None) -> None:
    _check(lib().moe_debug_get_hidden(_ptr(h), _stream(stream)))


def moe_debug_check(stream=None) -> None:
    _check(lib().moe_debug_check(_stream(stream)))


def moe_workspace_bytes(max_tokens: int, max_d: int, max_f: int, max_E: int, max_k: int) -> int:
    return int(lib().moe_workspace_bytes(max_tokens, max_d, max_f, max_E, max_k))


def moe_profile_begin() -> None:
    _check(lib().moe_profile_begin())


def moe_profile_end() -> dict:
    """{group name: (total ms, launches)} for the groups that ran."""
    ms = (ctypes.c_float * 8)()
    n = (ctypes.c_int * 8)()
    _check(lib().moe_profile_end(ms, n))
    return {PROF_GROUPS[i]: (float(ms[i]), int(n[i])) for i in range(8) if n[i] > 0}


def moe_profile_kernel_launches() -> int:
    """Kernels launched (or captured) since moe_profile_begin."""
    return int(lib().moe_profile_kernel_launches())


def moe_layer_forward_static(x, router_w, router_scale, gate_up_q4, down_q4, expert_scale,
                             T: int, d: int, f: int, E: int, k: int, out, stream=None) -> None:
    """Decode path with a fixed static device scratch: no workspace, no allocation."""
    _check(lib().moe_layer_forward_static(_ptr(x), _ptr(router_w), _ptr(router_scale),
                                          _ptr(gate_up_q4), _ptr(down_q4), _ptr(expert_scale),
                                          T, d, f, E, k, _ptr(out), _stream(stream)))


def moe_layer_forward_static_check(stream=None) -> None:
    """Raise MoeError(MOE_ERR_DEVICE_TIMEOUT) if a static-entry call timed out since the last check."""
    _check(lib().moe_layer_forward_static_check(_stream(stream)))


def moe_debug_set_wait_ns(ns: int) -> None:
    _check(lib().moe_debug_set_wait_ns(int(ns)))


def moe_debug_inject(fault: int) -> None:
    _check(lib().moe_debug_inject(int(fault)))
