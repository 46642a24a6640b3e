"""The C ABI library without a GPU: it builds, loads, exports every declared symbol and
rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from mixture_experts_gemv_b200 import build
    build.build()
    import mixture_experts_gemv_b200 as moe
    return moe.lib()


def _declared():
    hdr = open(os.path.join(ROOT, "include", "moe.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", hdr)))


def test_exports_every_declared_symbol(L):
    import mixture_experts_gemv_b200 as moe
    names = _declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), f"libmoe.so does not export {n}"
    assert sorted(moe.EXPORTED) == names


def test_workspace_size_is_positive_and_monotone(L):
    a = L.moe_workspace_bytes(16, 2816, 704, 128, 8)
    b = L.moe_workspace_bytes(4096, 2816, 704, 128, 8)
    assert 0 < a < b
    assert L.moe_workspace_bytes(0, 2816, 704, 128, 8) == 0


@pytest.mark.parametrize("T,d,f,E,k", [(-1, 64, 32, 4, 2), (1, 48, 32, 4, 2), (1, 64, 40, 4, 2),
                                       (1, 64, 32, 0, 1), (1, 64, 32, 4, 5), (1, 64, 32, 4, 0),
                                       (1, 64, 32, 1024, 2)])
def test_bad_shapes_are_rejected_without_a_device(L, T, d, f, E, k):
    fake = ctypes.c_void_p(4096)
    rc = L.moe_layer_forward(fake, fake, fake, fake, fake, fake, T, d, f, E, k, fake, None)
    assert rc == -2
    assert len(L.moe_last_error()) > 0


def test_null_and_misaligned_pointers(L):
    fake = ctypes.c_void_p(4096)
    rc = L.moe_layer_forward(None, fake, fake, fake, fake, fake, 1, 64, 32, 4, 2, fake, None)
    assert rc == -2
    odd = ctypes.c_void_p(4096 + 2)
    rc = L.moe_layer_forward(fake, fake, fake, odd, fake, fake, 1, 64, 32, 4, 2, fake, None)
    assert rc == -3


def test_not_initialised(L):
    fake = ctypes.c_void_p(4096)
    L.moe_destroy()
    rc = L.moe_layer_forward(fake, fake, fake, fake, fake, fake, 1, 64, 32, 4, 2, fake, None)
    assert rc == -1
    assert L.moe_debug_check(None) == -1


def test_init_argument_checks(L):
    assert L.moe_init(0, 0, 64, 32, 4, 2) == -2
    assert L.moe_init(0, 8, 48, 32, 4, 2) == -2
    assert L.moe_init(0, 8, 64, 32, 4, 5) == -2
    assert L.moe_set_path(7, 16) == -2
    assert L.moe_set_path(0, 16) == 0


def test_init_without_a_gpu_fails_cleanly(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc = L.moe_init(0, 8, 64, 32, 4, 2)
    assert rc in (-4, -6)


def test_binding_raises(L):
    import mixture_experts_gemv_b200 as moe
    with pytest.raises(moe.MoeError):
        moe.moe_set_path(9)


def test_product_path_does_not_reference_the_oracle():
    pkg = os.path.join(ROOT, "mixture_experts_gemv_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, fn)).read()
                assert "oracle" not in src.lower(), f"{fn} mentions the oracle"
