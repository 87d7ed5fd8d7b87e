"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/moe.h declares, and rejects bad arguments before
touching the device."""
import ctypes
import os
import re

import pytest

import mxfp4_latent_moe_router_b200 as moe
from mxfp4_latent_moe_router_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.load_library()


def _declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)
    return names


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert set(moe.ABI_SYMBOLS) <= set(declared)
    for n in declared:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in range(8):
        assert moe.moe_status_str(code)
    assert "invalid" in moe.moe_status_str(1)


def test_bad_config_rejected_on_host(lib):
    h = ctypes.c_void_p()
    assert lib.moe_plan_create(None, 0, ctypes.byref(h)) == 1
    cfg = moe.moe_config(100, 256, 16, 2, 128, 256, 1, 0, 1, 1.0)  # H not a multiple of 32
    assert lib.moe_plan_create(ctypes.byref(cfg), 0, ctypes.byref(h)) == 1
    cfg = moe.moe_config(512, 256, 16, 17, 128, 256, 1, 0, 1, 1.0)  # k > E
    assert lib.moe_plan_create(ctypes.byref(cfg), 0, ctypes.byref(h)) == 1
    cfg = moe.moe_config(512, 256, 2048, 2, 128, 256, 1, 0, 1, 1.0)  # E beyond the limit
    assert lib.moe_plan_create(ctypes.byref(cfg), 0, ctypes.byref(h)) == 2
    cfg = moe.moe_config(512, 256, 16, 2, 128, 256, 256, 0, 1, 1.0)  # B beyond the limit
    assert lib.moe_plan_create(ctypes.byref(cfg), 0, ctypes.byref(h)) == 2


def test_null_plan_calls(lib):
    assert lib.moe_forward(None, None, 1, None, None) == 1
    assert lib.moe_sync_status(None) == 1
    assert lib.moe_set_next_layer(None, None, 0) == 1
    assert lib.moe_set_next_layer(None, None, 1 << 20) == 1
    lib.moe_plan_destroy(None)


def test_no_device_means_no_fallback(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    h = ctypes.c_void_p()
    cfg = moe.moe_config(512, 256, 16, 2, 128, 256, 1, 0, 1, 1.0)
    assert lib.moe_plan_create(ctypes.byref(cfg), 0, ctypes.byref(h)) == 2
