"""The C-ABI library loads on a machine without a GPU, exports every entry
point include/moe.h declares, and rejects bad arguments before touching the
device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("moe_create", "moe_load_layer", "moe_forward", "moe_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from quantized_expert_ffn_token_b200 import capi
    out = subprocess.check_output(["nm", "-D", "--defined-only", capi.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in _declared():
        assert n in exported, n
        assert hasattr(capi.lib, n)
    assert sorted(capi.EXPORTED) == sorted(_declared())
    # nothing else of the library leaks out as a dynamic symbol
    ours = {s for s in exported if "qeffn" in s or s.startswith("moe_")}
    assert ours == set(_declared())


def test_argument_checks_need_no_device():
    from quantized_expert_ffn_token_b200 import capi
    h = ctypes.c_void_p()
    assert capi.lib.moe_create(None, 0, ctypes.byref(h)) == capi.MOE_ERR_INVALID_ARG
    c = capi.moe_config(256, 16, 128, 2, 1, 128, 1, 8, 9, 0, 0)      # fmt 9 does not exist
    assert capi.lib.moe_create(ctypes.byref(c), 0, ctypes.byref(h)) == capi.MOE_ERR_INVALID_ARG
    c = capi.moe_config(250, 16, 128, 2, 1, 128, 1, 8, capi.MOE_Q4B32, 0, 0)   # d not a multiple of 256
    assert capi.lib.moe_create(ctypes.byref(c), 0, ctypes.byref(h)) == capi.MOE_ERR_UNSUPPORTED
    c = capi.moe_config(256, 16, 128, 17, 1, 128, 1, 8, capi.MOE_Q4B32, 0, 0)  # k > E
    assert capi.lib.moe_create(ctypes.byref(c), 0, ctypes.byref(h)) == capi.MOE_ERR_INVALID_ARG
    assert capi.lib.moe_forward(None, 0, None, 1, None, None, None, None, None) == capi.MOE_ERR_INVALID_ARG
    assert capi.lib.moe_destroy(None) == capi.MOE_OK
    assert capi.status_string(capi.MOE_ERR_NOT_LOADED) == "layer not loaded"
