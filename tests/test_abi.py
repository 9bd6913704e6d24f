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


def test_plain_c_program_compiles_links_and_calls_the_abi(tmp_path):
    """The public header is plain C: a C99 program includes it, links against
    the library and calls the entry points that need no device (argument
    checks, status strings)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "quantized_expert_ffn_token_b200")
    src = tmp_path / "use_abi.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "moe.h"
int main(void) {
    moe_ctx *ctx = 0;
    moe_config c;
    memset(&c, 0, sizeof c);
    if (moe_create(0, 0, &ctx) != MOE_ERR_INVALID_ARG) return 1;
    c.fmt = (moe_qformat)9;
    if (moe_create(&c, 0, &ctx) != MOE_ERR_INVALID_ARG || ctx != 0) return 2;
    if (moe_forward(0, 0, 0, 1, 0, 0, 0, 0, 0) != MOE_ERR_INVALID_ARG) return 3;
    if (moe_destroy(0) != MOE_OK) return 4;
    printf("%s\n", moe_status_string(MOE_ERR_NOT_LOADED));
    return 0;
}
''')
    exe = tmp_path / "use_abi"
    subprocess.check_call([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(root, "include"),
                           "-o", str(exe), str(src), "-L", pkg, "-lqeffn", "-Wl,-rpath," + pkg])
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert r.stdout.strip() == "layer not loaded"
