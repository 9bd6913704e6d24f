"""A fresh checkout builds: the tracked sources, copied without any built
library, compile through ``__graft_entry__.build()`` (nvcc for sm_100a and gcc
for the oracle, no GPU needed) and the package then imports."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_fresh_checkout_builds_and_imports(tmp_path):
    if not (shutil.which("nvcc") or os.path.exists("/usr/local/cuda/bin/nvcc")):
        pytest.skip("nvcc not available")
    if shutil.which("git") is None or subprocess.run(
            ["git", "rev-parse", "--is-inside-work-tree"], cwd=ROOT, capture_output=True).returncode != 0:
        pytest.skip("not a git checkout")
    files = subprocess.check_output(["git", "ls-files"], cwd=ROOT, text=True).split("\n")
    for f in files:
        if not f or not os.path.isfile(os.path.join(ROOT, f)):
            continue
        dst = tmp_path / f
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy2(os.path.join(ROOT, f), dst)
    assert not (tmp_path / "quantized_expert_ffn_token_b200" / "libqeffn.so").exists()
    r = subprocess.run([sys.executable, "-c",
                        "import __graft_entry__ as g; g.build(); "
                        "import quantized_expert_ffn_token_b200.capi as c; print(c.LIB_PATH)"],
                       cwd=tmp_path, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stderr[-2000:]
    assert os.path.samefile(r.stdout.strip().splitlines()[-1],
                            tmp_path / "quantized_expert_ffn_token_b200" / "libqeffn.so")
