"""Host logic of the token-count sweep (``bench.py --sweep``): which paths a
token count can run on, the library's default choice, and the summary that
compares them."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from quantized_expert_ffn_token_b200 import capi  # noqa: E402


def test_flags_match_the_binding():
    assert bench.sweep_flags("single-token kernel") == capi.MOE_FLAG_NO_MULTI_DECODE
    assert bench.sweep_flags("few-token kernel") == 0
    assert bench.sweep_flags("cuda-core") == capi.MOE_FLAG_NO_DECODE_KERNEL | capi.MOE_FLAG_NO_TENSOR_PREFILL
    assert bench.sweep_flags("tensor-core") == capi.MOE_FLAG_NO_DECODE_KERNEL


@pytest.mark.parametrize("T, paths, default", [
    (1, {"single-token kernel", "cuda-core"}, "single-token kernel"),
    (2, {"single-token kernel", "few-token kernel", "cuda-core"}, "few-token kernel"),
    (8, {"single-token kernel", "few-token kernel", "cuda-core"}, "few-token kernel"),
    (9, {"few-token kernel", "cuda-core", "tensor-core"}, "few-token kernel"),
    (16, {"few-token kernel", "cuda-core", "tensor-core"}, "few-token kernel"),
    (17, {"few-token kernel", "cuda-core", "tensor-core"}, "few-token kernel"),
    (32, {"few-token kernel", "cuda-core", "tensor-core"}, "few-token kernel"),
    (33, {"cuda-core", "tensor-core"}, "tensor-core"),
    (8192, {"cuda-core", "tensor-core"}, "tensor-core"),
])
def test_eligible_paths_and_default(T, paths, default):
    assert {p for p in bench.SWEEP_PATHS if bench.sweep_eligible(p, T)} == paths
    assert bench.default_path(T) == default
    assert bench.sweep_eligible(default, T)   # the default is always among the timed paths


def test_summary_names_the_fastest_path_and_checks_the_default():
    rows = [{"T": 8, "path": "few-token kernel", "ms": 0.20},
            {"T": 8, "path": "cuda-core", "ms": 0.15},
            {"T": 128, "path": "cuda-core", "ms": 1.0},
            {"T": 128, "path": "tensor-core", "ms": 0.4},
            {"T": 64, "path": "tensor-core", "ms": 0.3}]
    s = {r["T"]: r for r in bench.sweep_summary(rows)}
    assert [r["T"] for r in bench.sweep_summary(rows)] == [8, 64, 128]
    assert s[8]["fastest"] == "cuda-core" and not s[8]["default_is_fastest"] and s[8]["default_ms"] == 0.20
    assert s[64]["fastest"] == "tensor-core" and s[64]["default_is_fastest"]
    assert s[128]["fastest"] == "tensor-core" and s[128]["default_is_fastest"] and s[128]["fastest_ms"] == 0.4


def test_sweep_token_counts_straddle_the_thresholds():
    Ts = set(bench.SWEEP_T) | {17}
    for t in (1, 2, bench.DISPATCH_SINGLE_MAX, bench.DISPATCH_SINGLE_MAX + 1, bench.DISPATCH_TC_MIN,
              bench.DISPATCH_FEW_MAX, bench.DISPATCH_FEW_MAX + 1):
        assert t in Ts


def test_thresholds_match_the_library_sources():
    """The sweep's copy of the dispatch thresholds follows the library's own constants."""
    import re
    csrc = os.path.join(ROOT, "quantized_expert_ffn_token_b200", "csrc")
    internal = open(os.path.join(csrc, "moe_internal.cuh")).read()
    m = re.search(r"constexpr int DECODE_TOKENS_MAX = (\d+);", internal)
    assert m and int(m.group(1)) == bench.DISPATCH_SINGLE_MAX
    m = re.search(r"constexpr int TC_MIN_TOKENS = DECODE_TOKENS_MAX \+ (\d+);", internal)
    assert m and bench.DISPATCH_SINGLE_MAX + int(m.group(1)) == bench.DISPATCH_TC_MIN
    m = re.search(r"constexpr int DECODE_MULTI_MAX = (\d+);", internal)
    assert m and int(m.group(1)) == bench.DISPATCH_FEW_MAX
    tc = open(os.path.join(csrc, "prefill_tc.cu")).read()
    assert "if (T < TC_MIN_TOKENS) return false;" in tc[tc.index("bool tc_supported("):]
