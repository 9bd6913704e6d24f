"""The bench's measured-traffic table: a figure is tied to the code of the
kernel sources it was captured on, so an edit to comments keeps it and an
edit to code voids it (the line then reports null)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_comments_and_blank_lines_do_not_count():
    a = "int f(int x) {\n    return x + 1;   // one more\n}\n"
    b = "/* a note\n   over lines */\nint f(int x) {\n\n    return x + 1;\n}  // end\n"
    assert bench._code_only(a) == bench._code_only(b)


def test_code_changes_count():
    a = "int f(int x) { return x + 1; }\n"
    b = "int f(int x) { return x + 2; }\n"
    assert bench._code_only(a) != bench._code_only(b)


def test_every_entry_names_existing_sources_and_a_profile():
    for m in bench.MEASURED_TRAFFIC:
        for rel in m["src"]:
            assert os.path.exists(os.path.join(ROOT, "quantized_expert_ffn_token_b200", "csrc", rel))
        assert os.path.exists(os.path.join(ROOT, m["profile"]))
        assert m["bytes_per_layer"] > 0


def test_lookup_needs_matching_code():
    m = bench.MEASURED_TRAFFIC[0]
    layers = 3
    got = bench.measured_traffic(m["kernel"], m["workload"], layers)
    want = m["bytes_per_layer"] * layers if bench._src_sha(m["src"]) == m["sha256"] else None
    assert got == want
    assert bench.measured_traffic(m["kernel"], "no such workload", layers) is None
