"""The kernel-code hash that keeps committed ncu traffic figures attached to a
kernel: comments and blank lines do not change it, code does."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_comments_and_blank_lines_do_not_change_the_code():
    a = "int f(int x) {\n  return x + 1;  // one more\n}\n"
    b = "// header\n/* block\n   comment */\nint f(int x) {\n\n  return x + 1;\n}\n"
    assert bench.source_code(a) == bench.source_code(b)


def test_a_code_change_changes_the_code():
    a = "int f(int x) {\n  return x + 1;\n}\n"
    b = "int f(int x) {\n  return x + 2;\n}\n"
    assert bench.source_code(a) != bench.source_code(b)


def test_committed_traffic_entries_match_the_sources():
    """Every entry of profiles/ncu_traffic.json names the sources of its kernel(s),
    which hash to the recorded value (else bench.py reports traffic as null), and a
    committed ncu summary."""
    import json
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        entries = {k: v for k, v in json.load(f).items() if not k.startswith("_")}
    for key, e in entries.items():
        assert e["sources"], key
        assert bench.source_sha(*e["sources"]) == e["source_sha"], key
        assert bench.ncu_traffic(key) == e["dram_bytes_per_launch"]
        assert os.path.exists(os.path.join(ROOT, "profiles", e["profile"]))
