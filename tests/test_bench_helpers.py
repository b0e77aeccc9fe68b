"""Host-side helpers of bench.py (CPU only): the source hash that keys the committed ncu traffic
figures, and the lookup that returns them only while the kernel's code is unchanged."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_sha_ignores_comments_and_blank_space():
    a = "int f(int x) {\n  return x + 1;  // add one\n}\n"
    b = "/* header */\nint f(int x) {\n\n    return x + 1;\n}  // trailing\n"
    assert bench.code_sha(a) == bench.code_sha(b)


def test_code_sha_changes_with_the_code():
    a = "int f(int x) { return x + 1; }"
    assert bench.code_sha(a) != bench.code_sha("int f(int x) { return x + 2; }")
    assert bench.code_sha(a) != bench.code_sha("int f(int y) { return y + 1; }")


def test_committed_traffic_figures_match_the_current_kernel_sources():
    """Every entry of profiles/ncu_traffic.json was captured from the code now in the tree, so
    bench.py reports it (it would report null after a code change)."""
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        entries = {k: v for k, v in json.load(f).items() if not k.startswith("_")}
    assert entries
    for key, e in entries.items():
        source = os.path.basename(e["source"])
        assert bench._traffic(key, source) == e["bytes_per_launch"] == e["read"] + e["write"], key
