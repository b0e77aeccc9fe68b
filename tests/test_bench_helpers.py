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


def test_traffic_figures_are_reported_only_for_unchanged_code():
    """Each entry of profiles/ncu_traffic.json is self-consistent, and bench.py reports its bytes
    exactly when the kernel's source still hashes to the captured code_sha (else null)."""
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        entries = {k: v for k, v in json.load(f).items() if not k.startswith("_")}
    assert entries
    for key, e in entries.items():
        assert e["bytes_per_launch"] == e["read"] + e["write"], key
        assert len(e["code_sha"]) == 16 and int(e["code_sha"], 16) >= 0, key
        source = os.path.basename(e["source"])
        with open(os.path.join(ROOT, e["source"]), encoding="utf-8") as f:
            current = bench.code_sha(f.read())
        expected = e["bytes_per_launch"] if current == e["code_sha"] else None
        assert bench._traffic(key, source) == expected, key
