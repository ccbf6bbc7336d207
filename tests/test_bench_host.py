"""Host-side pieces of bench.py that need no GPU: the kernel-code hash that keys
the committed DRAM counters (comment edits must not invalidate them), and the
shape of the traffic table."""

import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_strip_comments_keeps_code_only():
    src = "int a = 1; // note\n/* block\n   comment */ int b;\n\n   \nfoo(); /* x */ bar();\n"
    assert bench.strip_comments(src) == "int a = 1;\n int b;\nfoo();  bar();"


def test_comment_edits_leave_the_code_hash_alone():
    base = "__global__ void k(int *p) {\n  p[0] = 1;  // store\n}\n"
    reworded = "// a kernel\n__global__ void k(int *p) {\n  p[0] = 1;  /* the store */\n}\n"
    changed = "__global__ void k(int *p) {\n  p[0] = 2;  // store\n}\n"
    assert bench.strip_comments(base) == bench.strip_comments(reworded)
    assert bench.strip_comments(base) != bench.strip_comments(changed)


def test_traffic_table_entries_are_positive_byte_counts():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    assert len(table["source_hash"]) == 16
    for name, passes in table.items():
        if name.startswith("_") or name == "source_hash":
            continue
        assert passes and all(isinstance(v, int) and v > 0 for v in passes.values()), name
