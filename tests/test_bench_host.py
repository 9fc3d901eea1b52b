"""Host-side logic of bench.py (no GPU): the hash that ties the recorded DRAM traffic of the
global prefill kernel to the code it was measured on."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_lines_drop_comments_and_blank_lines():
    src = "\n".join([
        "// a file comment",
        "int a = 1;   // trailing comment",
        "",
        "    ",
        'const char* s = "http://x";  // a // inside a string stays',
        "  int b = a + 2;",
    ])
    assert bench._code_lines(src) == ['int a = 1;', 'const char* s = "http://x";', "  int b = a + 2;"]


def test_comment_edits_keep_the_code_the_same_and_code_edits_do_not():
    base = "int f(int x) {\n    return x + 1;   // one more\n}\n"
    reworded = "// f adds one\nint f(int x) {\n\n    return x + 1;   // the successor\n}\n"
    changed = "int f(int x) {\n    return x + 2;   // one more\n}\n"
    assert bench._code_lines(base) == bench._code_lines(reworded)
    assert bench._code_lines(base) != bench._code_lines(changed)


def test_recorded_traffic_matches_only_its_own_hash():
    with open(bench.TRAFFIC_JSON) as f:
        rec = json.load(f)
    assert bench.recorded_traffic(rec["kernel_source_hash"]) == float(rec["dram_bytes_per_full_launch"])
    assert bench.recorded_traffic("0" * 16) is None
