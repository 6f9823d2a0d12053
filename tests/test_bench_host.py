"""Host logic of bench.py that needs no GPU: the recorded DRAM traffic is
tied to the kernel's code, not to its comments or layout."""
from __future__ import annotations

import bench


def test_comment_and_layout_edits_keep_the_code_hash():
    code = 'int f(int x) {\n  // scale\n  return x * 2; /* twice */\n}\nconst char* s = "a // b";\n'
    edited = '// header\nint f(int x)\n{\n    return x * 2;  // doubled\n}\nconst char* s = "a // b";\n'
    assert bench.strip_comments(code) == bench.strip_comments(edited)


def test_code_and_literal_edits_change_the_code_hash():
    code = 'int f(int x) { return x * 2; }\nconst char* s = "a // b";\n'
    assert bench.strip_comments(code) != bench.strip_comments(code.replace("x * 2", "x * 3"))
    assert bench.strip_comments(code) != bench.strip_comments(code.replace('"a // b"', '"a // c"'))
    assert bench.strip_comments(code) != bench.strip_comments(code.replace("return x", "return  y"))


def test_recorded_traffic_only_for_the_code_it_was_taken_on(monkeypatch):
    import json
    import os

    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)["k_decode_int8_sm100@decode"]
    monkeypatch.setattr(bench, "kernel_source_sha", lambda k: rec["source_sha"])
    assert bench.recorded_traffic("k_decode_int8_sm100", "decode") == rec["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "kernel_source_sha", lambda k: "0" * 16)
    assert bench.recorded_traffic("k_decode_int8_sm100", "decode") is None
    assert bench.recorded_traffic("k_decode_int8_sm100", "no-such-workload") is None
