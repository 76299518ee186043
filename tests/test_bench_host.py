"""Host logic of bench.py that needs no GPU: the source fingerprint that decides whether a committed
DRAM-traffic capture of a workload's gate/up GEMM (a json traffic block in a profiles/*.md summary) still
describes the kernel being timed."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_tokens_ignores_comments_and_layout():
    a = "int a = 1; // one\n\n    int  b;   /* two\n lines */ int c;\n"
    b = "int a = 1;\nint b;\nint c; // other words\n"
    assert bench.code_tokens(a) == bench.code_tokens(b) == "int a = 1; int b; int c;"


def test_code_tokens_sees_code_changes():
    assert bench.code_tokens("x = a + b;") != bench.code_tokens("x = a - b;")
    assert bench.code_tokens("f(1, 2);") != bench.code_tokens("f(1, 3);")


def test_code_tokens_keeps_literals():
    # comment markers and whitespace runs inside string and character literals are code
    src = 's = "a  // b /* c */"; q = \'\\\'\'; t = "\\"//";'
    assert bench.code_tokens(src) == src
    assert bench.code_tokens('s = "a  b";') != bench.code_tokens('s = "a b";')


def test_traffic_only_for_the_captured_workload():
    # a capture of one workload never stands in for another
    assert bench.measured_traffic("no-such-workload") is None


def _fake_tree(tmp_path, src_text, captured_text, workload="wl-a"):
    import hashlib
    import json
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cu").write_text(src_text)
    h = hashlib.sha256(bench.code_tokens(captured_text).encode()).hexdigest()
    meta = {"workload": workload, "dram_bytes_per_launch": 12345, "sources": ["k.cu"], "sources_sha256": h}
    (tmp_path / "profiles" / "cap.md").write_text("# capture\n\n```json traffic\n" + json.dumps(meta) + "\n```\n")


def test_traffic_found_in_any_profile_while_its_sources_match(tmp_path, monkeypatch):
    _fake_tree(tmp_path, "int f() { return 1; }  // now with a comment", "int f() { return 1; }")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("wl-a") == 12345     # comments and layout do not matter
    assert bench.measured_traffic("wl-b") is None      # another workload's capture never stands in


def test_traffic_dropped_once_the_captured_code_changes(tmp_path, monkeypatch):
    _fake_tree(tmp_path, "int f() { return 2; }", "int f() { return 1; }")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("wl-a") is None
