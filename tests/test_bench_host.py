"""Host logic of bench.py that needs no GPU: the source fingerprint that decides whether the committed
DRAM-traffic capture of the gate/up GEMM still describes the kernel being timed."""
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
