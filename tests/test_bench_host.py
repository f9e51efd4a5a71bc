"""Host-side pieces of bench.py that need no GPU."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def test_code_only_ignores_comments_and_blank_lines():
    a = "int f(int x) {\n  // old note\n  return x + 1;  /* tail */\n}\n"
    b = "/* header\n   spanning lines */\nint f(int x) {\n\n  // a different note\n  return x + 1;\n}\n"
    assert bench.code_only(a) == bench.code_only(b)


def test_code_only_sees_code_changes():
    a = "int f(int x) { return x + 1; }\n"
    b = "int f(int x) { return x + 2; }  // same comment\n"
    assert bench.code_only(a) != bench.code_only(b)

