"""The kernel-source digest that ties a committed profile to the kernel it measured: comments
and whitespace do not change it, code does, and string literals are kept as code."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_comments_and_whitespace_are_ignored():
    a = "int f(int x) {\n  return x + 1;  // one more\n}\n"
    b = "/* a function */\nint f(int x) {\n    return x + 1;\n}"
    assert bench._code_only(a) == bench._code_only(b)


def test_code_changes_are_seen():
    assert bench._code_only("return x + 1;") != bench._code_only("return x + 2;")


def test_literals_are_code():
    src = 'asm("add.f32 %0, %1; // not a comment"); char c = \'/\'; const char *s = "/* nor this */";'
    out = bench._code_only(src)
    assert "// not a comment" in out and "/* nor this */" in out and "'/'" in out


def test_escaped_quote_inside_a_literal():
    src = 'const char *s = "a\\"b // x"; int y; // tail'
    assert bench._code_only(src) == 'const char *s = "a\\"b // x"; int y;'


def test_digest_is_sixteen_hex_digits():
    d = bench.source_digest()
    assert len(d) == 16 and all(c in "0123456789abcdef" for c in d)
