"""Host-side pieces of bench.py that need no GPU."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_tokens_ignore_comments_and_layout():
    a = 'int f(int x) {  // add one\n  return x + 1; /* done */\n}\n'
    b = '/* header\n   lines */\nint f(int x) {\n\n  return x + 1;\n}  // trailing\n'
    assert bench._code_tokens(a) == bench._code_tokens(b)
    # a code change is seen
    assert bench._code_tokens(a) != bench._code_tokens(a.replace("x + 1", "x + 2"))


def test_code_tokens_keep_string_literals():
    # comment markers inside string and character literals are code
    src = 'const char* s = "http://x /* y */"; char c = \'/\'; asm("a; // b");\n'
    toks = bench._code_tokens(src)
    assert '"http://x /* y */"' in toks and "'/'" in toks and '"a; // b"' in toks

