"""Host-side pieces of bench.py that need no GPU.

The bench reports ncu's DRAM traffic for a kernel only while the kernel's
code is the code that was captured; the check hashes the sources without
their comments, so a comment edit keeps the figure and a code edit drops it.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_strip_comments_keeps_code_and_literals():
    src = ('int a = 1;  // trailing\n'
           '/* block\n   comment */ float b = 2.f;\n'
           '\n'
           'const char *s = "x // not a comment /* nor this */";\n'
           "char c = '/';  /* c */\n"
           'asm volatile("fence.acq_rel.gpu;" ::: "memory");\n')
    assert bench.strip_comments(src) == (
        'int a = 1;\n'
        ' float b = 2.f;\n'
        'const char *s = "x // not a comment /* nor this */";\n'
        "char c = '/';\n"
        'asm volatile("fence.acq_rel.gpu;" ::: "memory");')


def test_digest_ignores_comments_but_not_code():
    base = ["int f(int x) {\n  return x + 1;  // add one\n}\n"]
    reworded = ["// helper\nint f(int x) {\n  return x + 1;  /* one more */\n}\n\n"]
    changed = ["int f(int x) {\n  return x + 2;  // add one\n}\n"]
    assert bench.source_digest(base) == bench.source_digest(reworded)
    assert bench.source_digest(base) != bench.source_digest(changed)


def test_traffic_only_for_the_captured_configuration():
    # another window or KV-head count than the captured run: no figure
    assert bench.captured_traffic("decode_b8_n8000", "decode", 512, None) is None
    assert bench.captured_traffic("decode_b8_n8000", "decode", None, 1) is None
    assert bench.captured_traffic("no_such_workload", "decode", None, None) is None
