"""Host logic of bench.py that needs no GPU: the source hash that keys the
stored ncu traffic figures ignores comments and nothing else."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_strip_comments_keeps_code_and_literals():
    src = ('int a = 1; // trailing\n'
           'const char* s = "x // not a comment /* nor this */";\n'
           '/* block\n   comment */ char c = \'/\'; char d = \'"\';\n'
           'float e = 2.0f; /**/ int f = a / 2;')
    out = bench._strip_comments(src)
    assert "trailing" not in out and "block" not in out
    assert '"x // not a comment /* nor this */"' in out
    assert "char c = '/';" in out and "char d = '\"';" in out
    assert "int f = a / 2;" in out


def test_hash_ignores_comment_edits_only(tmp_path, monkeypatch):
    csrc = tmp_path / "dequantize_absmax_reduce_b200" / "csrc"
    inc = tmp_path / "include"
    csrc.mkdir(parents=True)
    inc.mkdir()
    for n in bench.TRAFFIC_SOURCES:
        (csrc / n).write_text("int x_%d = 1; // note\n" % len(n))
    (inc / "bq.h").write_text("/* header */ int bq_f(void);\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench._kernel_source_hash()
    (inc / "bq.h").write_text("/* a reworded header comment */ int bq_f(void); // more\n")
    assert bench._kernel_source_hash() == h0
    (inc / "bq.h").write_text("/* header */ int bq_g(void);\n")
    assert bench._kernel_source_hash() != h0
