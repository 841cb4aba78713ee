"""Host-side logic of bench.py that needs no GPU: the source digest that keys
the recorded ncu traffic, and the lookup that drops a stale record."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_strip_comments_keeps_code_and_literals():
    src = ('int a = 1; // trailing\n'
           '/* block\n   comment */ const char *s = "a//b /* not */";\n'
           "char q = '\"'; x = y / z; /**/ w;\n\n")
    assert bench.strip_comments(src) == ('int a = 1;\nconst char *s = "a//b /* not */";\n'
                                         "char q = '\"'; x = y / z; w;")


@pytest.fixture
def fake_tree(tmp_path, monkeypatch):
    csrc = tmp_path / "dense_sparse_quantized_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("__global__ void k() { int a = 1; }  // v1\n")
    (csrc / "h.h").write_text("#define N 4\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def test_digest_ignores_comments_but_not_code(fake_tree):
    csrc = fake_tree / "dense_sparse_quantized_b200" / "csrc"
    d0 = bench.kernel_source_digest()
    (csrc / "k.cu").write_text("// header\n__global__  void k() { int a = 1; }  /* v2 */\n\n")
    assert bench.kernel_source_digest() == d0
    (csrc / "k.cu").write_text("__global__ void k() { int a = 2; }\n")
    assert bench.kernel_source_digest() != d0


def test_traffic_record_is_dropped_when_its_sources_change(fake_tree):
    csrc = fake_tree / "dense_sparse_quantized_b200" / "csrc"
    rec = {"c9_b1": {"dram_bytes_per_launch": 123.0, "sources": ["k.cu"],
                     "source_digest": bench.kernel_source_digest(["k.cu"]), "note": "n"}}
    (fake_tree / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("c9", 1) == (123.0, "n")
    (csrc / "h.h").write_text("#define N 8\n")  # not one of the record's sources
    assert bench.recorded_traffic("c9", 1) == (123.0, "n")
    (csrc / "k.cu").write_text("__global__ void k() { int a = 3; }\n")
    assert bench.recorded_traffic("c9", 1) == (None, None)
    assert bench.recorded_traffic("c9", 2) == (None, None)
