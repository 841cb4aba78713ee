"""Host-side logic of bench.py that needs no GPU: the source digest that keys
the recorded ncu traffic, and the lookup that drops a stale record."""
import json
import os
import sys

import numpy as np

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


def _json_lines(out: str):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def _check_reference_line(line):
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["higher_is_better"] is True and line["dtype"] == "f64"
    assert line["config"]["workload"].startswith("c2:")
    # the same workload keys as the GPU arm's line
    for key in ("batch", "rows", "cols", "bits", "mode", "nnz", "canonical_bytes_per_call"):
        assert key in line["config"], key
    assert (line["config"]["rows"], line["config"]["cols"], line["config"]["bits"]) == (11008, 4096, 3)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    assert cb["nproc"] >= cb["cores"] and cb["cpu_model"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_runs_the_oracle_on_host_cores():
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_reference_line(lines[0])


def test_reference_arm_under_two_ranks_prints_once():
    """Under torchrun only rank 0 times the oracle and prints; rank 1 exits 0."""
    import socket
    import subprocess
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_reference_line(lines[0])


def test_oracle_rate_threads_cover_every_row_once(monkeypatch):
    """The all-core CPU baseline runs the unmodified oracle on row slices in
    threads: together the slices compute exactly the full product."""
    import oracle
    import synth
    p = synth.make_problem(97, 256, 3, "affine", 0.01, "uniform", 3, 1)
    orc = oracle.load()
    seen = []
    real = orc.gemv

    def spy(q, x=None, rows=None):
        seen.append(np.asarray(rows).copy())
        return real(q, x=x, rows=rows)

    monkeypatch.setattr(orc, "gemv", spy)
    gbs, n, el = bench.oracle_rate(p, 0.0, threads=4)
    assert n == 1 and gbs > 0
    assert len(seen) == 4
    assert np.array_equal(np.sort(np.concatenate(seen)), np.arange(p.rows))
