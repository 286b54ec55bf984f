"""Host-side helpers of bench.py: the workload description shared by both arms and the
roofline traffic record lookup (used only while the GEMM code is unchanged)."""
import importlib.util
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def test_config_same_for_both_arms(bench):
    class A:
        config = "8b"
    shape = bench.shape_for("8b")
    c1 = bench.config_for(A, shape, 1)
    assert c1["global_batch"] == 8192 and c1["parallelism"] == "dp1"
    assert "T=8192" in c1["workload"] and "d=4096" in c1["workload"] and "f=14336" in c1["workload"]
    assert bench.config_for(A, shape, 4)["global_batch"] == 4 * 8192


def test_digest_ignores_comments_only(bench, tmp_path, monkeypatch):
    csrc = tmp_path / "lora_fine_tuning_rmsnorm_b200" / "csrc"
    csrc.mkdir(parents=True)
    for n in bench.KERNEL_SOURCES:
        (csrc / n).write_text("int f(int x) {\n  return x + 1;  // add one\n}\n/* note */\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d0 = bench.sources_digest()
    (csrc / bench.KERNEL_SOURCES[0]).write_text("int f(int x) {  // other words\n  return x + 1;\n}\n")
    assert bench.sources_digest() == d0
    (csrc / bench.KERNEL_SOURCES[0]).write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert bench.sources_digest() != d0


def test_traffic_record_lookup(bench, tmp_path, monkeypatch):
    rec = tmp_path / "traffic.md"
    dig = bench.sources_digest()
    rec.write_text("text\ntraffic-record: kernel=k1 config=8b bytes_per_launch=123 sources=%s\n"
                   "traffic-record: kernel=k1 config=8b-4bit bytes_per_launch=77 sources=deadbeef\n" % dig)
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    assert bench.measured_traffic("k1", "8b") == 123.0
    assert bench.measured_traffic("k1", "8b-4bit") is None   # taken on other sources
    assert bench.measured_traffic("k2", "8b") is None
