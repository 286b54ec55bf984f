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
    import json
    rec = tmp_path / "traffic.json"
    dig = bench.sources_digest()
    rec.write_text(json.dumps({"records": [
        {"kernel": "k1", "config": "8b", "bytes_per_launch": 123, "sources": dig},
        {"kernel": "k1", "config": "8b-4bit", "bytes_per_launch": 77, "sources": "deadbeef"}]}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    assert bench.measured_traffic("k1", "8b") == 123.0
    assert bench.measured_traffic("k1", "8b-4bit") is None   # taken on other sources
    assert bench.measured_traffic("k2", "8b") is None


def test_dtype_label_names_the_weight_format(bench):
    assert bench.dtype_for("8b") == "bf16"
    assert "4-bit" in bench.dtype_for("8b-4bit")


def test_codebook_loader_reads_the_stored_codebook(bench):
    from tests.parity import load_codebook
    assert bench.load_codebook() == load_codebook()


@pytest.mark.timeout(300)
def test_gpus_flag_launches_that_many_ranks_cpu_stub():
    """`bench.py --gpus 2` without torchrun relaunches itself as 2 ranks; with the CPU stub
    step (gloo) the line must report n_gpus 2, the max over ranks of the per-rank times and
    a correct flat-buffer all-reduce."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--stub-cpu", "--steps", "3",
                        "--warmup", "3"], capture_output=True, text=True, timeout=240,
                       env={k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(ln) for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    ln = lines[0]
    assert ln["n_gpus"] == 2 and ln["allreduce_ok"] is True
    assert ln["ms_max_over_ranks"] == 20.0     # rank 1's 20 ms, not rank 0's 10 ms
