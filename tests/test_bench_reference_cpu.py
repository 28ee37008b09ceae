"""bench.py --impl reference times the CPU oracle on the benchmark workload
(a bounded row sample per step) and prints the contract's JSON line."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference"
    assert j["unit"] == "vocab-rows/s" and j["higher_is_better"] is True
    assert j["value"] > 0 and j["steps"] == 2 and j["warmup"] == 1
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] >= 1
    assert j["cpu_baseline"]["nproc"] == os.cpu_count() and j["cpu_baseline"]["cpu_model"]
    assert j["config"]["parallelism"] == "replicas x1"
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["d2h_bytes_per_step"] == 0
    assert j["config"]["V"] == 256000


def test_reference_arm_on_the_row_decode_workload():
    """decode512: the oracle's bf16 row rebuild of 512 Zipf ids, one line with
    the same metric, unit and workload description as the CUDA arm."""
    sys.path.insert(0, ROOT)
    import bench
    from lut_logits_serving_b200 import synth
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "decode512", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["metric"] == bench.DEC_METRIC
    assert j["unit"] == "rows/s" and j["value"] > 0
    assert j["config"] == dict(bench.decode_config(synth.WORKLOADS["decode512"]),
                               parallelism="replicas x1")
    assert j["config"]["ids"] == 512
    assert j["cpu_baseline"]["value"] == j["value"] and j["e2e"]["value"] == j["value"]
