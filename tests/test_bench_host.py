"""Host-side pieces of bench.py that need no GPU: the clock record taken
during the timed region, the code layout both arms name, the byte counts the
roofline divides by, and the rule that committed DRAM counters count only for
the kernel source they were taken on."""
import json
import os
import stat
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from lut_logits_serving_b200 import synth  # noqa: E402


def fake_smi(tmp_path, lines):
    """An `nvidia-smi` on PATH that prints the given CSV rows and then waits
    like the real one in its sampling loop."""
    d = tmp_path / "bin"
    d.mkdir()
    body = "\n".join(f"echo '{l}'" for l in lines)
    p = d / "nvidia-smi"
    p.write_text(f"#!/bin/sh\n{body}\nexec sleep 30\n")
    p.chmod(p.stat().st_mode | stat.S_IEXEC)
    return str(d)


def sample(idx, sm, mx, reasons=("Not Active",) * 4):
    return ", ".join([str(idx), str(sm), str(mx), "700.5", "0x0"] + list(reasons))


def test_clock_record_median_max_and_reasons(tmp_path, monkeypatch):
    rows = [sample(0, 1965, 1965),
            sample(0, 1860, 1965, ("Not Active", "Not Active", "Not Active", "Active")),
            sample(0, 1890, 1965),
            "garbage line"]
    monkeypatch.setenv("PATH", fake_smi(tmp_path, rows) + os.pathsep + os.environ["PATH"])
    with bench.ClockSampler(0) as clk:
        time.sleep(0.5)
    s = clk.summary()
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1890.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_record_flags_the_slowdowns_that_void_a_run(tmp_path, monkeypatch):
    rows = [sample(0, 1500, 1965, ("Active", "Not Active", "Active", "Not Active"))]
    monkeypatch.setenv("PATH", fake_smi(tmp_path, rows) + os.pathsep + os.environ["PATH"])
    with bench.ClockSampler(0) as clk:
        time.sleep(0.3)
    assert clk.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_record_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    with bench.ClockSampler(0) as clk:
        pass
    assert clk.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_headline_layout_of_each_workload():
    W = synth.WORKLOADS
    assert bench.headline_layout(W["g2_b1"]) == "sched"
    assert bench.headline_layout(W["g2_b32"]) == "u16"
    assert bench.headline_layout(W["packed_b64"]) == "packed10"
    assert bench.headline_layout(W["packed_b64"], "u8") == "packed10"
    assert bench.headline_layout(W["g2_b1"], "u16") == "u16"
    assert bench.headline_layout(W["g2_b32"], "u8") == "u8"


def test_byte_counts_the_rooflines_divide_by():
    W = synth.WORKLOADS
    assert bench.code_bytes(W["g2_b1"]) == 256000 * 768 * 2          # 393.2 MB
    assert bench.code_bytes(W["g2_b1"], "u8") == 256000 * 768
    assert bench.code_bytes(W["packed_b64"]) == 256000 * 960         # 245.8 MB
    # per id: its code row, one 24-byte codeword per (m, l), its bf16 row
    assert bench.decode_bytes(W["decode512"]) == 512 * (1536 + 768 * 24 + 4608)


def test_committed_counters_count_only_for_their_source(tmp_path, monkeypatch):
    csrc = tmp_path / "lut_logits_serving_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in ("logits_chunk.cu", "decode_rows.cu", "logits_decode_mma.cu", "rq_common.cuh"):
        (csrc / name).write_text(f"// {name}\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    key = "decode_rows_pair_kernel/u16/decode512"
    entry = {key: {"source_sha": bench.kernel_source_hash(key), "dram_bytes_per_launch": 123}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(entry))
    assert bench.profiled_traffic(key) == 123
    assert bench.profiled_traffic("logits_chunk_u16_kernel/sched/g2_b1") is None
    # the decode counters follow decode_rows.cu, not the code-pass source
    (csrc / "logits_chunk.cu").write_text("// changed\n")
    assert bench.profiled_traffic(key) == 123
    (csrc / "decode_rows.cu").write_text("// changed\n")
    assert bench.profiled_traffic(key) is None
    (tmp_path / "profiles" / "traffic.json").unlink()
    assert bench.profiled_traffic(key) is None


def parse_argv(argv):
    old = sys.argv
    try:
        sys.argv = ["bench.py"] + argv
        return bench.parse()
    finally:
        sys.argv = old


def test_workload_choices_cover_the_workloads():
    for name in ("g2_b1", "g2_b1_packed10", "g2_b32", "packed_b64", "decode512", "encode_g2",
                 "g2_b1_topk50",
                 "mlp_gate_b1", "mlp_down_b1"):
        assert name in synth.WORKLOADS
        assert parse_argv(["--workload", name]).workload == name
    with pytest.raises(SystemExit):
        parse_argv(["--workload", "nope"])
    a = parse_argv([])
    assert (a.gpus, a.workload, a.impl) == (1, "g2_b1", "ours") and a.warmup >= 3


def test_packed_code_bytes_on_a_uint16_workload():
    """A batch-1 workload timed on 10-bit packed codes divides by the packed
    matrix (960 B per row), not by the uint16 one."""
    assert bench.code_bytes(synth.WORKLOADS["g2_b1"], "packed10") == 256000 * 960
    # the rotated slices add one byte per 32 codes
    assert bench.code_bytes(synth.WORKLOADS["g2_b1"], "rot10") == 256000 * (960 + 24)
    c = bench.workload_config(synth.WORKLOADS["g2_b1"], "packed10")
    assert c["codes"] == "packed10" and "packed10 (960 B/row)" in c["workload"]
    assert "rotated" in bench.workload_config(synth.WORKLOADS["g2_b1"], "rot10")["workload"]
