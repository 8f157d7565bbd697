"""Host-side checks of the benchmark's reporting logic (no GPU): the reference
arm's JSON line on a small workload, the whole-job throughput formula, and the
rule that a profiled DRAM traffic figure is used only while its recorded
kernel-source hash matches the current source."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_job_throughput_counts_every_rank():
    # 2 ranks x 10 units per step x 4 steps in 2 s (slowest rank) = 40 units/s
    assert bench.job_throughput(10, 4, 2, 2000.0) == pytest.approx(40.0)
    assert bench.job_throughput(10, 4, 1, 2000.0) == pytest.approx(20.0)


def test_reference_arm_json_line():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
         "tiny_gpt_t2", "--steps", "1", "--warmup", "1"],
        capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["warmup"] >= 3
    assert line["value"] > 0 and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    # the arm reports the workload it timed, under the same config as the GPU arm
    assert line["config"] == bench.layer_config(bench.TI.WORKLOADS["tiny_gpt_t2"], "tiny_gpt_t2")
    assert line["config"]["batch"] == 2 and "2 x seq 128" in line["cpu_baseline"]["sample"]


def test_profiled_traffic_needs_matching_source_hash(tmp_path, monkeypatch):
    csrc = tmp_path / "tensor_transformer_layer_tp_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("kernel v1\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.source_hash(["k.cu"])
    (tmp_path / "profiles" / "k.md").write_text(
        f"# k\nsource_hash: {h}\ndram_bytes_per_launch: 1234\n")
    assert bench.profiled_traffic("k.md", ["k.cu"]) == 1234.0
    (csrc / "k.cu").write_text("kernel v2\n")          # source changed since the capture
    assert bench.profiled_traffic("k.md", ["k.cu"]) is None
    assert bench.profiled_traffic("missing.md", ["k.cu"]) is None
