"""The CPU-side legs of bench.py: the oracle baseline and the reference arm (`--impl reference`,
the oracle timed on the host cores), run here on the tiny workload. CPU only."""
import json
import os
import subprocess
import sys

import bench
import gca_inputs as gi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_oracle_baseline_reports_its_sample_and_core_counts():
    v, d = bench.oracle_frames_per_s(gi.workload("tiny"), [2, 5])
    assert v > 0
    for key in ("bookkeeping_s", "attention_s_sampled", "estimated_stream_s", "nproc",
                "torch_threads"):
        assert key in d
    assert d["nproc"] >= 1 and d["torch_threads"] >= 1


def test_reference_arm_prints_one_json_line():
    res = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                          "--steps", "2", "--warmup", "3"], cwd=ROOT, capture_output=True,
                         text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "frames/s" and line["value"] > 0
    assert line["higher_is_better"] is True and line["steps"] == 2 and line["warmup"] == 3
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
