"""The attention work split on the CPU: tests/c/split_check.cu includes the library's internal
header and checks the split functions the attention kernel, the combine kernel and the host
planner share (CTA ranges cover the steps in order, the step -> CTA inverse is exact, partial
record slots are distinct and within the planned scratch, and a CTA that moves to another work
unit is charged for it) over 1,440 shapes. Host code only: nvcc compiles it without a GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "paged_kv_cache_gca_b200", "csrc")


def _nvcc():
    from paged_kv_cache_gca_b200 import build

    path = build.nvcc()
    return path if (os.path.exists(path) or shutil.which(path)) else None


def test_split_bookkeeping(tmp_path):
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not installed")
    exe = tmp_path / "split_check"
    subprocess.run([nvcc, "-std=c++17", "-O2", "-Wno-deprecated-gpu-targets", "-I", CSRC,
                    os.path.join(ROOT, "tests", "c", "split_check.cu"), "-o", str(exe)],
                   check=True, capture_output=True, timeout=600)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok "), r.stdout
