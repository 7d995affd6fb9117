"""The whole path driven from plain C through the C ABI (tests/c/abi_gpu.c: a cudaMalloc'd
workspace, gca_cache_create with a permuted page order, gca_append_frame and gca_attend over six
frames; no Python framework in the process), its outputs checked against the oracle on the same
inputs, which the program writes out with its outputs."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle.gca_oracle as orc
from gca_testutil import check_attention

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.join(ROOT, "paged_kv_cache_gca_b200")
T, H, D, FRAMES, PAGES = 68, 2, 64, 6, 24  # the program's configuration


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def test_c_client_matches_the_oracle(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not installed")
    from paged_kv_cache_gca_b200 import build

    build.build()
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = tmp_path / "abi_gpu"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE,
                    "-I", os.path.join(cuda, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_gpu.c"), "-L", PKG, "-lgca",
                    "-L", os.path.join(cuda, "lib64"), "-lcudart", f"-Wl,-rpath,{PKG}",
                    f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}", "-o", str(exe)], check=True)
    data = tmp_path / "frames.bin"
    r = subprocess.run([str(exe), str(data)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    raw = np.fromfile(data, dtype=np.uint16).reshape(FRAMES, 4, T, H, D)
    o = orc.GcaOracle(num_heads=H, head_dim=D, page_size=16, grid_h=8, grid_w=8, num_special=4,
                      anchor_frames=1, window_frames=2, keep_tokens=4, rope_base=10000.0,
                      initial_free=[(7 * i + 5) % PAGES for i in range(PAGES)],
                      frame_source=lambda t: tuple(_bf16(raw[t, j]) for j in range(3)))
    for t in range(FRAMES):
        o.append(t)
        got = _bf16(raw[t, 3]).double().numpy()
        check_attention(got, o.attend(t), f"C client t={t}")
