"""Builds libgca.so (the C-ABI library) in-tree for sm_100a with nvcc.

    python -m paged_kv_cache_gca_b200.build [--verbose]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libgca.so")
SOURCES = ["gca_api.cu", "gca_append.cu", "gca_attn.cu", "gca_combine.cu", "gca_decode.cu",
           "gca_noalloc.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def build_command(verbose: bool = False, out: str | None = None) -> list[str]:
    """The nvcc command line that builds the library (sm_100a only)."""
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-cudart", "static", "-o", (LIB if out is None else out) + ".tmp", *srcs, "-ldl",
           "-lrt", "-lpthread"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def build(verbose: bool = False, force: bool = False) -> str:
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    deps = srcs + [os.path.join(CSRC, "gca_internal.h"),
                   os.path.join(os.path.dirname(HERE), "include", "gca.h")]
    if not force and os.path.exists(LIB):
        lib_t = os.path.getmtime(LIB)
        if all(os.path.getmtime(d) <= lib_t for d in deps):
            return LIB
    cmd = build_command(verbose)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force=True)
    print(LIB)
