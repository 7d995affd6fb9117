"""The C ABI from plain C, with no GPU: include/gca.h compiles as C11 and as C++17 with warnings as
errors, and a C program linked against the library (tests/c/abi_check.c) calls its host-side
entry points -- config validation, workspace sizing, status strings."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.join(ROOT, "paged_kv_cache_gca_b200")


@pytest.mark.parametrize("compiler,std,ext", [("gcc", "-std=c11", "c"), ("g++", "-std=c++17", "cpp")])
def test_header_compiles_cleanly(tmp_path, compiler, std, ext):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not installed")
    src = tmp_path / f"header.{ext}"
    src.write_text('#include "gca.h"\nint main(void) { return 0; }\n')
    subprocess.run([compiler, std, "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INCLUDE,
                    "-c", str(src), "-o", str(tmp_path / "header.o")], check=True)


def test_c_client_links_and_runs(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not installed")
    from paged_kv_cache_gca_b200 import build

    build.build()
    exe = tmp_path / "abi_check"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE,
                    os.path.join(ROOT, "tests", "c", "abi_check.c"), "-L", PKG, "-lgca",
                    f"-Wl,-rpath,{PKG}", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    print(r.stdout)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "FAIL" not in r.stdout
