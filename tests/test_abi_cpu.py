"""The C-ABI library builds, loads and exports every symbol include/gca.h declares; host-only
entry points (validation, workspace sizing, status names) work without a GPU."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import gca_inputs as gi
import paged_kv_cache_gca_b200 as gca
from paged_kv_cache_gca_b200 import build as gbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    return gca.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "gca.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gca_[a-z_]+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert header_functions() == sorted(gca.EXPORTED_SYMBOLS)


def test_library_exports_every_header_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", gca.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in header_functions():
        assert name in exported, name
        assert getattr(L, name) is not None


def test_library_is_built_for_sm100a_only():
    # the one target the build passes to nvcc: real sm_100a code, no PTX for other GPUs
    assert gbuild.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert "-arch" not in gbuild.build_command()
    assert gbuild.ARCH[0] in gbuild.build_command()


def test_status_strings(L):
    for code, name in gca.STATUS.items():
        assert gca.gca_status_string(code) == name


@pytest.mark.parametrize("name", list(gi.WORKLOADS))
def test_workloads_validate_and_size(L, name):
    w = gi.workload(name)
    cfg = gca.config_for(w)
    assert gca.gca_validate_config(cfg) == 0
    n = gca.gca_workspace_bytes(cfg)
    pools = 2 * w.num_pages * w.num_heads * w.page_size * w.head_dim * 2
    assert pools < n < pools + 64 * 2**20 + 8 * w.max_frames * 64
    assert n % 1024 == 0


def test_invalid_configs(L):
    base = gca.config_for(gi.workload("w16_320"))

    def with_(**kw):
        c = gca.GcaConfig()
        ctypes.memmove(ctypes.byref(c), ctypes.byref(base), ctypes.sizeof(c))
        for k, v in kw.items():
            setattr(c, k, v)
        return c

    assert gca.gca_validate_config(with_(window_frames=0)) == -1
    assert gca.gca_validate_config(with_(num_heads=0)) == -1
    assert gca.gca_validate_config(with_(keep_tokens=2000)) == -1
    assert gca.gca_validate_config(with_(rope_base=-1.0)) == -1
    assert gca.gca_validate_config(with_(num_pages=0)) == -1
    assert gca.gca_validate_config(with_(head_dim=128)) == -5
    assert gca.gca_validate_config(with_(page_size=32)) == -5
    assert gca.gca_validate_config(with_(keep_tokens=80)) == -5
    assert gca.gca_workspace_bytes(with_(window_frames=0)) == 0
    assert L.gca_validate_config(None) == -1


def test_create_rejects_bad_arguments_before_touching_cuda(L):
    cfg = gca.config_for(gi.workload("tiny"))
    h = ctypes.c_void_p()
    n = gca.gca_workspace_bytes(cfg)
    # null out-pointer, null workspace, misaligned workspace, too-small workspace
    assert L.gca_cache_create(ctypes.byref(cfg), 1024, n, None, None, None) == -1
    assert L.gca_cache_create(ctypes.byref(cfg), None, n, None, None, ctypes.byref(h)) == -1
    assert L.gca_cache_create(ctypes.byref(cfg), 1024 + 16, n, None, None, ctypes.byref(h)) == -1
    assert L.gca_cache_create(ctypes.byref(cfg), 1024, n - 1, None, None, ctypes.byref(h)) == -1
    # a misaligned device free list is rejected before any CUDA call
    assert L.gca_cache_create(ctypes.byref(cfg), 1024, n, 4096 + 2, None, ctypes.byref(h)) == -1
    assert h.value is None
    # calls on a null handle
    assert L.gca_append_frame(None, 0, 1, 1, 1, 1, None) == -1
    assert L.gca_attend(None, 0, 1, 1, None) == -1
    assert L.gca_reset(None, None) == -1
    assert L.gca_check(None) == -1
    assert L.gca_cache_destroy(None) == 0
    assert L.gca_append_frame_ex(None, 0, 0, 0, 1, 1, 1, 1, None) == -1
    assert L.gca_rollback_last_frame(None, 0, None) == -1
    assert L.gca_attend_prefill(None, 1, 1, 1, None) == -1
    # batched append: empty or oversized batch, null arrays, null cache
    VP, I64 = ctypes.c_void_p, ctypes.c_int64
    one = (VP * 1)(1)
    idx = (I64 * 1)(0)
    nul = (VP * 1)(None)
    assert L.gca_append_frames(one, 0, idx, one, one, one, one, None) == -1
    assert L.gca_append_frames(one, 129, idx, one, one, one, one, None) == -1
    assert L.gca_append_frames(None, 1, idx, one, one, one, one, None) == -1
    assert L.gca_append_frames(one, 1, None, one, one, one, one, None) == -1
    assert L.gca_append_frames(nul, 1, idx, one, one, one, one, None) == -1


def test_binding_routes_each_call_to_its_entry_point(L):
    # a cache object whose handle is NULL: the library rejects every call before touching CUDA,
    # and the error names the entry point the binding chose
    cache = gca.GcaCache.__new__(gca.GcaCache)
    cache.handle = None
    x = torch.zeros(4, dtype=torch.bfloat16)

    def where(fn, *a, **kw):
        with pytest.raises(gca.GcaError) as e:
            fn(*a, **kw)
        assert e.value.status == -1
        return str(e.value).split(":")[0]

    assert where(cache.append_frame, 0, x, x, x, x, stream=0) == "gca_append_frame"
    assert where(cache.append_frame, 0, x, x, x, x, stream=0, transient=True) == \
        "gca_append_frame_ex"
    assert where(cache.append_frame, 0, x, x, x, x, stream=0, rope_frame=3) == \
        "gca_append_frame_ex"
    assert where(cache.attend, 0, x, x, stream=0) == "gca_attend"
    assert where(cache.attend_prefill, 2, x, x, stream=0) == "gca_attend_prefill"
    assert where(cache.rollback, 0) == "gca_rollback_last_frame"
    assert where(cache.reset, stream=0) == "gca_reset"
    assert where(gca.gca_append_frames, [None], [0], [1], [1], [1], [1], 0) == \
        "gca_append_frames"
