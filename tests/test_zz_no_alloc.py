"""gca_attend_noalloc, the attention entry point that allocates nothing, against gca_attend.

Some callers may not allocate device memory while they run: a process that budgets all GPU
memory at start-up, a plugin whose host application owns the device allocator, or a loop where
a cudaMalloc could synchronise the device. gca_attend_noalloc serves them by keeping its
scratch (the split-KV partial records) in a fixed array inside the library. These tests call it
through the C ABI, twice in a row, and compare with gca_attend within the attention tolerance
the other tests use. The file name makes pytest collect it last.
"""
import numpy as np
import pytest
import torch

import gca_inputs as gi
import paged_kv_cache_gca_b200 as gca
from gca_testutil import check_attention, device_ring

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_gca_b200 import build

    build.build()


def test_noalloc_matches_attend_on_two_calls_in_a_row():
    w = gi.workload("w16_320").replace(frames=48, max_frames=48)
    cache = gca.GcaCache(gca.config_for(w))
    ring = device_ring(w)
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    q_rot = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    ref = torch.empty_like(q_rot)
    got = [torch.empty_like(q_rot), torch.empty_like(q_rot)]
    stream = torch.cuda.current_stream().cuda_stream
    checked = split = 0
    for t in range(w.frames):
        q, k, v = ring[t % w.ring]
        cache.append_frame(t, q, k, v, q_rot)
        if t in (0, 17, w.frames - 1):
            cache.attend(t, q_rot, ref)
            # gca_attend_noalloc plans the same launch (the same grid here: the scratch holds
            # every record this config needs), so gca_attend's info tells whether the key
            # ranges were split, i.e. whether the call went through the library's array
            split += cache.attend_info().split
            if t == 0:
                # set-up call: the first call on a device looks up the array's address, and
                # CUDA's lazy module loading commits the array's 16 MiB at that moment
                gca.gca_attend_noalloc(cache.handle, t, q_rot.data_ptr(), got[0].data_ptr(),
                                       stream)
            torch.cuda.synchronize()
            free_before = torch.cuda.mem_get_info()[0]
            for g in got:  # two calls in a row share (and reuse) the library's scratch array
                gca.gca_attend_noalloc(cache.handle, t, q_rot.data_ptr(), g.data_ptr(), stream)
            torch.cuda.synchronize()
            assert torch.cuda.mem_get_info()[0] == free_before  # nothing was allocated
            r = ref.double().cpu().numpy()
            for g in got:
                check_attention(g.double().cpu().numpy(), r, f"noalloc t={t}")
            checked += 1
    assert checked == 3
    assert split >= 2  # frames 17 and 47 split their key ranges: the combine read the array
    assert cache.check() == 0


def test_noalloc_rejects_frames_beyond_its_scratch():
    # 64 heads x 4 pairs of query tiles need 2 x 256 partial records at least: the array holds 496
    w = gi.workload("w16_320").replace(num_heads=64, num_pages=64, frames=1, max_frames=4)
    cache = gca.GcaCache(gca.config_for(w))
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    q = torch.randn(shape, device="cuda").to(torch.bfloat16)
    q_rot = torch.empty_like(q)
    out = torch.empty_like(q)
    cache.append_frame(0, q, q, q, q_rot)
    with pytest.raises(gca.GcaError) as e:
        gca.gca_attend_noalloc(cache.handle, 0, q_rot.data_ptr(), out.data_ptr(),
                               torch.cuda.current_stream().cuda_stream)
    assert e.value.status == -5
    cache.attend(0, q_rot, out)  # the workspace path still serves this config
    torch.cuda.synchronize()
    assert cache.check() == 0
    assert torch.isfinite(out.float()).all()
