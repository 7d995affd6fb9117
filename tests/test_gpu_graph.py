"""The hot path under CUDA graph capture: one frame's gca_append_frame + gca_attend captured
into a graph (their launches carry programmatic-serialization attributes, which capture turns
into programmatic graph edges), replayed once, and compared bit-for-bit with a cache that ran
the same frame eagerly. The host mirror advances at capture time, so a captured frame is
replayed once (a graph of a fixed frame)."""
import pytest
import torch

import gca_inputs as gi
import paged_kv_cache_gca_b200 as gca

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_gca_b200 import build

    build.build()
    torch.cuda.init()


def test_captured_frame_matches_eager():
    w = gi.workload("w16_320").replace(window_frames=4, frames=24, max_frames=24, ring=8,
                                       num_pages=600)
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    ring = gi.draw_ring(w).cuda()
    eager, graphed = gca.GcaCache(gca.config_for(w)), gca.GcaCache(gca.config_for(w))
    qa, qb = (torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    oa, ob = torch.empty_like(qa), torch.empty_like(qa)
    last = w.frames - 1
    for t in range(last):  # both caches past the window (frame 23 evicts frame 19)
        q, k, v = ring[t % w.ring]
        for c, qr, o in ((eager, qa, oa), (graphed, qb, ob)):
            c.append_frame(t, q, k, v, qr)
            c.attend(t, qr, o)
    torch.cuda.synchronize()
    q, k, v = ring[last % w.ring]
    eager.append_frame(last, q, k, v, qa)
    eager.attend(last, qa, oa)
    g = torch.cuda.CUDAGraph()
    ob.zero_()
    with torch.cuda.graph(g):
        graphed.append_frame(last, q, k, v, qb)
        graphed.attend(last, qb, ob)
    torch.cuda.synchronize()
    assert not ob.any()  # capture alone runs nothing
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(ob.view(torch.int16), oa.view(torch.int16))
    assert torch.equal(qb.view(torch.int16), qa.view(torch.int16))
    assert graphed.state().frames_appended == eager.state().frames_appended
    assert graphed.free_list() == eager.free_list()
    assert graphed.check() == 0 and eager.check() == 0
