"""The attention kernel's bounded waits, made to run out without faulting anything.

gca_test_withhold_copies arms the next attention launch so that its CTA 0 never issues the copies
of its first key tile (nothing is in flight for that tile at any time). With a short wait limit
(gca_set_wait_limit) that CTA's MMA issuer gives up, the kernel records GCA_DEVERR_WAIT_TIMEOUT in
the cache's sticky error word, every CTA winds down (copies and MMAs it issued are waited for,
tensor memory is freed) and the call ends. The combine launch sees the sticky word and writes
nothing, so the output (every work unit of a full-size frame is split across CTAs) is untouched;
gca_check reports the error, and after gca_reset the cache streams exactly as a fresh one.
"""
import pytest
import torch

import gca_inputs as gi
import paged_kv_cache_gca_b200 as gca
from gca_testutil import device_ring

pytestmark = pytest.mark.gpu

TIMEOUT_BIT = 0x2


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_gca_b200 import build

    build.build()
    torch.cuda.init()


def _outputs(cache, ring, w, frames, q_rot, out):
    res = []
    for t in range(frames):
        q, k, v = ring[t % w.ring]
        cache.append_frame(t, q, k, v, q_rot)
        cache.attend(t, q_rot, out)
        res.append(out.clone())
    torch.cuda.synchronize()
    return res


def test_wait_runs_out_reports_and_the_cache_recovers():
    w = gi.workload("w16_320").replace(frames=24, max_frames=24)
    ring = device_ring(w)
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    q_rot = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q_rot)

    fresh = gca.GcaCache(gca.config_for(w))
    ref = _outputs(fresh, ring, w, 20, q_rot, out)
    assert fresh.check() == 0

    cache = gca.GcaCache(gca.config_for(w))
    for t in range(19):
        q, k, v = ring[t % w.ring]
        cache.append_frame(t, q, k, v, q_rot)
        cache.attend(t, q_rot, out)
    q, k, v = ring[19 % w.ring]
    cache.append_frame(19, q, k, v, q_rot)
    torch.cuda.synchronize()
    assert cache.check() == 0
    sentinel = torch.full_like(out, 7.0)
    gca.gca_set_wait_limit(cache.handle, 1_000_000)  # 1 ms
    gca.gca_test_withhold_copies(cache.handle)
    cache.attend(19, q_rot, sentinel)
    gca.gca_set_wait_limit(cache.handle, 0)  # back to the default bound
    assert cache.attend_info().split == 1  # every unit split: all rows go through the combine
    torch.cuda.synchronize()  # the call ends (bounded waits)
    assert cache.check() == -6
    assert cache.state().device_error & TIMEOUT_BIT
    assert bool((sentinel == 7.0).all())  # nothing written
    # the sticky word keeps later attentions from writing until reset
    cache.attend(19, q_rot, sentinel)
    torch.cuda.synchronize()
    assert bool((sentinel == 7.0).all())

    cache.reset()
    again = _outputs(cache, ring, w, 20, q_rot, out)
    assert cache.check() == 0
    for t in range(20):
        assert torch.equal(again[t], ref[t]), t
