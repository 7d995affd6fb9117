"""Keyframe-only caching on the GPU (gca_append_frame_ex with GCA_APPEND_TRANSIENT, then
gca_attend, then gca_rollback_last_frame) against the CPU oracle's keyframe stream.

Non-keyframes append without evicting, attend over the cache plus themselves and roll back;
keyframes take the next cache frame. Every frame's page row, slot map, free list and
trajectory pages are compared bit-exactly with the oracle (before and after each rollback),
the attention of keyframes and non-keyframes within the attention tolerance, and the pool
contents of the live frames at the end (rollbacks must not disturb them).
"""
import numpy as np
import pytest
import torch

import gca_inputs as gi
import paged_kv_cache_gca_b200 as gca
from gca_testutil import check_attention, check_book, make_oracle
from test_gpu_parity import check_pool_contents

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_gca_b200 import build

    build.build()
    torch.cuda.init()


def _workload():
    return gi.workload("w16_320").replace(window_frames=4, frames=28, max_frames=32, ring=8,
                                          num_pages=420, permuted_free_list=True, seed=21)


@pytest.mark.parametrize("interval", [3, 1])
def test_keyframe_stream_matches_the_oracle(interval):
    w = _workload()
    cache = gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w))
    o = make_oracle(w)
    ring = gi.draw_ring(w).cuda()
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    q_rot = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q_rot)
    rows = np.arange(0, w.tokens_per_frame, 11)
    seen = {True: 0, False: 0}
    for g in range(w.frames):
        s = o.book.frames
        key = g % interval == 0
        q, k, v = ring[g % w.ring]
        cache.append_frame(s, q, k, v, q_rot, rope_frame=g, transient=not key)
        o.append(s, g, transient=not key)
        assert cache.state().transient == (0 if key else 1)
        cache.attend(s, q_rot, out)
        torch.cuda.synchronize()
        check_book(cache, o.book, s)
        assert cache.attend_info().visible_keys == len(o.visible(s))
        check_attention(out.double().cpu().numpy()[rows], o.attend(s, rows),
                        f"video frame {g} slot {s} key={key}")
        seen[key] += 1
        if not key:
            cache.rollback(s)
            o.rollback(s)
            st = cache.state()
            assert st.frames_appended == o.book.frames and st.transient == 0
            assert cache.free_list() == list(o.book.alloc.free)
    assert seen[True] > 0 and (interval == 1 or seen[False] > 0)
    check_pool_contents(cache, o, sorted(o.book.frame_pages))
    assert cache.check() == 0


def test_transient_frame_equals_a_frame_of_a_one_wider_window():
    w = _workload().replace(permuted_free_list=False, frames=10, num_pages=460)
    narrow = gca.GcaCache(gca.config_for(w))
    wide = gca.GcaCache(gca.config_for(w.replace(window_frames=w.window_frames + 1)))
    ring = gi.draw_ring(w).cuda()
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    qa, qb = (torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    oa, ob = torch.empty_like(qa), torch.empty_like(qa)
    for t in range(w.frames):
        q, k, v = ring[t % w.ring]
        wide.append_frame(t, q, k, v, qb)
        wide.attend(t, qb, ob)
        narrow.append_frame(t, q, k, v, qa, transient=True)
        narrow.attend(t, qa, oa)
        torch.cuda.synchronize()
        assert torch.equal(oa.view(torch.int16), ob.view(torch.int16)), f"frame {t}"
        narrow.rollback(t)
        narrow.append_frame(t, q, k, v, qa)
    assert narrow.check() == 0 and wide.check() == 0


def test_rollback_and_transient_errors():
    w = _workload().replace(frames=4)
    cache = gca.GcaCache(gca.config_for(w))
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    x = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    qr = torch.empty_like(x)

    def status(fn, *a):
        with pytest.raises(gca.GcaError) as e:
            fn(*a)
        return e.value.status

    cache.append_frame(0, x, x, x, qr)
    assert status(cache.rollback, 0) == -3  # a kept frame does not roll back
    p = x.data_ptr()
    assert status(gca.gca_append_frame_ex, cache.handle, 1, 1, 2, p, p, p, p, None) == -1
    assert status(gca.gca_append_frame_ex, cache.handle, 1, w.max_frames, 0, p, p, p, p,
                  None) == -1  # no RoPE row for that position
    cache.append_frame(1, x, x, x, qr, rope_frame=7, transient=True)
    assert status(cache.append_frame, 2, x, x, x, qr) == -3  # rollback first
    assert status(cache.rollback, 0) == -3  # wrong frame
    before = cache.state()
    cache.rollback(1)
    after = cache.state()
    assert after.frames_appended == 1 and after.free_head == before.free_head - 63
    cache.append_frame(1, x, x, x, qr, transient=True)
    cache.reset()
    st = cache.state()
    assert st.transient == 0 and st.frames_appended == 0
    cache.append_frame(0, x, x, x, qr)
    torch.cuda.synchronize()
    assert cache.check() == 0
