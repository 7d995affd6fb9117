"""gca_append_frames (one launch appending a frame to several caches) against per-cache appends.

The batched form must leave every cache bit-identical to the state its own gca_append_frame
calls produce: K/V pools, page tables, slot maps, free lists, trajectory pages and the rotated
queries. The caches differ in window, kept tokens, RoPE base, page budget and free-list order
(same tokens per frame and heads, as the entry point requires), so evictions, trajectory page
pops and free-list wraps happen at different frames in different caches of one launch. One
batched cache is also checked against the CPU oracle, and its attention against the oracle's.
"""
import numpy as np
import pytest
import torch

import gca_inputs as gi
import paged_kv_cache_gca_b200 as gca
from gca_testutil import check_attention, check_book, make_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_gca_b200 import build

    build.build()
    torch.cuda.init()


def _variants():
    base = gi.workload("w16_320").replace(frames=22, max_frames=24, ring=8)
    return [
        base.replace(window_frames=4, num_pages=420, seed=11),
        base.replace(anchor_frames=0, window_frames=3, keep_tokens=0, num_pages=270,
                     rope_base=14142.0, seed=12),
        base.replace(anchor_frames=2, window_frames=5, keep_tokens=20, num_pages=560,
                     permuted_free_list=True, seed=13),
        base.replace(window_frames=6, keep_tokens=7, num_pages=530, rope_base=20000.0,
                     permuted_free_list=True, seed=14),
    ]


def _caches(ws):
    return [gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w)) for w in ws]


def _snapshot(cache, t):
    """Device state after frame t (page-table rows of later frames are not yet written)."""
    v = cache.views()
    st = cache.state()
    return {
        "k": v["k_pool"].clone(), "v": v["v_pool"].clone(),
        "frame_pages": v["frame_pages"][:t + 1].clone(), "slot_map": v["slot_map"].clone(),
        "traj": v["traj_pages"].clone(), "free": cache.free_list(),
        "state": (st.frames_appended, st.free_head, st.free_tail, st.traj_len, st.traj_pages),
    }


def _same(a, b):
    for key in a:
        if isinstance(a[key], torch.Tensor):
            assert torch.equal(a[key].view(torch.int16) if a[key].dtype == torch.bfloat16
                               else a[key], b[key].view(torch.int16)
                               if b[key].dtype == torch.bfloat16 else b[key]), key
        else:
            assert a[key] == b[key], key


def test_batched_append_is_bit_identical_to_per_cache_appends():
    ws = _variants()
    single, batched = _caches(ws), _caches(ws)
    rings = [gi.draw_ring(w).cuda() for w in ws]
    shape = (ws[0].tokens_per_frame, ws[0].num_heads, ws[0].head_dim)
    qr_s = [torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in ws]
    qr_b = [torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in ws]
    stream = torch.cuda.current_stream().cuda_stream
    for t in range(ws[0].frames):
        frames = [r[t % 8] for r in rings]
        for c, f, qr in zip(single, frames, qr_s):
            c.append_frame(t, f[0], f[1], f[2], qr)
        gca.gca_append_frames([c.handle for c in batched], [t] * len(ws),
                              [f[0].data_ptr() for f in frames], [f[1].data_ptr() for f in frames],
                              [f[2].data_ptr() for f in frames], [q.data_ptr() for q in qr_b],
                              stream)
        for a, b in zip(qr_s, qr_b):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"q_rot t={t}"
        if t in (5, 13, ws[0].frames - 1):
            for cs, cb in zip(single, batched):
                _same(_snapshot(cs, t), _snapshot(cb, t))
    for c in single + batched:
        assert c.check() == 0

    # the permuted-free-list cache against the oracle (book bit-exact, attention in tolerance)
    w = ws[2]
    o = make_oracle(w)
    for t in range(w.frames):
        o.append(t)
    check_book(batched[2], o.book, w.frames - 1)
    out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    batched[2].attend(w.frames - 1, qr_b[2], out)
    torch.cuda.synchronize()
    rows = np.arange(0, w.tokens_per_frame, 7)
    check_attention(out.double().cpu().numpy()[rows], o.attend(w.frames - 1, rows),
                    "batched cache attend")


def test_batched_append_is_all_or_nothing():
    ws = _variants()[:3]
    caches = _caches(ws)
    shape = (ws[0].tokens_per_frame, ws[0].num_heads, ws[0].head_dim)
    x = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    qr = [torch.empty_like(x) for _ in ws]
    stream = torch.cuda.current_stream().cuda_stream

    def call(cs, frames):
        n = len(cs)
        gca.gca_append_frames([c.handle for c in cs], frames, [x.data_ptr()] * n,
                              [x.data_ptr()] * n, [x.data_ptr()] * n,
                              [q.data_ptr() for q in qr[:n]], stream)

    call(caches, [0, 0, 0])
    before = [c.state().frames_appended for c in caches]
    heads = [c.state().free_head for c in caches]
    with pytest.raises(gca.GcaError) as e:  # the second cache is asked for the wrong frame
        call(caches, [1, 2, 1])
    assert e.value.status == -3
    with pytest.raises(gca.GcaError) as e:  # the same cache twice
        call([caches[0], caches[1], caches[0]], [1, 1, 1])
    assert e.value.status == -1
    other = gca.GcaCache(gca.config_for(ws[0].replace(num_heads=8, num_pages=100)))
    with pytest.raises(gca.GcaError) as e:  # different head count
        call([caches[0], other], [1, 0])
    assert e.value.status == -1
    tight = gca.GcaCache(gca.config_for(ws[0].replace(num_pages=70)))
    call([tight], [0])
    with pytest.raises(gca.GcaError) as e:  # the last cache runs out of pages
        call([caches[0], caches[1], tight], [1, 1, 1])
    assert e.value.status == -2
    assert [c.state().frames_appended for c in caches] == before
    assert [c.state().free_head for c in caches] == heads
    call(caches, [1, 1, 1])  # still usable, in order
    torch.cuda.synchronize()
    assert [c.state().frames_appended for c in caches] == [2, 2, 2]
    for c in caches + [other, tight]:
        assert c.check() == 0
