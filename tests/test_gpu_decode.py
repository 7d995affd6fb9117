"""The decode kernel on the GPU: query sets of at most 4 rows per head (the causal camera head's
cache, one camera token per frame, and its joint prefill) attend on CUDA cores in one launch,
the key pages split across CTAs and merged by the last CTA of each head. Checked against the
CPU oracle for 1 to 4 query rows over streams that pass from one split to several, the joint
prefill of the scale frames, the no-allocation entry point, run-to-run bit equality, the
sticky error word, and the 5-row boundary where the tensor-core kernel takes over.
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


def _small(rows, frames=220, **kw):
    # `rows` special tokens per frame, no patch grid: `rows` query rows per head
    args = dict(num_special=rows, frames=frames, max_frames=frames, ring=32, num_pages=96,
                permuted_free_list=True, seed=40 + rows)
    args.update(kw)
    return gi.workload("camera4").replace(**args)


def _stream(w, checks, outs=None):
    cache = gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w))
    o = make_oracle(w)
    ring = gi.draw_ring(w).cuda()
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    q_rot = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q_rot)
    splits = set()
    for t in range(w.frames):
        q, k, v = ring[t % w.ring]
        cache.append_frame(t, q, k, v, q_rot)
        o.append(t)
        cache.attend(t, q_rot, out)
        info = cache.attend_info()
        assert info.launches == 1  # one launch: the splits merge inside it
        splits.add(info.split)
        if t in checks:
            torch.cuda.synchronize()
            check_book(cache, o.book, t)
            check_attention(out.double().cpu().numpy(), o.attend(t), f"rows={w.num_special} t={t}")
            if outs is not None:
                outs.append(out.clone())
    assert cache.check() == 0
    return splits


@pytest.mark.parametrize("rows", [1, 2, 3, 4])
def test_small_query_sets_match_the_oracle(rows):
    w = _small(rows)
    splits = _stream(w, {0, 1, 7, 15, 16, 17, 40, 129, w.frames - 1})
    assert splits == {0, 1}  # early frames in one CTA per head, later ones split and merged


def test_five_rows_take_the_tensor_core_kernel():
    w = _small(5, frames=60)
    _stream(w, {0, 16, 17, 59})


def test_decode_gives_the_same_bits_twice():
    w = _small(1, frames=300)
    checks = {150, 299}
    a, b = [], []
    _stream(w, checks, a)
    _stream(w, checks, b)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_camera_prefill_rows_match_the_oracle():
    # the joint attention of n scale frames with one camera token each: n query rows per head
    w = gi.workload("camera4").replace(anchor_frames=4, frames=4, max_frames=8, ring=8,
                                       num_pages=32, seed=47)
    for n in (2, 4):
        T, H, D = w.tokens_per_frame, w.num_heads, w.head_dim
        cache = gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w))
        o = make_oracle(w)
        ring = gi.draw_ring(w).cuda()
        q_all = torch.empty((n * T, H, D), dtype=torch.bfloat16, device="cuda")
        out_all = torch.empty_like(q_all)
        for t in range(n):
            q, k, v = ring[t % w.ring]
            cache.append_frame(t, q, k, v, q_all[t * T:(t + 1) * T])
            o.append(t)
        cache.attend_prefill(n, q_all, out_all)
        torch.cuda.synchronize()
        assert cache.attend_info().visible_keys == n * T
        check_attention(out_all.double().cpu().numpy(), o.attend_prefill(n, np.arange(n * T)),
                        f"camera prefill of {n} frames")
        assert cache.check() == 0


def test_noalloc_decode_matches_attend():
    w = _small(1, frames=120)
    cache = gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w))
    ring = gi.draw_ring(w).cuda()
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    q_rot = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    ref = torch.empty_like(q_rot)
    got = torch.empty_like(q_rot)
    stream = torch.cuda.current_stream().cuda_stream
    for t in range(w.frames):
        q, k, v = ring[t % w.ring]
        cache.append_frame(t, q, k, v, q_rot)
        if t in (3, 119):
            cache.attend(t, q_rot, ref)
            gca.gca_attend_noalloc(cache.handle, t, q_rot.data_ptr(), got.data_ptr(), stream)
            torch.cuda.synchronize()
            assert torch.equal(got, ref)  # the same launch, records in the library's array
    assert cache.check() == 0


def test_sticky_error_makes_decode_a_noop():
    w = _small(1, frames=4)
    free = torch.zeros(w.num_pages, dtype=torch.int32)  # not a permutation
    cache = gca.GcaCache(gca.config_for(w), initial_free=free)
    assert cache.check() == -6
    q, k, v = (x.cuda() for x in gi.draw_frame(w, 0))
    q_rot = torch.empty_like(q)
    out = torch.full_like(q, 3.0)
    cache.append_frame(0, q, k, v, q_rot)
    cache.attend(0, q_rot, out)
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())


def test_full_camera_stream_uses_eight_way_clusters():
    # 1,024 frames with K = 1: ~80 key pages per head, so the decode launch splits every head
    # over a full cluster of 8 CTAs
    w = gi.workload("camera4").replace(permuted_free_list=True, seed=48)
    cache = gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w))
    o = make_oracle(w)
    ring = gi.draw_ring(w).cuda()
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    q_rot = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q_rot)
    for t in range(w.frames):
        q, k, v = ring[t % w.ring]
        cache.append_frame(t, q, k, v, q_rot)
        o.append(t)
        if t in (511, w.frames - 1):
            cache.attend(t, q_rot, out)
            torch.cuda.synchronize()
            info = cache.attend_info()
            assert info.launches == 1
            if t == w.frames - 1:
                assert info.grid == 8 * w.num_heads
            check_book(cache, o.book, t)
            check_attention(out.double().cpu().numpy(), o.attend(t), f"camera t={t}")
    assert cache.check() == 0
