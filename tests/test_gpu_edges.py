"""Edge configurations on the GPU, each against the CPU oracle (book bit-exact, attention within
the stated bar): the largest head count on both attention kernels, the largest number of kept
tokens per evicted frame, a history made only of the trajectory pool (no anchors, a window of
one frame), ragged query tiles (a last tile of one row; a tile pair whose second tile is past
the frame), and a page pool exactly as large as the stream's peak need, so that the FIFO
allocator hands every freed page out again within a few frames ("How the Geometric Context
Transformer Enables Streaming 3D Reconstruction in LingBot-Map", KV-Cache Initialization and
FlashInferBlock; "LingBot-Map runs 10,000 frames on monocular video", the three pools).
"""
import numpy as np
import pytest
import torch

import gca_inputs as gi
import oracle.gca_oracle as orc
import paged_kv_cache_gca_b200 as gca
from gca_testutil import check_attention, check_book, make_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_gca_b200 import build

    build.build()
    torch.cuda.init()


def _base(**kw):
    args = dict(name="edge", num_heads=4, head_dim=64, page_size=16, grid_h=8, grid_w=8,
                num_special=4, anchor_frames=1, window_frames=4, keep_tokens=4, frames=40,
                seed=91, value_scale=0.5, permuted_free_list=True, ring=16, num_pages=400,
                max_frames=None)
    args.update(kw)
    if args["max_frames"] is None:  # RoPE table as long as the stream
        args["max_frames"] = args["frames"]
    return gi.Workload(**args)


def _peak_pages(w):
    """Pages the stream needs at its busiest step: the ones in use before the step plus the
    step's pops (the new frame's pages, then new trajectory pages; the evicted frame's pages
    return to the free list only after them)."""
    book = orc.CacheBook(T=w.tokens_per_frame, page_size=w.page_size,
                         anchor_frames=w.anchor_frames, window_frames=w.window_frames,
                         kept=orc.kept_token_indices(w.num_special, w.grid_h * w.grid_w,
                                                     w.keep_tokens),
                         initial_free=list(range(100000)))
    need = 0
    for t in range(w.frames):
        before, traj_before = book.pages_in_use(), len(book.traj_pages)
        book.append(t)
        need = max(need, before + book.ppf + len(book.traj_pages) - traj_before)
    return need


def _stream(w, checks, rows=None):
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
        cache.attend(t, q_rot, out)
        if t in checks:
            torch.cuda.synchronize()
            check_book(cache, o.book, t)
            r = None if rows is None else np.asarray(rows)
            got = out.double().cpu().numpy() if r is None else out.double().cpu().numpy()[r]
            check_attention(got, o.attend(t, r), f"{w.name} t={t}")
    assert cache.check() == 0
    return cache


def test_64_heads_tensor_core_kernel():
    w = _base(name="h64", num_heads=64, frames=30)
    _stream(w, {0, 4, 5, 29}, rows=np.arange(0, 68, 5))


def test_64_heads_decode_kernel():
    w = _base(name="h64_decode", num_heads=64, grid_h=0, grid_w=0, num_special=1,
              keep_tokens=1, window_frames=8, frames=160, num_pages=200)
    _stream(w, {0, 8, 9, 100, 159})


def test_64_kept_tokens_per_evicted_frame():
    w = _base(name="k64", keep_tokens=64, window_frames=3, frames=30, num_pages=600)
    _stream(w, {3, 4, 5, 29}, rows=np.arange(0, 68, 3))


def test_history_from_the_trajectory_pool_only():
    # no anchor frames and a window of one frame: every frame attends over itself and the
    # trajectory pool only
    w = _base(name="traj_only", anchor_frames=0, window_frames=1, keep_tokens=6, frames=40)
    _stream(w, {0, 1, 2, 17, 39})


@pytest.mark.parametrize("grid", [(8, 16), (16, 16)])
def test_ragged_query_tiles(grid):
    # T = 129: the second 128-row tile holds one row; T = 257: three tiles, so the second pair
    # of tiles has one tile past the frame
    w = _base(name=f"ragged{grid[0] * grid[1] + 1}", grid_h=grid[0], grid_w=grid[1],
              num_special=1, keep_tokens=3, window_frames=3, frames=14, num_pages=300)
    T = w.tokens_per_frame
    rows = sorted({0, 1, 126, 127, 128, T - 2, T - 1})
    _stream(w, {0, 3, 4, 13}, rows=rows)


def test_pool_exactly_as_large_as_the_peak_need():
    w = _base(name="tight", frames=60)
    w = w.replace(num_pages=_peak_pages(w))
    cache = _stream(w, {10, 30, 59})
    # one page fewer does not fit: the library says so before enqueueing anything
    w2 = w.replace(num_pages=w.num_pages - 1)
    c2 = gca.GcaCache(gca.config_for(w2), initial_free=gi.initial_free_list(w2))
    ring = gi.draw_ring(w2).cuda()
    q_rot = torch.empty((w2.tokens_per_frame, w2.num_heads, w2.head_dim), dtype=torch.bfloat16,
                        device="cuda")
    with pytest.raises(gca.GcaError) as e:
        for t in range(w2.frames):
            q, k, v = ring[t % w2.ring]
            c2.append_frame(t, q, k, v, q_rot)
    assert e.value.status == -2  # GCA_ERR_OUT_OF_PAGES
    assert c2.check() == 0
    assert cache.state().pages_in_use <= w.num_pages
