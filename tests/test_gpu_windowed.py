"""Windowed restart on the GPU (paged_kv_cache_gca_b200.windowed over gca_reset + appends with
local frame indices) against the oracle's windowed stream (reading R14)."""
import numpy as np
import pytest
import torch

import gca_inputs as gi
import oracle as orc
import paged_kv_cache_gca_b200 as gca
from gca_testutil import check_attention, check_book, make_oracle
from paged_kv_cache_gca_b200 import windowed

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_gca_b200 import build

    build.build()
    torch.cuda.init()


def test_windowed_stream_matches_the_oracle():
    N, V, total = 16, 4, 40
    w = gi.workload("w16_320").replace(window_frames=4, max_frames=N, ring=8, num_pages=420,
                                       permuted_free_list=True, seed=41)
    cache = gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w))
    drv = windowed.WindowedStream(cache, N, V)
    o = make_oracle(w)
    ring = gi.draw_ring(w).cuda()
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    q_rot = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q_rot)
    rows = np.arange(0, w.tokens_per_frame, 17)
    checked = 0
    for win, g, loc in orc.windowed_frames(total, N, V):
        q, k, v = ring[g % w.ring]
        drv.step(loc, q, k, v, q_rot, out)
        if loc == 0:
            o.restart()
        o.append(loc, g, rope_pos=loc)
        if loc in (0, V, N - 1) or g == total - 1:
            torch.cuda.synchronize()
            check_book(cache, o.book, loc)
            check_attention(out.double().cpu().numpy()[rows], o.attend(loc, rows),
                            f"window {win} frame {g} local {loc}")
            checked += 1
    assert checked >= 8
    assert cache.check() == 0
