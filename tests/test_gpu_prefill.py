"""Joint (bidirectional) attention of the scale frames on the GPU (gca_attend_prefill) against
the CPU oracle, then causal streaming on the same cache.

The first n <= A frames are appended, their q_rot written back to back into one [n*T, H, D]
buffer, and the n*T queries attend over every token of those frames with no mask across
frames. Checked on sampled rows of every frame; the last scale frame's rows also against the
causal gca_attend of that frame (same key set). The stream then continues causally (window,
eviction into the trajectory pool past the anchors) and is checked against the oracle.
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


@pytest.mark.parametrize("n", [8, 3])
def test_prefill_then_causal_stream_match_the_oracle(n):
    w = gi.workload("scale8").replace(frames=n + 22 if n == 8 else n, max_frames=32, ring=16,
                                      num_pages=1650)
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
    info = cache.attend_info()
    assert info.visible_keys == n * T and info.query_tiles == -(-n * T // 128)
    rows = np.arange(0, n * T, 13)
    check_attention(out_all.double().cpu().numpy()[rows], o.attend_prefill(n, rows),
                    f"prefill of {n} frames")
    # the last scale frame sees the same keys causally
    last = torch.empty((T, H, D), dtype=torch.bfloat16, device="cuda")
    cache.attend(n - 1, q_all[(n - 1) * T:], last)
    torch.cuda.synchronize()
    check_attention(out_all[(n - 1) * T:].double().cpu().numpy(), last.double().cpu().numpy(),
                    "prefill rows of the last scale frame vs its causal attention")

    q_rot = torch.empty((T, H, D), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q_rot)
    r1 = np.arange(0, T, 9)
    for t in range(n, w.frames):
        q, k, v = ring[t % w.ring]
        cache.append_frame(t, q, k, v, q_rot)
        o.append(t)
        cache.attend(t, q_rot, out)
        if t in (n, n + 16, w.frames - 1):
            torch.cuda.synchronize()
            check_book(cache, o.book, t)
            check_attention(out.double().cpu().numpy()[r1], o.attend(t, r1), f"causal t={t}")
    assert cache.check() == 0


def test_prefill_errors():
    w = gi.workload("scale8").replace(frames=2, max_frames=8, num_pages=600)
    T, H, D = w.tokens_per_frame, w.num_heads, w.head_dim
    cache = gca.GcaCache(gca.config_for(w))
    x = torch.zeros((T, H, D), dtype=torch.bfloat16, device="cuda")
    buf = torch.empty((9 * T, H, D), dtype=torch.bfloat16, device="cuda")
    res = torch.empty_like(buf)

    def status(n):
        with pytest.raises(gca.GcaError) as e:
            cache.attend_prefill(n, buf, res)
        return e.value.status

    assert status(1) == -3  # nothing appended yet
    cache.append_frame(0, x, x, x, buf[:T])
    cache.append_frame(1, x, x, x, buf[T:2 * T])
    assert status(0) == -1
    assert status(9) == -1  # more than the 8 anchor frames
    assert status(1) == -3  # two frames are appended
    cache.attend_prefill(2, buf, res)
    torch.cuda.synchronize()
    assert cache.check() == 0
