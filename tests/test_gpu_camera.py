"""The causal camera head's cache on the GPU: one camera token per frame (grid 0 x 0), 32 heads,
the aggregator's window policy with K = 1, a RoPE base of its own -- the decode-like regime (one
query row per head, a few hundred to a thousand keys) -- against the CPU oracle.
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


@pytest.mark.parametrize("base", [10000.0, 100.0])
def test_camera_token_cache_matches_the_oracle(base):
    w = gi.workload("camera4").replace(frames=300, max_frames=300, ring=32, num_pages=60,
                                       rope_base=base, permuted_free_list=True, seed=31)
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
        if t == 0:
            torch.cuda.synchronize()
            assert torch.equal(out.view(torch.int16), v.view(torch.int16))  # one key: its v
        if t % 23 == 0 or t == w.frames - 1:
            torch.cuda.synchronize()
            assert cache.attend_info().visible_keys == t + 1  # every camera token so far
            check_book(cache, o.book, t)
            check_attention(out.double().cpu().numpy(), o.attend(t), f"camera t={t}")
    assert cache.check() == 0


def test_camera_trunk_caches_appended_in_one_launch():
    # the 4 layer caches of the camera trunk, appended together, attend like separate ones
    w = gi.workload("camera4").replace(frames=40, max_frames=40, ring=8, num_pages=40)
    n = w.num_layers
    caches = [gca.GcaCache(gca.config_for(w, rope_base=1000.0 * (l + 1))) for l in range(n)]
    oracles = [make_oracle(w, rope_base=1000.0 * (l + 1)) for l in range(n)]
    ring = gi.draw_ring(w).cuda()
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    qr = [torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for t in range(w.frames):
        f = ring[t % w.ring]
        gca.gca_append_frames([c.handle for c in caches], [t] * n, [f[0].data_ptr()] * n,
                              [f[1].data_ptr()] * n, [f[2].data_ptr()] * n,
                              [x.data_ptr() for x in qr], stream)
        for o in oracles:
            o.append(t)
    for l in range(n):
        caches[l].attend(w.frames - 1, qr[l], out)
        torch.cuda.synchronize()
        check_book(caches[l], oracles[l].book, w.frames - 1)
        check_attention(out.double().cpu().numpy(), oracles[l].attend(w.frames - 1),
                        f"layer {l}")
    assert all(c.check() == 0 for c in caches)
