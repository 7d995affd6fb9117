"""gca_append_attend -- a frame's append (RoPE, paged scatter, eviction) and its attention in one
launch -- against the CPU oracle and against the two separate calls.

The fused launch must leave exactly the state gca_append_frame leaves (page tables, slot maps,
free list, trajectory list and pool contents, bit for bit: "How the Geometric Context Transformer
Enables Streaming 3D Reconstruction in LingBot-Map", FlashInferBlock: append_frame, then
evict_frames) and produce the frame's attention over its three pools ("LingBot-Map runs 10,000
frames on monocular video", section "How GCT's Anchor-Pose-Trajectory Pools Make Monocular 3D
Tractable") within the attention tolerance.
"""
import numpy as np
import pytest
import torch

import gca_inputs as gi
import paged_kv_cache_gca_b200 as gca
from gca_testutil import check_attention, check_book, device_ring, make_oracle
from test_gpu_parity import check_pool_contents

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_gca_b200 import build

    build.build()
    torch.cuda.init()


def _np(x):
    return x.double().cpu().numpy()


def _out(w):
    return torch.empty((w.tokens_per_frame, w.num_heads, w.head_dim), dtype=torch.bfloat16,
                       device="cuda")


def test_tiny_fused_every_frame_everything():
    w = gi.workload("tiny")
    cache = gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w))
    o = make_oracle(w)
    ring = device_ring(w)
    out = _out(w)
    for t in range(w.frames):
        q, k, v = ring[t % w.ring]
        cache.append_attend(t, q, k, v, out)
        torch.cuda.synchronize()
        o.append(t)
        check_book(cache, o.book, t)
        check_pool_contents(cache, o, range(t + 1))
        check_attention(_np(out), o.attend(t), f"tiny fused t={t}")
    assert cache.check() == 0


def test_w16_320_fused_full_stream_sampled_frames():
    w = gi.workload("w16_320")
    cache = gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w))
    o = make_oracle(w)
    ring = device_ring(w)
    out = _out(w)
    samples = {0, 1, 15, 16, 17, 18, 101, 250, 319}
    for t in range(w.frames):
        q, k, v = ring[t % w.ring]
        cache.append_attend(t, q, k, v, out)
        o.append(t)
        if t in samples:
            torch.cuda.synchronize()
            check_book(cache, o.book, t)
            check_pool_contents(cache, o, [t])
            check_attention(_np(out), o.attend(t), f"w16_320 fused t={t}")
    assert cache.check() == 0


def test_fused_state_is_bit_identical_to_separate_calls():
    w = gi.workload("w64_1000").replace(frames=90, max_frames=90)  # fragmented free list
    ring = device_ring(w)
    free = gi.initial_free_list(w)
    sep = gca.GcaCache(gca.config_for(w), initial_free=free)
    fus = gca.GcaCache(gca.config_for(w), initial_free=free)
    q_rot, out_s, out_f = _out(w), _out(w), _out(w)
    for t in range(w.frames):
        q, k, v = ring[t % w.ring]
        sep.append_frame(t, q, k, v, q_rot)
        sep.attend(t, q_rot, out_s)
        fus.append_attend(t, q, k, v, out_f)
        if t % 7 == 0 or t == w.frames - 1:
            torch.cuda.synchronize()
            # outputs: same keys, another order of key tiles -> rounding only
            d = (out_s.float() - out_f.float()).abs()
            assert d.max().item() <= 4e-3, (t, d.max().item())
    torch.cuda.synchronize()
    vs, vf = sep.views(), fus.views()
    for name in ("k_pool", "v_pool", "free_ring", "frame_pages", "traj_pages", "slot_map"):
        assert torch.equal(vs[name], vf[name]), name
    assert sep.free_list() == fus.free_list()
    assert sep.check() == 0 and fus.check() == 0


def test_fused_long_trajectory_with_needles():
    # the 10,000-frame layer on a 1,200-frame stream: ~14k trajectory tokens split over CTAs;
    # needles make rows rescale late and the combine merge far-apart maxima
    w = gi.workload("w32_10k").replace(frames=1200, value_scale=1.0, needle_every=11,
                                       needle_slot=5, needle_q_gain=8.0, needle_k_gain=16.0)
    cache = gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w))
    o = make_oracle(w)
    ring = device_ring(w)
    out = _out(w)
    rng = np.random.default_rng(9)
    samples = {33, 600, 1198, 1199}
    for t in range(w.frames):
        q, k, v = ring[t % w.ring]
        cache.append_attend(t, q, k, v, out)
        o.append(t)
        if t in samples:
            torch.cuda.synchronize()
            check_book(cache, o.book, t)
            rows = np.sort(rng.choice(w.tokens_per_frame, 64, False))
            gpu = _np(out[torch.as_tensor(rows, device="cuda")])
            ref = o.attend(t, rows)
            d = np.abs(gpu - ref)
            # unit-scale values: the absolute bars scale with the values (8x the workloads')
            assert d.max() <= 0.16 and d.mean() <= 0.016, (t, d.max(), d.mean())
            rel = np.linalg.norm(gpu - ref) / np.linalg.norm(ref)
            assert rel <= 1e-2, (t, rel)
    cnt = cache.counters()
    assert cnt.rescaled_rows > 0 and cnt.wide_merge_rows > 0
    assert cache.check() == 0


def test_fused_mixed_with_separate_calls_and_reset():
    w = gi.workload("w16_320").replace(frames=40, max_frames=40)
    ring = device_ring(w)
    cache = gca.GcaCache(gca.config_for(w))
    o = make_oracle(w)
    q_rot, out = _out(w), _out(w)
    checked = (0, 17, 18, 39)
    first = {}
    for rep in range(2):
        for t in range(w.frames):
            q, k, v = ring[t % w.ring]
            if t % 3 == 1:
                cache.append_frame(t, q, k, v, q_rot)
                cache.attend(t, q_rot, out)
            else:
                cache.append_attend(t, q, k, v, out)
            if rep == 0:
                o.append(t)
            if t in checked:
                torch.cuda.synchronize()
                if rep == 0:
                    check_book(cache, o.book, t)
                    check_attention(_np(out), o.attend(t), f"mixed t={t}")
                    first[t] = out.clone()
                else:  # the same calls after gca_reset: the same bits
                    assert torch.equal(out, first[t]), t
        cache.reset()
    assert cache.check() == 0


def test_fused_on_concurrent_streams():
    # 4 streams x 6 caches, every cache fused on its stream's queue: launches of different
    # streams may share the GPU; each completes on its own (no launch waits for another)
    w = gi.workload("stack24x4").replace(frames=30, max_frames=30)
    ring = device_ring(w)
    streams = [torch.cuda.Stream() for _ in range(4)]
    caches, outs = {}, {}
    for s in range(4):
        with torch.cuda.stream(streams[s]):
            for layer in range(6):
                caches[s, layer] = gca.GcaCache(
                    gca.config_for(w, gi.rope_base_for_layer(w, layer)), stream=streams[s])
                outs[s, layer] = _out(w)
    for t in range(w.frames):
        for s in range(4):
            q, k, v = ring[(4 * t + s) % w.ring]
            for layer in range(6):
                caches[s, layer].append_attend(t, q, k, v, outs[s, layer], stream=streams[s])
    torch.cuda.synchronize()
    for (s, layer), c in caches.items():
        assert c.check() == 0
    # cache (1, 3) against the oracle at the last frame
    o = make_oracle(w, rope_base=gi.rope_base_for_layer(w, 3),
                    source=lambda t: gi.draw_frame(w, 4 * t + 1))
    for t in range(w.frames):
        o.append(t)
    check_attention(_np(outs[1, 3]), o.attend(w.frames - 1), "stream 1 layer 3")


def test_fused_rejects_bad_arguments():
    w = gi.workload("tiny")
    cache = gca.GcaCache(gca.config_for(w))
    q, k, v = (x.cuda() for x in gi.draw_frame(w, 0))
    for bad_out in (q, k, v):
        with pytest.raises(gca.GcaError) as e:
            cache.append_attend(0, q, k, v, bad_out)
        assert e.value.status == -1
    out = torch.empty_like(q)
    with pytest.raises(gca.GcaError) as e:
        cache.append_attend(1, q, k, v, out)
    assert e.value.status == -3
    assert cache.state().frames_appended == 0
    cache.append_attend(0, q, k, v, out)
    torch.cuda.synchronize()
    assert cache.check() == 0
