"""GPU path (through the C ABI) against the CPU oracle.

Page tables, slot maps, free lists and trajectory pages are compared bit-exactly; rotated
q/k within one bf16 rounding; v copies bit-exactly; attention within max abs 2e-2, mean abs
2e-3 and a relative-error bound (gca_testutil). The full-size workloads run in the same launch
configuration the benchmark times and are checked on sampled frames and rows.
"""
import numpy as np
import pytest
import torch

import gca_inputs as gi
import oracle as orc
import paged_kv_cache_gca_b200 as gca
from gca_testutil import (bf16_close, check_attention, check_book, device_ring, make_oracle)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_gca_b200 import build

    build.build()
    torch.cuda.init()


def _bufs(w):
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    return (torch.empty(shape, dtype=torch.bfloat16, device="cuda"),
            torch.empty(shape, dtype=torch.bfloat16, device="cuda"))


def _np(x):
    return x.double().cpu().numpy()


def check_pool_contents(cache, o, frames):
    """Every live token of `frames` and every trajectory token sits at its (page, slot)."""
    v = cache.views()
    kp, vp = v["k_pool"], v["v_pool"]
    for f in frames:
        if f not in o.book.frame_pages:
            continue
        row = torch.tensor(o.book.frame_pages[f], device="cuda")
        toks = torch.arange(o.T, device="cuda")
        pages, slots = row[toks // o.ps], toks % o.ps
        k_gpu = _np(kp[pages, :, slots, :])
        v_gpu = vp[pages, :, slots, :].cpu()
        assert bf16_close(k_gpu, o.k_rot(f)), f"k_rot of frame {f}"
        raw_v = o.raw32(f)[2]
        assert np.array_equal(v_gpu.float().numpy(), raw_v), f"v of frame {f}"
    if o.book.traj_len:
        n = np.arange(o.book.traj_len)
        pages = torch.tensor([o.book.traj_pages[i // o.ps] for i in n], device="cuda")
        slots = torch.tensor(n % o.ps, device="cuda")
        k_gpu = _np(kp[pages, :, slots, :])
        v_gpu = vp[pages, :, slots, :].float().cpu().numpy()
        for idx, (e, tok) in enumerate(o.book.traj_tokens):
            assert bf16_close(k_gpu[idx], o.k_rot(e, [tok])[0]), ("traj k", idx)
            assert np.array_equal(v_gpu[idx], o.raw32(e)[2][tok]), ("traj v", idx)


def test_tiny_stream_everything_every_frame():
    w = gi.workload("tiny")
    cache = gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w))
    o = make_oracle(w)
    ring = device_ring(w)
    q_rot, out = _bufs(w)
    for t in range(w.frames):
        q, k, v = ring[t % w.ring]
        cache.append_frame(t, q, k, v, q_rot)
        cache.attend(t, q_rot, out)
        torch.cuda.synchronize()
        o.append(t)
        check_book(cache, o.book, t)
        assert bf16_close(_np(q_rot), o.q_rot(t))
        check_pool_contents(cache, o, range(t + 1))
        check_attention(_np(out), o.attend(t), f"tiny t={t}")
    assert cache.check() == 0


def test_reset_restores_a_new_stream():
    w = gi.workload("tiny")
    cache = gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w))
    ring = device_ring(w)
    q_rot, out = _bufs(w)
    outs = []
    for rep in range(2):
        for t in range(w.frames):
            q, k, v = ring[t % w.ring]
            cache.append_frame(t, q, k, v, q_rot)
            cache.attend(t, q_rot, out)
        torch.cuda.synchronize()
        outs.append(out.clone())
        cache.reset()
    assert torch.equal(outs[0], outs[1])
    assert cache.free_list() == gi.initial_free_list(w).tolist()


def _sampled_frames(w, extra, seed):
    A, W, n = w.anchor_frames, w.window_frames, w.frames
    base = {0, A, A + W - 1, A + W, A + W + 1, n - 1}
    rng = np.random.default_rng(seed)
    base |= set(int(x) for x in rng.integers(0, n, size=extra))
    return sorted(t for t in base if 0 <= t < n)


def _stream_and_check(name, rows=None, extra=4, pool_check=False):
    w = gi.workload(name)
    free = gi.initial_free_list(w)
    cache = gca.GcaCache(gca.config_for(w), initial_free=free)
    o = make_oracle(w)
    ring = device_ring(w)
    q_rot, out = _bufs(w)
    samples = set(_sampled_frames(w, extra, w.seed))
    rng = np.random.default_rng(100 + w.seed)
    worst = []
    for t in range(w.frames):
        q, k, v = ring[t % w.ring]
        cache.append_frame(t, q, k, v, q_rot)
        cache.attend(t, q_rot, out)
        o.append(t)
        if t in samples:
            torch.cuda.synchronize()
            check_book(cache, o.book, t)
            r = None if rows is None else np.sort(rng.choice(w.tokens_per_frame, rows, False))
            gpu = _np(out) if r is None else _np(out[torch.as_tensor(r, device="cuda")])
            worst.append(check_attention(gpu, o.attend(t, r), f"{name} t={t}"))
            if pool_check:
                check_pool_contents(cache, o, [t])
    assert cache.check() == 0
    return worst


def test_w16_320_full_stream_sampled_frames():
    _stream_and_check("w16_320", rows=None, extra=4, pool_check=True)


def test_w64_1000_fragmented_pool_sampled_frames():
    _stream_and_check("w64_1000", rows=64, extra=3)


def test_w32_10k_long_trajectory_split_kv():
    _stream_and_check("w32_10k", rows=64, extra=2)


def test_stack_24_layers_4_streams():
    w = gi.workload("stack24x4")
    T, H, D = w.tokens_per_frame, w.num_heads, w.head_dim
    ring = device_ring(w)
    streams = [torch.cuda.Stream() for _ in range(w.num_streams)]
    caches, bufs = {}, {}
    for s in range(w.num_streams):
        with torch.cuda.stream(streams[s]):
            for layer in range(w.num_layers):
                base = gi.rope_base_for_layer(w, layer)
                caches[s, layer] = gca.GcaCache(gca.config_for(w, rope_base=base),
                                                stream=streams[s])
                bufs[s, layer] = _bufs(w)
    checked = [(0, 0), (1, 7), (3, 23)]
    sample_t = [0, 11, 12, 13, 250, w.frames - 1]
    saved = {}
    for t in range(w.frames):
        for s in range(w.num_streams):
            with torch.cuda.stream(streams[s]):
                q, k, v = ring[t % w.ring]
                for layer in range(w.num_layers):
                    c = caches[s, layer]
                    q_rot, out = bufs[s, layer]
                    c.append_frame(t, q, k, v, q_rot, stream=streams[s])
                    c.attend(t, q_rot, out, stream=streams[s])
                    if (s, layer) in checked and t in sample_t:
                        saved[s, layer, t] = out.clone()
    torch.cuda.synchronize()
    rng = np.random.default_rng(7)
    for s, layer in checked:
        o = make_oracle(w, rope_base=gi.rope_base_for_layer(w, layer))
        for t in range(w.frames):
            o.append(t)
            if t in sample_t:
                rows = np.sort(rng.choice(T, 64, False))
                gpu = _np(saved[s, layer, t][torch.as_tensor(rows, device="cuda")])
                check_attention(gpu, o.attend(t, rows), f"stack s={s} l={layer} t={t}")
        assert caches[s, layer].check() == 0


def _custom_source(frames):
    return lambda t: frames[t]


def _run_custom(wl, frames, initial_free=None, rope_base=None):
    """Stream explicit frames (dict t -> (q,k,v) bf16 CPU) through a cache; outputs per frame."""
    cache = gca.GcaCache(gca.config_for(wl, rope_base), initial_free=initial_free)
    q_rot, out = _bufs(wl)
    outs = []
    for t in range(len(frames)):
        q, k, v = (x.cuda() for x in frames[t])
        cache.append_frame(t, q, k, v, q_rot)
        cache.attend(t, q_rot, out)
        outs.append(out.clone())
    torch.cuda.synchronize()
    assert cache.check() == 0
    return cache, outs


def test_single_key_returns_v_exactly():
    wl = gi.Workload(name="one", num_heads=4, head_dim=64, page_size=16, grid_h=1, grid_w=1,
                     num_special=0, anchor_frames=0, window_frames=1, keep_tokens=0, frames=5,
                     seed=11, value_scale=1.0, permuted_free_list=False, ring=5, num_pages=4,
                     max_frames=8)
    frames = {t: gi.draw_frame(wl, t) for t in range(wl.frames)}
    _, outs = _run_custom(wl, frames)
    for t in range(wl.frames):
        assert torch.equal(outs[t].cpu(), frames[t][2])


def test_page_permutation_gives_identical_bits():
    w = gi.workload("tiny")
    frames = {t: gi.draw_frame(w, t) for t in range(w.frames)}
    results = []
    for seed in (None, 5, 9):
        free = (torch.arange(w.num_pages, dtype=torch.int32) if seed is None
                else gi.initial_free_list(w, seed=seed))
        _, outs = _run_custom(w, frames, initial_free=free)
        results.append(outs)
    for outs in results[1:]:
        for a, b in zip(results[0], outs):
            assert torch.equal(a, b)


@pytest.mark.parametrize("pool", ["anchor", "window", "trajectory"])
def test_needle_in_each_pool(pool):
    w = gi.workload("tiny")
    T = w.tokens_per_frame
    frames = {t: tuple(x.clone() for x in gi.draw_frame(w, t)) for t in range(w.frames)}
    o0 = make_oracle(w)
    t, row, h = 5, 40, 1
    frame, token = {"anchor": (0, 9), "window": (4, 30), "trajectory": (2, o0.kept[2])}[pool]
    pq = orc.token_positions(t, w.num_special, w.grid_h, w.grid_w)[row]
    pk = orc.token_positions(frame, w.num_special, w.grid_h, w.grid_w)[token]
    ang = orc.rope_angles((pq - pk)[None, :], w.head_dim, w.rope_base)
    qf = frames[t][0].double().numpy()
    needle = 3.0 * orc.rotate_pairs(qf[row][None, :, :], ang)[0, h]
    target = torch.linspace(-2, 2, w.head_dim).to(torch.bfloat16)
    frames[frame][1][token, h] = torch.from_numpy(needle).to(torch.bfloat16)
    frames[frame][2][token, h] = target
    _, outs = _run_custom(w, frames, initial_free=gi.initial_free_list(w))
    got = outs[t][row, h].double().cpu()
    assert torch.allclose(got, target.double(), atol=2e-2)
    o = make_oracle(w, source=_custom_source(frames))
    for f in range(t + 1):
        o.append(f)
    check_attention(_np(outs[t]), o.attend(t), f"needle {pool}")


def test_q_rot_may_alias_q():
    w = gi.workload("tiny")
    frames = {t: gi.draw_frame(w, t) for t in range(w.frames)}
    _, ref = _run_custom(w, frames)
    cache = gca.GcaCache(gca.config_for(w))
    out = torch.empty_like(frames[0][0]).cuda()
    for t in range(w.frames):
        q, k, v = (x.cuda() for x in frames[t])
        cache.append_frame(t, q, k, v, q)  # rotate in place
        cache.attend(t, q, out)
        torch.cuda.synchronize()
        assert torch.equal(out, ref[t])


def test_two_caches_on_two_streams_match_sequential():
    w = gi.workload("w16_320").replace(frames=40, max_frames=40)
    ring = device_ring(w)
    seq = []
    for rep in range(2):
        cache = gca.GcaCache(gca.config_for(w, rope_base=1e4 * (rep + 1)))
        q_rot, out = _bufs(w)
        for t in range(w.frames):
            q, k, v = ring[t % w.ring]
            cache.append_frame(t, q, k, v, q_rot)
            cache.attend(t, q_rot, out)
        torch.cuda.synchronize()
        seq.append(out.clone())
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    caches = [gca.GcaCache(gca.config_for(w, rope_base=1e4 * (r + 1)), stream=streams[r])
              for r in range(2)]
    bufs = [_bufs(w) for _ in range(2)]
    for t in range(w.frames):
        for r in range(2):
            with torch.cuda.stream(streams[r]):
                q, k, v = ring[t % w.ring]
                caches[r].append_frame(t, q, k, v, bufs[r][0], stream=streams[r])
                caches[r].attend(t, bufs[r][0], bufs[r][1], stream=streams[r])
    torch.cuda.synchronize()
    for r in range(2):
        assert torch.equal(bufs[r][1], seq[r])


def test_host_detected_errors():
    w = gi.workload("tiny")
    ring = device_ring(w)
    q_rot, out = _bufs(w)
    cache = gca.GcaCache(gca.config_for(w.replace(num_pages=12)))
    q, k, v = ring[0]
    with pytest.raises(gca.GcaError) as e:
        cache.append_frame(1, q, k, v, q_rot)
    assert e.value.status == -3
    with pytest.raises(gca.GcaError) as e:
        cache.attend(0, q_rot, out)
    assert e.value.status == -3
    # q_rot_out may be q itself, but no other overlap with q, k or v: a shifted overlap would
    # let one thread overwrite a chunk another has yet to read
    big = torch.empty((3 * w.tokens_per_frame + 8, w.num_heads, w.head_dim),
                      dtype=torch.bfloat16, device="cuda")
    T = w.tokens_per_frame
    qb, kb = big[:T], big[T:2 * T]
    for bad in (big[1:T + 1], big[T:2 * T], big[T - 1:2 * T - 1]):
        with pytest.raises(gca.GcaError) as e:
            cache.append_frame(0, qb, kb, v, bad)
        assert e.value.status == -1
    assert cache.state().frames_appended == 0
    cache.append_frame(0, q, k, v, q_rot)
    cache.append_frame(1, q, k, v, q_rot)
    # 12 pages, 5 per frame: the third frame does not fit
    with pytest.raises(gca.GcaError) as e:
        cache.append_frame(2, q, k, v, q_rot)
    assert e.value.status == -2
    assert cache.state().frames_appended == 2
    assert cache.check() == 0


def test_bad_initial_free_list_is_reported():
    w = gi.workload("tiny")
    free = torch.zeros(w.num_pages, dtype=torch.int32)  # not a permutation
    cache = gca.GcaCache(gca.config_for(w), initial_free=free)
    assert cache.check() == -6
    assert cache.state().device_error & 0x4
    # the sticky word makes later attentions no-ops: no output is written
    q, k, v = (x.cuda() for x in gi.draw_frame(w, 0))
    q_rot = torch.empty_like(q)
    out = torch.full_like(q, 3.0)
    cache.append_frame(0, q, k, v, q_rot)
    cache.attend(0, q_rot, out)
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())
    assert cache.check() == -6
