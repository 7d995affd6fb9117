"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against a closed form, a library routine, brute force on tiny
inputs, an invariant the mathematics fixes, or a number the pages print. A plausible slip in
the oracle (a dropped pool, a wrong sign, index or scale, a transposed operand, a wrong
eviction or allocation order) fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import expit

import gca_inputs as gi
import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def make_oracle(*, H=2, D=64, ps=16, gh=3, gw=4, S=2, A=1, W=2, K=3, base=10000.0,
                seed=7, scale=1.0, free=None, num_pages=64, frames_override=None):
    T = S + gh * gw

    def src(t):
        if frames_override is not None and t in frames_override:
            return frames_override[t]
        g = torch.Generator().manual_seed(seed * 1009 + t)
        return tuple((torch.randn(T, H, D, generator=g) * scale).to(torch.bfloat16)
                     for _ in range(3))

    if free is None:
        free = list(range(num_pages))
    return orc.GcaOracle(num_heads=H, head_dim=D, page_size=ps, grid_h=gh, grid_w=gw,
                         num_special=S, anchor_frames=A, window_frames=W, keep_tokens=K,
                         rope_base=base, initial_free=free, frame_source=src)


def dense_masked_attention(o, t):
    """Brute force: every token of frames 0..t as a key, an explicit [T x N_all] pool mask
    built from the pool rule, and torch's own scaled_dot_product_attention in fp64."""
    T = o.T
    frames = np.repeat(np.arange(t + 1), T)
    tokens = np.tile(np.arange(T), t + 1)
    kept = set(o.kept)
    vis = np.zeros(len(frames), dtype=bool)
    for n, (f, i) in enumerate(zip(frames, tokens)):
        if t < o.A:
            vis[n] = True
        elif f < o.A:
            vis[n] = True
        elif f >= t - o.W + 1:
            vis[n] = True
        else:
            vis[n] = i in kept
    qr = torch.from_numpy(o.q_rot(t))  # [T, H, D]
    ks = torch.from_numpy(np.concatenate([o.k_rot(f) for f in range(t + 1)]))
    vs = torch.from_numpy(np.concatenate([o.raw(f)[2] for f in range(t + 1)]))
    mask = torch.from_numpy(np.broadcast_to(vis[None, :], (T, len(vis))).copy())
    out = torch.nn.functional.scaled_dot_product_attention(
        qr.permute(1, 0, 2), ks.permute(1, 0, 2), vs.permute(1, 0, 2), attn_mask=mask)
    return out.permute(1, 0, 2).numpy()


# ------------------------------------------------------------------ attention definition

@pytest.mark.parametrize("A,W,K", [(a, w, k) for a in (0, 1, 2) for w in (1, 2, 3)
                                   for k in (0, 4, 6)])
def test_oracle_matches_dense_masked_sdpa(A, W, K):
    o = make_oracle(A=A, W=W, K=K, S=4 if K == 4 else 2)
    for t in range(7):
        o.append(t)
        np.testing.assert_allclose(o.attend(t), dense_masked_attention(o, t), rtol=0,
                                   atol=1e-12)


def test_tiny_workload_matches_dense_masked_sdpa():
    w = gi.workload("tiny")
    o = orc.GcaOracle(num_heads=w.num_heads, head_dim=w.head_dim, page_size=w.page_size,
                      grid_h=w.grid_h, grid_w=w.grid_w, num_special=w.num_special,
                      anchor_frames=w.anchor_frames, window_frames=w.window_frames,
                      keep_tokens=w.keep_tokens, rope_base=w.rope_base,
                      initial_free=gi.initial_free_list(w).tolist(),
                      frame_source=lambda t: gi.draw_frame(w, t))
    for t in range(w.frames):
        o.append(t)
        np.testing.assert_allclose(o.attend(t), dense_masked_attention(o, t), rtol=0,
                                   atol=1e-12)


def test_softmax_attention_is_sdpa():
    rng = np.random.default_rng(0)
    q, k, v = rng.standard_normal((5, 64)), rng.standard_normal((37, 64)), rng.standard_normal((37, 64))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])[0]
    np.testing.assert_allclose(orc.softmax_attention(q, k, v), ref.numpy(), rtol=0, atol=1e-13)


def test_single_key_returns_v_exactly():
    o = make_oracle(gh=1, gw=1, S=0, A=0, W=1, K=0)
    for t in range(3):
        o.append(t)
        out = o.attend(t)
        assert np.array_equal(out, o.raw(t)[2])


def test_zero_query_returns_mean_of_visible_v():
    T = 2 + 12
    zero = torch.zeros(T, 2, 64, dtype=torch.bfloat16)
    g = torch.Generator().manual_seed(3)
    frames = {t: (zero, torch.randn(T, 2, 64, generator=g).to(torch.bfloat16),
                  torch.randn(T, 2, 64, generator=g).to(torch.bfloat16)) for t in range(6)}
    o = make_oracle(A=1, W=2, K=3, frames_override=frames)
    kept = orc.kept_token_indices(2, 12, 3)
    for t in range(6):
        o.append(t)
        # visible set by hand: anchor frame 0, frames max(1,t-1)..t, kept tokens of the rest
        rows = [frames[0][2].double()] if t >= 1 else []
        lo = max(1, t - 1) if t >= 1 else 0
        rows += [frames[f][2].double() for f in range(lo, t + 1)]
        rows += [frames[f][2].double()[kept] for f in range(1, lo)]
        mean = torch.cat(rows).mean(dim=0).numpy()
        out = o.attend(t)
        np.testing.assert_allclose(out, np.broadcast_to(mean, out.shape), rtol=0, atol=1e-13)


def test_two_keys_follow_the_logistic_function():
    rng = np.random.default_rng(1)
    for _ in range(20):
        q = rng.standard_normal((1, 64))
        k = rng.standard_normal((2, 64))
        v = rng.standard_normal((2, 64))
        s = (k @ q[0]) / 8.0
        w1 = expit(s[1] - s[0])
        expect = v[0] + w1 * (v[1] - v[0])
        np.testing.assert_allclose(orc.softmax_attention(q, k, v)[0], expect, rtol=0, atol=1e-13)


# ------------------------------------------------------------------ RoPE

def test_rope_band_widths():
    assert orc.rope_band_widths(64) == (24, 20, 20)
    assert orc.rope_band_widths(12) == (4, 4, 4)
    assert sum(orc.rope_band_widths(96)) == 96


def test_rope_is_complex_multiplication():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((9, 3, 64))
    pos = rng.integers(0, 50, size=(9, 3))
    ang = orc.rope_angles(pos, 64, 10000.0)
    out = orc.rotate_pairs(x, ang)
    z = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * ang)[:, None, :]
    np.testing.assert_allclose(out[..., 0::2], z.real, atol=1e-13)
    np.testing.assert_allclose(out[..., 1::2], z.imag, atol=1e-13)


def test_rope_preserves_norm_and_is_identity_at_origin():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((20, 2, 64))
    pos = rng.integers(0, 10000, size=(20, 3))
    out = orc.rotate_pairs(x, orc.rope_angles(pos, 64, 10000.0))
    np.testing.assert_allclose(np.linalg.norm(out, axis=-1), np.linalg.norm(x, axis=-1),
                               rtol=1e-12)
    zero = orc.rotate_pairs(x, orc.rope_angles(np.zeros((20, 3), np.int64), 64, 10000.0))
    assert np.array_equal(zero, x)


@pytest.mark.parametrize("axis", [0, 1, 2])
def test_rope_scores_depend_only_on_relative_offset(axis):
    rng = np.random.default_rng(4 + axis)
    q = rng.standard_normal((1, 1, 64))
    k = rng.standard_normal((1, 1, 64))
    for _ in range(10):
        pq = rng.integers(0, 300, size=(1, 3))
        pk = rng.integers(0, 300, size=(1, 3))
        shift = np.zeros((1, 3), np.int64)
        shift[0, axis] = rng.integers(1, 500)
        dot = lambda a, b: float((orc.rotate_pairs(q, orc.rope_angles(a, 64, 1e4))
                                  * orc.rotate_pairs(k, orc.rope_angles(b, 64, 1e4))).sum())
        assert abs(dot(pq, pk) - dot(pq + shift, pk + shift)) < 1e-10


def test_rope_bands_touch_their_own_dims():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, 1, 64))
    base = orc.rotate_pairs(x, orc.rope_angles(np.array([[3, 2, 5]]), 64, 1e4))
    bands = [(0, 24), (24, 44), (44, 64)]
    for axis, (lo, hi) in enumerate(bands):
        p = np.array([[3, 2, 5]])
        p[0, axis] += 7
        moved = orc.rotate_pairs(x, orc.rope_angles(p, 64, 1e4))
        changed = np.nonzero(np.abs(moved - base)[0, 0] > 1e-12)[0]
        assert changed.min() >= lo and changed.max() < hi


def test_token_positions_row_major_after_special_tokens():
    pos = orc.token_positions(9, 5, 27, 37)
    assert pos.shape == (1004, 3)
    assert (pos[:, 0] == 9).all()
    assert (pos[:5, 1:] == 0).all()
    assert tuple(pos[5]) == (9, 1, 1)
    assert tuple(pos[5 + 36]) == (9, 1, 37)
    assert tuple(pos[5 + 37]) == (9, 2, 1)
    assert tuple(pos[-1]) == (9, 27, 37)


# Angles of the RoPE reading written out by hand (3D RoPE of the GCT page: bands t, y, x of
# 24, 20, 20 dims at head_dim 64; pair j of a band of width d turns by pos * base^(-2j/d)).
# The column of pair j is j in the time band, 12 + j in the y band and 22 + j in the x band.
# Each value is the exponent simplified by hand, e.g. 10000^(-2*1/24) = 10^(-1/3).
ROPE_HAND_VALUES = [
    # (base, (t, y, x), column, angle)
    (10000.0, (7, 3, 11), 0, 7.0),                      # t * 10000^0
    (10000.0, (7, 3, 11), 1, 3.2491121835289450),       # 7 * 10^(-1/3)
    (10000.0, (7, 3, 11), 6, 0.07),                     # 7 * 10000^(-12/24) = 7 * 10^-2
    (10000.0, (7, 3, 11), 11, 7 * 2.1544346900318823e-4),  # 7 * 10^(-11/3)
    (10000.0, (7, 3, 11), 12, 3.0),                     # y * 10000^0
    (10000.0, (7, 3, 11), 15, 0.18928720334405799),     # 3 * 10000^(-6/20) = 3 * 10^(-1.2)
    (10000.0, (7, 3, 11), 17, 0.03),                    # 3 * 10000^(-10/20) = 3 * 10^-2
    (10000.0, (7, 3, 11), 22, 11.0),                    # x * 10000^0
    (10000.0, (7, 3, 11), 24, 1.7433825117072247),      # 11 * 10000^(-4/20) = 11 * 10^(-0.8)
    (10000.0, (7, 3, 11), 31, 0.0027630750746605374),   # 11 * 10000^(-18/20) = 11 * 10^(-3.6)
    (500.0, (7, 3, 11), 6, 0.31304951684997057),        # 7 * 500^(-1/2)
    (500.0, (7, 3, 11), 17, 0.13416407864998738),       # 3 * 500^(-1/2)
    (500.0, (7, 3, 11), 27, 0.49193495504995373),       # 11 * 500^(-1/2)
    (500.0, (7, 3, 11), 3, 7 * 0.21147425268811282),    # 7 * 500^(-1/4)
]


@pytest.mark.parametrize("base,pos,col,angle", ROPE_HAND_VALUES)
def test_rope_angles_match_hand_values(base, pos, col, angle):
    ang = orc.rope_angles(np.array([pos], dtype=np.int64), 64, base)
    assert ang.shape == (1, 32)
    assert abs(ang[0, col] - angle) <= 1e-13 * max(1.0, abs(angle))


def test_rope_rotation_of_a_unit_pair_by_hand():
    # the time-band pair j = 6 of a token at t = 7 turns (1, 0) into (cos 0.07, sin 0.07)
    x = np.zeros((1, 1, 64))
    x[0, 0, 12] = 1.0
    out = orc.rotate_pairs(x, orc.rope_angles(np.array([[7, 3, 11]]), 64, 10000.0))
    assert abs(out[0, 0, 12] - 0.99755100025327959) < 1e-14   # cos(0.07)
    assert abs(out[0, 0, 13] - 0.06994284733753277) < 1e-14   # sin(0.07)
    assert np.count_nonzero(out[0, 0]) == 2


# ------------------------------------------------------------------ pools and kept tokens

def test_kept_tokens_match_the_stride_rule():
    assert orc.kept_token_indices(5, 999, 12) == [0, 1, 2, 3, 4] + [5 + 142 * j for j in range(7)]
    assert orc.kept_token_indices(4, 64, 4) == [0, 1, 2, 3]
    assert orc.kept_token_indices(5, 999, 0) == []


def nk_closed_form(t, A, W, T, K):
    if t < A:
        return (t + 1) * T
    return A * T + min(W, t + 1 - A) * T + max(0, t + 1 - A - W) * K


@pytest.mark.parametrize("name", list(gi.WORKLOADS))
def test_visible_count_closed_form(name):
    w = gi.workload(name)
    T, K = w.tokens_per_frame, w.keep_tokens
    kept = orc.kept_token_indices(w.num_special, w.grid_h * w.grid_w, K)
    for t in list(range(min(w.frames, 80))) + [w.frames - 1]:
        n = orc.visible_key_count(t, w.anchor_frames, w.window_frames, T, K)
        assert n == nk_closed_form(t, w.anchor_frames, w.window_frames, T, K)
        if t < 40 and name in ("tiny", "w16_320"):
            assert len(orc.visible_keys(t, w.anchor_frames, w.window_frames, T, kept)) == n


def test_pool_sizes_at_the_last_frame():
    expect = {"w16_320": (20704, 3636), "w64_1000": (76480, 11220),
              "w32_10k": (152736, 119604), "stack24x4": (12048, 0), "tiny": (216, 12)}
    for name, (nk, traj) in expect.items():
        w = gi.workload(name)
        t = w.frames - 1
        _, _, ev = orc.pool_frames(t, w.anchor_frames, w.window_frames)
        assert len(ev) * w.keep_tokens == traj
        assert orc.visible_key_count(t, w.anchor_frames, w.window_frames,
                                     w.tokens_per_frame, w.keep_tokens) == nk


def test_pages_print_the_shapes():
    facts = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    (wpx, hpx), p = facts["image_width_height"]["value"], facts["patch_size"]["value"]
    gw_, gh_ = wpx // p, hpx // p
    assert (gh_, gw_) == (27, 37) and gh_ * gw_ == 999
    # every 518x378 workload lays its patches out as 27 rows x 37 columns
    for name, wl in gi.WORKLOADS.items():
        if wl.tokens_per_frame == 1004:
            assert (wl.grid_h, wl.grid_w) == (gh_, gw_), name
    w = gi.workload("w16_320")
    assert facts["embed_dim"]["value"] == w.num_heads * w.head_dim
    # per-frame context growth: T tokens (full causal) vs K kept tokens
    ratio = w.tokens_per_frame / w.keep_tokens
    assert abs(ratio - facts["context_growth_reduction"]["value"]) / 80 < 0.1
    lo, hi = facts["training_window_frames"]["value"]
    assert lo <= gi.workload("w16_320").window_frames <= hi
    assert lo <= gi.workload("w64_1000").window_frames <= hi
    ab = facts["abot_window"]["value"]
    s = gi.workload("stack24x4")
    assert s.window_frames == ab["frames"] and s.anchor_frames == 0
    # the 12-frame window sees exactly 11 cached frames plus the current one
    _, win, ev = orc.pool_frames(100, 0, s.window_frames)
    assert len(win) - 1 == ab["cached_previous"] and ev == list(range(0, 89))
    assert gi.workload("w16_320").frames == facts["rope_training_views"]["value"]


def test_causality_and_eviction_perturbations():
    base = make_oracle(A=1, W=2, K=3)
    T = base.T
    for t in range(7):
        base.append(t)
    ref = {t: base.attend(t) for t in range(7)}

    def perturbed(frame, token):
        q, k, v = base.source(frame)
        k, v = k.clone(), v.clone()
        k[token] += 1.0
        v[token] += 1.0
        return make_oracle(A=1, W=2, K=3, frames_override={frame: (q, k, v)})

    # a later frame never changes an earlier output
    o = perturbed(4, 0)
    for t in range(7):
        o.append(t)
    for t in range(4):
        assert np.array_equal(o.attend(t), ref[t])
    # a dropped token of an evicted frame: frame 1 leaves the window at t=3
    dropped = [i for i in range(T) if i not in base.kept][0]
    o = perturbed(1, dropped)
    for t in range(7):
        o.append(t)
    assert not np.array_equal(o.attend(2), ref[2])
    for t in range(3, 7):
        assert np.array_equal(o.attend(t), ref[t])
    # a kept token keeps influencing every later frame
    o = perturbed(1, base.kept[-1])
    for t in range(7):
        o.append(t)
    for t in range(3, 7):
        assert not np.allclose(o.attend(t), ref[t], atol=1e-6)


@pytest.mark.parametrize("pool", ["anchor", "window", "trajectory"])
def test_needles_in_each_pool(pool):
    o0 = make_oracle(A=1, W=2, K=3, S=2)
    T = o0.T
    t, row, h = 5, 7, 1
    frame, token = {"anchor": (0, 9), "window": (4, 11), "trajectory": (2, o0.kept[1])}[pool]
    q, k, v = (x.clone() for x in o0.source(t))
    qf = q.double().numpy()
    # key = c * R(p_q - p_k) q so that after both rotations it lines up with the query
    pq = orc.token_positions(t, 2, 3, 4)[row]
    pk = orc.token_positions(frame, 2, 3, 4)[token]
    ang = orc.rope_angles((pq - pk)[None, :], 64, 1e4)
    needle = 4.0 * orc.rotate_pairs(qf[row][None, :, :], ang)[0]
    fq, fk, fv = (x.clone() for x in o0.source(frame))
    if frame == t:
        fq = q
    fk[token, h] = torch.from_numpy(needle[h]).to(torch.bfloat16)
    fv[token, h] = torch.linspace(-3, 3, 64).to(torch.bfloat16)
    o = make_oracle(A=1, W=2, K=3, S=2, frames_override={frame: (fq, fk, fv)})
    for f in range(t + 1):
        o.append(f)
    out = o.attend(t, rows=[row])[0, h]
    np.testing.assert_allclose(out, torch.linspace(-3, 3, 64).to(torch.bfloat16).double().numpy(),
                               atol=1e-3)


# ------------------------------------------------------------------ allocator

def test_fifo_order_on_a_small_stream():
    # T = 32 -> 2 pages per frame; A = 0, W = 1, K = 0: each step frees the previous frame
    book = orc.CacheBook(T=32, page_size=16, anchor_frames=0, window_frames=1, kept=[],
                         initial_free=range(6))
    book.append(0)
    assert book.frame_pages[0] == [0, 1] and list(book.alloc.free) == [2, 3, 4, 5]
    book.append(1)
    assert book.frame_pages[1] == [2, 3] and list(book.alloc.free) == [4, 5, 0, 1]
    assert book.slot_map[:3] == [32, 33, 34] and book.slot_map[16] == 48
    book.append(2)
    assert book.frame_pages[2] == [4, 5] and list(book.alloc.free) == [0, 1, 2, 3]


def test_trajectory_pops_after_the_frame_pages():
    # T = 20 -> 2 pages, last page holds 4 slots. A = 1, W = 1, K = 3.
    book = orc.CacheBook(T=20, page_size=16, anchor_frames=1, window_frames=1, kept=[0, 1, 2],
                         initial_free=range(12))
    book.append(0)  # anchor [0,1]
    book.append(1)  # [2,3]
    book.append(2)  # [4,5]; evict 1: traj page 6, then push 2,3
    assert book.frame_pages[2] == [4, 5]
    assert book.traj_pages == [6] and book.traj_len == 3
    assert list(book.alloc.free) == [7, 8, 9, 10, 11, 2, 3]
    for t in range(3, 7):
        book.append(t)
    # 5 evictions x 3 tokens = 15 tokens -> still one page; the 6th eviction needs a second
    assert book.traj_pages == [6] and book.traj_len == 15
    book.append(7)
    assert len(book.traj_pages) == 2 and book.traj_len == 18


@pytest.mark.parametrize("name", ["tiny", "w16_320", "w64_1000", "stack24x4"])
def test_allocator_conserves_pages(name):
    w = gi.workload(name)
    kept = orc.kept_token_indices(w.num_special, w.grid_h * w.grid_w, w.keep_tokens)
    free0 = gi.initial_free_list(w).tolist()
    book = orc.CacheBook(T=w.tokens_per_frame, page_size=w.page_size,
                         anchor_frames=w.anchor_frames, window_frames=w.window_frames,
                         kept=kept, initial_free=free0)
    ppf = -(-w.tokens_per_frame // w.page_size)
    frames = w.frames if name != "stack24x4" else 60
    for t in range(frames):
        book.append(t)
        used = [p for r in book.frame_pages.values() for p in r] + book.traj_pages
        assert len(set(used)) == len(used)
        assert sorted(used + list(book.alloc.free)) == list(range(w.num_pages))
        _, win, ev = orc.pool_frames(t, w.anchor_frames, w.window_frames)
        live = min(t + 1, w.anchor_frames) + (len(win) if t >= w.anchor_frames else 0)
        assert book.pages_in_use() == ppf * live + -(-book.traj_len // w.page_size)
        assert book.traj_len == len(ev) * w.keep_tokens
    book.reset()
    assert list(book.alloc.free) == free0 and book.frames == 0


def test_long_stream_trajectory_size():
    w = gi.workload("w32_10k")
    kept = orc.kept_token_indices(w.num_special, w.grid_h * w.grid_w, w.keep_tokens)
    book = orc.CacheBook(T=w.tokens_per_frame, page_size=w.page_size, anchor_frames=1,
                         window_frames=32, kept=kept, initial_free=range(w.num_pages))
    for t in range(w.frames):
        book.append(t)
    assert book.traj_len == 119604
    assert len(book.traj_pages) == 7476
    assert book.pages_in_use() == 63 * 33 + 7476 <= w.num_pages


def test_out_of_pages():
    book = orc.CacheBook(T=32, page_size=16, anchor_frames=1, window_frames=1, kept=[],
                         initial_free=range(3))
    book.append(0)
    with pytest.raises(orc.OutOfPages):
        book.append(1)


def test_page_permutation_does_not_change_attention():
    outs = []
    for seed in (None, 1, 2):
        free = list(range(64))
        if seed is not None:
            free = np.random.default_rng(seed).permutation(64).tolist()
        o = make_oracle(A=1, W=2, K=3, free=free)
        for t in range(6):
            o.append(t)
        outs.append(o.attend(5))
        if seed is not None:
            assert o.book.frame_pages[5] != list(range(5 * 2, 5 * 2 + 2))
    assert all(np.array_equal(outs[0], x) for x in outs[1:])
