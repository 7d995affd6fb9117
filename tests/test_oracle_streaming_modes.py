"""Pins of the oracle's streaming modes beyond the plain stream, each against something other
than the code under test.

Keyframe-only caching (reading R11): transient append, rollback and the keyframe stream driver.

- a dense brute force that restates the visibility rule in video-frame terms (keys built from
  the raw inputs, an explicit mask, torch's scaled_dot_product_attention in fp64);
- the keyframe-only book: interleaving transient appends and rollbacks must leave the
  allocator bit-identical to a book that never saw the non-keyframes;
- a special case that reduces to the plain (already pinned) path: a transient frame sees
  exactly what a normal frame of a cache with one more window frame sees;
- interval 1, which is the plain stream;
- the closed form of the transient frame's visible-key count, and brute force over the book.

Scale-frame prefill (reading R12): a dense unmasked SDPA brute force over the concatenated
frames; the last scale frame's rows equal its causal rows (same key set); an earlier frame's
rows change with a later frame's keys (bidirectional), its causal rows do not.
"""
import random

import numpy as np
import pytest
import torch

import oracle as orc


def make_oracle(*, H=2, D=64, ps=16, gh=3, gw=4, S=2, A=1, W=2, K=3, base=10000.0, seed=11,
                num_pages=96, free=None):
    T = S + gh * gw

    def src(g):
        gen = torch.Generator().manual_seed(seed * 1009 + g)
        return tuple(torch.randn(T, H, D, generator=gen).to(torch.bfloat16) for _ in range(3))

    return orc.GcaOracle(num_heads=H, head_dim=D, page_size=ps, grid_h=gh, grid_w=gw,
                         num_special=S, anchor_frames=A, window_frames=W, keep_tokens=K,
                         rope_base=base, initial_free=free or list(range(num_pages)),
                         frame_source=src)


def _rotated(o, g, which):
    """q or k of video frame g, rotated at time position g (from the raw inputs)."""
    x = o.source(g)[which].float().numpy().astype(np.float64)
    pos = orc.token_positions(g, o.S, o.gh, o.gw)
    return orc.rotate_pairs(x, orc.rope_angles(pos, o.D, o.base))


def dense_keyframe_attention(o, g, interval):
    """Brute force in video-frame terms. The cache holds the keyframes before g; the i-th of
    them is cache frame i. Frame g (keyframe or not) sees: every token of the first A kept
    frames; every token of the most recent kept frames -- W of them counting g itself when g
    is a keyframe, W plus g itself when it is not (nothing was evicted before its attention);
    only the kept tokens of the older ones; and every token of itself."""
    keyframes = [f for f in range(g) if f % interval == 0]
    frames = keyframes + [g]
    n_prev = len(keyframes)
    recent = o.W - 1 if g % interval == 0 else o.W
    kept = set(o.kept)
    vis = []
    for i, f in enumerate(frames):
        for tok in range(o.T):
            if f == g or i < o.A or i >= n_prev - recent:
                vis.append(True)
            else:
                vis.append(tok in kept)
    vis = np.asarray(vis)
    q = torch.from_numpy(_rotated(o, g, 0))
    k = torch.from_numpy(np.concatenate([_rotated(o, f, 1) for f in frames]))
    v = torch.from_numpy(np.concatenate([o.source(f)[2].float().numpy() for f in frames])
                         .astype(np.float64))
    mask = torch.from_numpy(np.broadcast_to(vis[None, :], (o.T, len(vis))).copy())
    out = torch.nn.functional.scaled_dot_product_attention(
        q.permute(1, 0, 2), k.permute(1, 0, 2), v.permute(1, 0, 2), attn_mask=mask)
    return out.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("A,W,K,N", [(1, 2, 3, 3), (0, 3, 0, 2), (2, 2, 4, 4), (1, 1, 3, 2),
                                     (1, 3, 3, 5)])
def test_keyframe_stream_matches_dense_masked_sdpa(A, W, K, N):
    o = make_oracle(A=A, W=W, K=K, S=4 if K == 4 else 2)
    checked = []

    def on_frame(g, slot, key):
        np.testing.assert_allclose(o.attend(slot), dense_keyframe_attention(o, g, N), rtol=0,
                                   atol=1e-12, err_msg=f"video frame {g} (slot {slot})")
        checked.append(key)

    kept = orc.keyframe_stream(o, 4 * N * (A + W) + 3, N, on_frame)
    assert kept == list(range(len(kept)))
    assert True in checked and False in checked


def test_rollback_restores_the_allocator_exactly():
    rng = random.Random(5)
    free = list(range(60))
    rng.shuffle(free)
    kw = dict(T=14, page_size=4, anchor_frames=1, window_frames=3, kept=[0, 5, 9],
              initial_free=free)
    plain, mixed = orc.CacheBook(**kw), orc.CacheBook(**kw)
    for s in range(25):
        for _ in range(rng.randrange(4)):  # non-keyframes between keyframes
            head = list(mixed.alloc.free)[:mixed.ppf]
            traj_before = list(mixed.traj_tokens)
            live_before = sorted(mixed.frame_pages)
            mixed.append(s, transient=True)
            assert mixed.frame_pages[s] == head  # the pages the next keyframe will take
            assert mixed.traj_tokens == traj_before  # nothing evicted ...
            assert sorted(mixed.frame_pages) == live_before + [s]  # ... every frame still live
            mixed.rollback(s)
        plain.append(s)
        mixed.append(s)
        assert list(mixed.alloc.free) == list(plain.alloc.free)
        assert mixed.frame_pages == plain.frame_pages
        assert mixed.traj_pages == plain.traj_pages
        assert mixed.traj_tokens == plain.traj_tokens
    with pytest.raises(ValueError):
        plain.rollback(24)  # a kept frame does not roll back
    mixed.append(25, transient=True)
    with pytest.raises(ValueError):
        mixed.append(26)  # a transient frame rolls back before the next append


@pytest.mark.parametrize("A,W,K", [(0, 2, 0), (1, 2, 3), (2, 3, 3), (1, 1, 3)])
def test_transient_frame_sees_what_a_one_wider_window_sees(A, W, K):
    o1 = make_oracle(A=A, W=W, K=K)
    o2 = make_oracle(A=A, W=W + 1, K=K)
    for s in range(9):
        o2.append(s)
        o1.append(s, transient=True)
        np.testing.assert_array_equal(o1.attend(s), o2.attend(s))
        o1.rollback(s)
        o1.append(s)


def test_interval_one_is_the_plain_stream():
    a, b = make_oracle(A=1, W=2, K=3), make_oracle(A=1, W=2, K=3)
    outs = []
    orc.keyframe_stream(a, 7, 1, lambda g, s, key: outs.append(a.attend(s)))
    for t in range(7):
        b.append(t)
        np.testing.assert_array_equal(outs[t], b.attend(t))
    assert list(a.book.alloc.free) == list(b.book.alloc.free)


def test_keyframe_slots_rotate_at_their_video_index():
    o = make_oracle(A=1, W=2, K=3)
    ref = make_oracle(A=1, W=2, K=3)
    seen = []

    def on_frame(g, slot, key):
        np.testing.assert_array_equal(o.q_rot(slot), ref.q_rot(g))
        np.testing.assert_array_equal(o.k_rot(slot), ref.k_rot(g))
        seen.append((g, slot))

    orc.keyframe_stream(o, 10, 4, on_frame)
    assert seen[5] == (5, 2)  # video frame 5 sits transiently in slot 2 (after keyframes 0, 4)
    assert o.positions([1], [0])[0, 0] == 4  # keyframe 4 holds slot 1


@pytest.mark.parametrize("A,W", [(0, 1), (1, 2), (2, 5), (1, 16)])
def test_transient_visible_count_closed_form(A, W):
    T, K = 14, 3
    kept = [0, 5, 9]
    for s in range(40):
        if s < A:
            want = (s + 1) * T
        else:
            want = A * T + min(W + 1, s + 1 - A) * T + max(0, s - A - W) * K
        assert orc.visible_key_count(s, A, W, T, K, transient=True) == want
        # brute force over the book: the live frames and the trajectory after the append
        book = orc.CacheBook(T=T, page_size=4, anchor_frames=A, window_frames=W, kept=kept,
                             initial_free=list(range(400)))
        for t in range(s):
            book.append(t)
        book.append(s, transient=True)
        anchor, window, evicted = orc.pool_frames(s, A, W, transient=True)
        assert sorted(book.frame_pages) == anchor + window
        assert sorted({e for e, _ in book.traj_tokens}) == evicted


# ---------------------------------------------------------------- scale-frame prefill (R12)

def dense_prefill(o, n):
    """Brute force: the n*T queries of frames 0..n-1 against every token of those frames,
    no mask, torch's scaled_dot_product_attention in fp64 (keys from the raw inputs)."""
    q = torch.from_numpy(np.concatenate([_rotated(o, f, 0) for f in range(n)]))
    k = torch.from_numpy(np.concatenate([_rotated(o, f, 1) for f in range(n)]))
    v = torch.from_numpy(np.concatenate([o.source(f)[2].float().numpy() for f in range(n)])
                         .astype(np.float64))
    out = torch.nn.functional.scaled_dot_product_attention(
        q.permute(1, 0, 2), k.permute(1, 0, 2), v.permute(1, 0, 2))
    return out.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("n,A", [(1, 1), (3, 4), (4, 4), (2, 2)])
def test_prefill_matches_dense_sdpa(n, A):
    o = make_oracle(A=A, W=2, K=3)
    for t in range(n):
        o.append(t)
    np.testing.assert_allclose(o.attend_prefill(n), dense_prefill(o, n), rtol=0, atol=1e-12)
    rows = np.array([0, o.T - 1, o.T, n * o.T - 1])
    rows = rows[rows < n * o.T]
    np.testing.assert_allclose(o.attend_prefill(n, rows), o.attend_prefill(n)[rows], rtol=0,
                               atol=1e-13)  # BLAS blocks by shape: equal to rounding


def test_prefill_last_frame_rows_are_the_causal_rows():
    o = make_oracle(A=4, W=2, K=3)
    for t in range(4):
        o.append(t)
    last = o.attend_prefill(4)[3 * o.T:]
    np.testing.assert_allclose(last, o.attend(3), rtol=0, atol=1e-13)


def test_prefill_is_bidirectional():
    # changing a later scale frame changes an earlier frame's rows (it would not, causally)
    base = make_oracle(A=3, W=2, K=3)
    other = make_oracle(A=3, W=2, K=3)
    k2 = torch.randn(other.T, other.H, other.D).to(torch.bfloat16)
    src = other.source
    other.source = lambda g: (src(g)[0], k2, src(g)[2]) if g == 2 else src(g)
    for o in (base, other):
        for t in range(3):
            o.append(t)
    a, b = base.attend_prefill(3), other.attend_prefill(3)
    assert np.abs(a[:base.T] - b[:base.T]).max() > 1e-6  # frame 0 sees frame 2's keys
    np.testing.assert_array_equal(base.attend(0), other.attend(0))  # causally it does not
    with pytest.raises(ValueError):
        base.attend_prefill(2)  # three frames are appended


# ------------------------------------------------- patch-free cache (causal camera head, R13)

def test_camera_token_cache_is_causal_attention_over_all_camera_tokens():
    """One camera token per frame and K = 1: every evicted frame keeps its token, so frame t
    sees the camera tokens of all frames 0..t. Brute force: torch SDPA over the rotated camera
    tokens of frames 0..t (rotated only in time: the token sits at (t, 0, 0))."""
    o = make_oracle(H=4, gh=0, gw=0, S=1, A=1, W=3, K=1, base=500.0)
    for t in range(12):
        o.append(t)
        assert orc.visible_key_count(t, o.A, o.W, o.T, o.K) == t + 1
        q = torch.from_numpy(_rotated(o, t, 0))
        k = torch.from_numpy(np.concatenate([_rotated(o, f, 1) for f in range(t + 1)]))
        v = torch.from_numpy(np.concatenate([o.source(f)[2].float().numpy()
                                             for f in range(t + 1)]).astype(np.float64))
        ref = torch.nn.functional.scaled_dot_product_attention(
            q.permute(1, 0, 2), k.permute(1, 0, 2), v.permute(1, 0, 2)).permute(1, 0, 2)
        np.testing.assert_allclose(o.attend(t), ref.numpy(), rtol=0, atol=1e-12)
    # frame 0 sees one key: the output is its v exactly
    o0 = make_oracle(H=4, gh=0, gw=0, S=1, A=1, W=3, K=1)
    o0.append(0)
    np.testing.assert_array_equal(o0.attend(0), o0.raw(0)[2])
    assert orc.token_positions(7, 1, 0, 0).tolist() == [[7, 0, 0]]


# ------------------------------------------------------------- windowed restart (R14)

@pytest.mark.parametrize("total,N,V", [(500, 128, 8), (128, 128, 8), (129, 128, 8), (10, 4, 1),
                                       (7, 7, 0), (1, 3, 2), (30, 5, 4)])
def test_windowed_schedule_closed_form(total, N, V):
    sched = orc.windowed_frames(total, N, V)
    n_windows = 1 if total <= N else 1 + -(-(total - N) // (N - V))
    assert sched[-1][0] == n_windows - 1
    assert all(0 <= loc < N for _, _, loc in sched)  # RoPE positions stay in the window
    assert sorted({g for _, g, _ in sched}) == list(range(total))  # every frame, in order
    assert len(sched) == total + V * (n_windows - 1)  # overlap frames run twice
    for w in range(1, n_windows):
        prev = [g for ww, g, _ in sched if ww == w - 1]
        cur = [g for ww, g, _ in sched if ww == w]
        assert prev[-V:] == cur[:V] if V else not set(prev) & set(cur)
        assert cur[0] == w * (N - V)


def test_windowed_stream_is_a_fresh_stream_per_window():
    """Each window's attention equals a new oracle streaming that window's frames from local
    index 0 (frame g at local position g - start, so its RoPE time is local)."""
    A, W, K, N, V = 1, 2, 3, 5, 2
    o = make_oracle(A=A, W=W, K=K)
    outs = {}
    for w, g, loc in orc.windowed_frames(12, N, V):
        if loc == 0:
            o.restart()
        o.append(loc, g, rope_pos=loc)
        outs[(w, g)] = o.attend(loc)
    for w in range(4):
        start = w * (N - V)
        ref = make_oracle(A=A, W=W, K=K)
        ref.source = (lambda s0: (lambda t: o.source(t + s0)))(start)
        ref._raw = {}
        for loc in range(min(N, 12 - start)):
            ref.append(loc)
            np.testing.assert_array_equal(outs[(w, start + loc)], ref.attend(loc))
